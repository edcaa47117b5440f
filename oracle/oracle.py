"""fp64 CPU oracle for the Gated DeltaNet layer -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` import this module.  The product package never imports it and
shares no code with it.  The arithmetic lives in ``gdn_oracle.c`` (plain C,
fp64, OpenMP over (sequence, value head)); this file only builds that library
with gcc and marshals numpy arrays into it.

All floating-point inputs are decoded to float64 exactly (bf16 and fp32 values
are exactly representable), so the oracle sees the very values the GPU path
reads.  Outputs are float64 and are never rounded here.

See ``gdn_oracle.c`` for what each function computes and which page passage
it follows.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "gdn_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

_dbl_p = ctypes.POINTER(ctypes.c_double)
_i32_p = ctypes.POINTER(ctypes.c_int32)


class _Cfg(ctypes.Structure):
    _fields_ = [
        ("HK", ctypes.c_int32),
        ("HV", ctypes.c_int32),
        ("dk", ctypes.c_int32),
        ("dv", ctypes.c_int32),
        ("K", ctypes.c_int32),
        ("scale", ctypes.c_double),
        ("eps", ctypes.c_double),
    ]


@dataclass(frozen=True)
class OracleCfg:
    HK: int
    HV: int
    dk: int
    dv: int
    K: int = 4
    scale: float = 0.0  # <= 0 -> 1/sqrt(dk)
    eps: float = 1e-6

    @property
    def conv_dim(self) -> int:
        return 2 * self.HK * self.dk + self.HV * self.dv

    def _c(self) -> _Cfg:
        return _Cfg(self.HK, self.HV, self.dk, self.dv, self.K, self.scale, self.eps)


def build(force: bool = False) -> str:
    """Compile gdn_oracle.c into liboracle.so next to it (gcc, -O3, OpenMP).

    GDN_ORACLE_LIB, when set, names an already built library to load instead
    (the mutation tests use it to load deliberately broken copies)."""
    override = os.environ.get("GDN_ORACLE_LIB")
    if override:
        return override
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O3", "-march=native", "-fopenmp", "-fPIC", "-shared", "-std=c11", "-o", tmp, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


def _L():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        for name in ("ora_gate_g", "ora_gate_beta", "ora_softplus_exported"):
            getattr(lib, name).restype = ctypes.c_double
        lib.ora_gate_g.argtypes = [ctypes.c_double] * 3
        lib.ora_gate_beta.argtypes = [ctypes.c_double]
        lib.ora_softplus_exported.argtypes = [ctypes.c_double]
        _lib = lib
    return _lib


def _f64(x) -> np.ndarray:
    """Exact float64 copy of a numpy array or a CPU torch tensor (bf16 included)."""
    if x is None:
        return None
    if hasattr(x, "detach"):  # torch tensor
        import torch

        x = x.detach().to("cpu")
        if x.dtype != torch.float64:
            x = x.to(torch.float64)
        return np.ascontiguousarray(x.numpy())
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _i32(x) -> np.ndarray:
    if x is None:
        return None
    if hasattr(x, "detach"):
        x = x.detach().to("cpu").numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.int32))


def _p(a, kind=_dbl_p):
    return None if a is None else a.ctypes.data_as(kind)


# ---------------------------------------------------------------------------
# single steps
# ---------------------------------------------------------------------------


def num_threads() -> int:
    """OpenMP threads the layer functions run on."""
    return int(_L().ora_num_threads())


def gate_g(A_log: float, a: float, dt_bias: float) -> float:
    return _L().ora_gate_g(float(A_log), float(a), float(dt_bias))


def gate_beta(b: float) -> float:
    return _L().ora_gate_beta(float(b))


def softplus(x: float) -> float:
    return _L().ora_softplus_exported(float(x))


def l2norm(x, eps: float = 1e-6) -> np.ndarray:
    y = _f64(x).copy()
    _L().ora_l2norm(_p(y), ctypes.c_int(y.size), ctypes.c_double(eps))
    return y


def conv_silu(x, w, hist=None, bias=None) -> np.ndarray:
    """x: [L, nch] raw rows; w: [nch, K]; hist: [nch, K-1] or None (zeros)."""
    x, w, hist, bias = _f64(x), _f64(w), _f64(hist), _f64(bias)
    L, nch = x.shape
    K = w.shape[1]
    y = np.zeros((L, nch))
    _L().ora_conv_silu(
        ctypes.c_int(L), ctypes.c_int(nch), ctypes.c_int(K), _p(x), ctypes.c_int64(nch), _p(hist), _p(w),
        _p(bias), _p(y),
    )
    return y


def core_recurrent(q, k, v, g, beta, S0, scale: float, return_states: bool = False):
    """Token-by-token gated delta rule for one head.  Returns (o [L,dv], S [dk,dv][, states])."""
    q, k, v, g, beta = map(_f64, (q, k, v, g, beta))
    S = _f64(S0).copy()
    L, dk = q.shape
    dv = v.shape[1]
    o = np.zeros((L, dv))
    st = np.zeros((L, dk, dv)) if return_states else None
    _L().ora_core_recurrent(
        ctypes.c_int(L), ctypes.c_int(dk), ctypes.c_int(dv), _p(q), _p(k), _p(v), _p(g), _p(beta),
        ctypes.c_double(scale), _p(S), _p(o), _p(st),
    )
    return (o, S, st) if return_states else (o, S)


def core_chunked(q, k, v, g, beta, S0, scale: float, chunk: int):
    q, k, v, g, beta = map(_f64, (q, k, v, g, beta))
    S = _f64(S0).copy()
    L, dk = q.shape
    dv = v.shape[1]
    o = np.zeros((L, dv))
    _L().ora_core_chunked(
        ctypes.c_int(L), ctypes.c_int(dk), ctypes.c_int(dv), _p(q), _p(k), _p(v), _p(g), _p(beta),
        ctypes.c_double(scale), ctypes.c_int(chunk), _p(S), _p(o),
    )
    return o, S


def core_bruteforce(q, k, v, g, beta, S0, scale: float):
    """Explicit product form.  Returns (o, S_stepwise, S_closed_sum)."""
    q, k, v, g, beta, S0 = map(_f64, (q, k, v, g, beta, S0))
    L, dk = q.shape
    dv = v.shape[1]
    o = np.zeros((L, dv))
    S1 = np.zeros((dk, dv))
    S2 = np.zeros((dk, dv))
    _L().ora_core_bruteforce(
        ctypes.c_int(L), ctypes.c_int(dk), ctypes.c_int(dv), _p(q), _p(k), _p(v), _p(g), _p(beta),
        ctypes.c_double(scale), _p(S0), _p(S1), _p(S2), _p(o),
    )
    return o, S1, S2


# ---------------------------------------------------------------------------
# the layer
# ---------------------------------------------------------------------------


def _layer_args(cfg: OracleCfg, params: dict, x, a, b):
    A_log = _f64(params["A_log"])
    dt_bias = _f64(params["dt_bias"])
    conv_w = _f64(params["conv_w"])
    conv_b = _f64(params.get("conv_b"))
    assert conv_w.shape == (cfg.conv_dim, cfg.K)
    return A_log, dt_bias, conv_w, conv_b, _f64(x), _f64(a), _f64(b)


def extend(cfg: OracleCfg, params: dict, x, a, b, cu_seqlens, state_indices, conv_state, ssm_state,
           has_initial_state=None, head_mask=None, chunk: int = 0):
    """Packed-varlen layer.  Returns (out [T,HV,dv], conv_state, ssm_state) as new float64 arrays.

    conv_state: [P, conv_dim, K-1]; ssm_state: [P, HV, dk, dv] (copied, not modified).
    chunk > 0 evaluates the chunked WY form instead of the token-by-token rule.
    head_mask: optional [HV] of 0/1 restricting which heads are computed
    (token-by-token form only); other heads' outputs are zero.
    """
    A_log, dt_bias, conv_w, conv_b, x, a, b = _layer_args(cfg, params, x, a, b)
    cu = _i32(cu_seqlens)
    slots = _i32(state_indices)
    hi = _i32(has_initial_state)
    hm = _i32(head_mask)
    cs = _f64(conv_state).copy()
    ss = _f64(ssm_state).copy()
    N = len(slots)
    T = int(cu[-1])
    P = cs.shape[0]
    out = np.zeros((T, cfg.HV, cfg.dv))
    c = cfg._c()
    if chunk > 0:
        assert hm is None
        rc = _L().ora_extend_chunked(
            ctypes.byref(c), _p(A_log), _p(dt_bias), _p(conv_w), _p(conv_b), _p(x), _p(a), _p(b),
            _p(cu, _i32_p), ctypes.c_int(N), _p(slots, _i32_p), _p(hi, _i32_p), _p(cs), _p(ss), ctypes.c_int(P),
            _p(out), ctypes.c_int(chunk),
        )
    else:
        rc = _L().ora_extend(
            ctypes.byref(c), _p(A_log), _p(dt_bias), _p(conv_w), _p(conv_b), _p(x), _p(a), _p(b),
            _p(cu, _i32_p), ctypes.c_int(N), _p(slots, _i32_p), _p(hi, _i32_p), _p(cs), _p(ss), ctypes.c_int(P),
            _p(out), _p(hm, _i32_p),
        )
    if rc != 0:
        raise ValueError(f"oracle extend rejected its arguments (code {rc})")
    return out, cs, ss


def decode(cfg: OracleCfg, params: dict, x, a, b, state_indices, conv_state, ssm_state):
    """One token per request.  Returns (out [B,HV,dv], conv_state, ssm_state)."""
    A_log, dt_bias, conv_w, conv_b, x, a, b = _layer_args(cfg, params, x, a, b)
    slots = _i32(state_indices)
    cs = _f64(conv_state).copy()
    ss = _f64(ssm_state).copy()
    B = len(slots)
    out = np.zeros((B, cfg.HV, cfg.dv))
    c = cfg._c()
    rc = _L().ora_decode(
        ctypes.byref(c), _p(A_log), _p(dt_bias), _p(conv_w), _p(conv_b), _p(x), _p(a), _p(b), ctypes.c_int(B),
        _p(slots, _i32_p), _p(cs), _p(ss), ctypes.c_int(cs.shape[0]), _p(out),
    )
    if rc != 0:
        raise ValueError(f"oracle decode rejected its arguments (code {rc})")
    return out, cs, ss


def verify(cfg: OracleCfg, params: dict, x, a, b, state_indices, D: int, conv_state, ssm_state,
           want_conv_ckpt: bool = True):
    """D draft tokens per request, pools read only.

    Returns (out [B*D,HV,dv], ckpt [B,D,HV,dk,dv], conv_ckpt [B,D,conv_dim,K-1] or None).
    """
    A_log, dt_bias, conv_w, conv_b, x, a, b = _layer_args(cfg, params, x, a, b)
    slots = _i32(state_indices)
    cs = _f64(conv_state)
    ss = _f64(ssm_state)
    B = len(slots)
    out = np.zeros((B * D, cfg.HV, cfg.dv))
    ckpt = np.zeros((B, D, cfg.HV, cfg.dk, cfg.dv))
    cck = np.zeros((B, D, cfg.conv_dim, cfg.K - 1)) if want_conv_ckpt else None
    c = cfg._c()
    rc = _L().ora_verify(
        ctypes.byref(c), _p(A_log), _p(dt_bias), _p(conv_w), _p(conv_b), _p(x), _p(a), _p(b), ctypes.c_int(B),
        ctypes.c_int(D), _p(slots, _i32_p), _p(cs), _p(ss), ctypes.c_int(cs.shape[0]), _p(ckpt), _p(cck), _p(out),
    )
    if rc != 0:
        raise ValueError(f"oracle verify rejected its arguments (code {rc})")
    return out, ckpt, cck


def commit(cfg: OracleCfg, state_indices, accepted, D: int, ckpt, conv_ckpt, conv_state, ssm_state):
    """Pools after committing each request's last accepted draft token (copies; inputs untouched).

    ckpt [B,D,HV,dk,dv] and conv_ckpt [B,D,conv_dim,K-1] (or None) as verify returns them.
    Returns (conv_state, ssm_state, code): code 0, 2 (a slot >= P) or 3 (an accepted count
    outside 0..D); such requests are skipped.
    """
    slots = _i32(state_indices)
    acc = _i32(accepted)
    cs = _f64(conv_state).copy()
    ss = _f64(ssm_state).copy()
    ck = _f64(ckpt)
    cck = _f64(conv_ckpt) if conv_ckpt is not None else None
    c = cfg._c()
    code = _L().ora_commit(ctypes.byref(c), ctypes.c_int(len(slots)), ctypes.c_int(D), _p(slots, _i32_p),
                           _p(acc, _i32_p), _p(ck), _p(cck), _p(cs), _p(ss), ctypes.c_int(ss.shape[0]))
    return cs, ss, int(code)


def extend_ckpt(cfg: OracleCfg, params: dict, x, a, b, cu_seqlens, state_indices, conv_state, ssm_state,
                ckpt_token_indices, ckpt_state_slots, num_ckpt: int, has_initial_state=None, want_conv: bool = True):
    """extend that also captures, per sequence, the state (and conv window) at one exclusive absolute
    packed-row boundary into row ckpt_state_slots[n] of the checkpoint buffers.

    Returns (out, conv_state, ssm_state, ckpt_states [num_ckpt,HV,dk,dv] (zeros where nothing was
    captured), ckpt_conv [num_ckpt,conv_dim,K-1] or None, code): code 0, or 4 when a boundary lies
    outside its sequence or a row >= num_ckpt (that sequence is skipped).
    """
    A_log, dt_bias, conv_w, conv_b, x, a, b = _layer_args(cfg, params, x, a, b)
    cu = _i32(cu_seqlens)
    slots = _i32(state_indices)
    hi = _i32(has_initial_state)
    idx = _i32(ckpt_token_indices)
    cks = _i32(ckpt_state_slots)
    cs = _f64(conv_state).copy()
    ss = _f64(ssm_state).copy()
    N = len(slots)
    T = int(cu[-1])
    P = cs.shape[0]
    out = np.zeros((T, cfg.HV, cfg.dv))
    ck = np.zeros((num_ckpt, cfg.HV, cfg.dk, cfg.dv))
    ckc = np.zeros((num_ckpt, cfg.conv_dim, cfg.K - 1)) if want_conv else None
    c = cfg._c()
    rc = _L().ora_extend_ckpt(
        ctypes.byref(c), _p(A_log), _p(dt_bias), _p(conv_w), _p(conv_b), _p(x), _p(a), _p(b), _p(cu, _i32_p),
        ctypes.c_int(N), _p(slots, _i32_p), _p(hi, _i32_p), _p(cs), _p(ss), ctypes.c_int(P), _p(out),
        _p(idx, _i32_p), _p(cks, _i32_p), _p(ck), _p(ckc), ctypes.c_int(num_ckpt),
    )
    if rc not in (0, 4):
        raise ValueError(f"oracle extend_ckpt rejected its arguments (code {rc})")
    return out, cs, ss, ck, ckc, int(rc)


def verify_tree(cfg: OracleCfg, params: dict, x, a, b, state_indices, parents, D: int, conv_state, ssm_state):
    """D draft tokens per request forming a tree: parents[i, t] is -1 (the slot) or an earlier token.
    Each token's output, state and conv window are those of running, from the slot, the path from the
    root to that token (the EAGLE tree verification of page "SGLang GDN hybrid linear attention test
    matrix").  Written as a replay of every path through ``extend`` (plain Python over small trees).

    Returns (out [B*D,HV,dv], ckpt [B,D,HV,dk,dv], conv_ckpt [B,D,conv_dim,K-1]); padded requests get
    zero outputs and zero checkpoints.
    """
    slots = _i32(state_indices)
    B = len(slots)
    par = _i32(parents).reshape(B, D)
    cs = _f64(conv_state)
    ss = _f64(ssm_state)
    xs, as_, bs = _f64(x), _f64(a), _f64(b)
    out = np.zeros((B * D, cfg.HV, cfg.dv))
    ckpt = np.zeros((B, D, cfg.HV, cfg.dk, cfg.dv))
    cck = np.zeros((B, D, cfg.conv_dim, cfg.K - 1))
    for i in range(B):
        slot = int(slots[i])
        if slot < 0:
            continue
        for t in range(D):
            path, nd = [], t
            while nd >= 0:
                assert par[i, nd] < nd, "a parent must precede its token"
                path.append(nd)
                nd = int(par[i, nd])
            rows = [i * D + q for q in reversed(path)]
            o, c1, s1 = extend(cfg, params, xs[rows], as_[rows], bs[rows], np.array([0, len(rows)], np.int32),
                               np.array([0], np.int32), cs[slot:slot + 1], ss[slot:slot + 1])
            out[i * D + t] = o[-1]
            ckpt[i, t] = s1[0]
            cck[i, t] = c1[0]
    return out, ckpt, cck
