"""Host-side checks of the C ABI that need no GPU: the library loads, exports
every entry point include/gdn.h declares, sizes workspaces, and rejects bad
arguments before anything is launched."""
import ctypes
import os
import re

import pytest
import torch

import hybrid_linear_attention_causal_b200 as gdn
from hybrid_linear_attention_causal_b200 import binding as B

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADERS = [os.path.join(ROOT, "include", h) for h in ("gdn.h", "ssd.h")]

FAKE = 0x10000  # aligned, never dereferenced by the host-side validation
FAKE_MIS = 0x10004


def declared_symbols():
    text = "".join(open(h).read() for h in HEADERS)
    return sorted(set(re.findall(r"GDN_API\s+[\w\s\*]+?\b((?:gdn|ssd)_\w+)\s*\(", text)))


def test_library_exports_every_declared_symbol():
    syms = declared_symbols()
    assert len(syms) >= 12 and "ssd_combined_fwd" in syms
    L = B.lib()
    for s in syms:
        assert hasattr(L, s), f"libgdn.so does not export {s}"


def test_strerror_codes():
    for code in (gdn.GDN_OK, gdn.GDN_ERR_INVALID_ARG, gdn.GDN_ERR_UNSUPPORTED, gdn.GDN_ERR_WORKSPACE,
                 gdn.GDN_ERR_CUDA):
        assert B.strerror(code) and "unknown" not in B.strerror(code)
    assert "unknown" in B.strerror(99)


def cfg(**kw):
    base = dict(num_qk_heads=16, num_v_heads=32, head_k_dim=128, head_v_dim=128)
    base.update(kw)
    return gdn.GdnConfig(**base)


def test_workspace_sizes():
    c = cfg()
    small = gdn.gdn_extend_workspace_size(c, 1, 64)
    big = gdn.gdn_extend_workspace_size(c, 8, 32768)
    assert 0 < small < big
    # every chunk of 64 rows holds the tiles the per-chunk step hands the state pass: fp16 [K ; Q] per qk
    # head (128 x dk), and per value head fp16 W (64 x dk), U^T (dv x 64), Aqk (64 x 64) and a 16-byte
    # gate vector per row
    per_chunk = 16 * 128 * 128 * 2 + 32 * (64 * 128 * 2 + 128 * 64 * 2 + 64 * 64 * 2 + 64 * 16)
    assert big >= (32768 // 64) * per_chunk
    assert gdn.gdn_decode_workspace_size(c, 256) == B.HEADER_BYTES
    assert gdn.gdn_verify_workspace_size(c, 256, 4) == B.HEADER_BYTES
    assert gdn.gdn_verify_workspace_size(c, 256, 17) == 0
    assert gdn.gdn_extend_workspace_size(cfg(head_k_dim=96), 1, 64) == 0
    assert gdn.gdn_extend_workspace_size(cfg(num_v_heads=24, num_qk_heads=16), 1, 64) == 0


def _params(mis=False):
    p = B.GdnParamsC(FAKE, FAKE, FAKE_MIS if mis else FAKE, None)
    return ctypes.byref(p)


def _extend(c, N=2, T=100, ws_bytes=1 << 40, params=None, x=FAKE, cu=FAKE, ws=FAKE, out=FAKE):
    return B.lib().gdn_extend(ctypes.byref(c.c()), params or _params(), x, FAKE, FAKE, cu, N, T, FAKE, None, FAKE,
                              FAKE, 4, out, ws, ws_bytes, None)


def _decode(c, Bn=3, ws_bytes=256, ws=FAKE, slots=FAKE):
    return B.lib().gdn_decode(ctypes.byref(c.c()), _params(), FAKE, FAKE, FAKE, slots, Bn, FAKE, FAKE, 8, FAKE, ws,
                              ws_bytes, None)


def _verify(c, Bn=3, D=4, ckpt=FAKE):
    return B.lib().gdn_verify(ctypes.byref(c.c()), _params(), FAKE, FAKE, FAKE, FAKE, Bn, D, FAKE, FAKE, 8, ckpt,
                              None, FAKE, FAKE, 256, None)


def test_extend_argument_validation():
    c = cfg()
    assert _extend(c, N=0) == gdn.GDN_OK  # nothing to do, nothing launched
    assert _extend(c, T=0) == gdn.GDN_OK
    assert _extend(c, N=-1) == gdn.GDN_ERR_INVALID_ARG
    assert _extend(c, x=None) == gdn.GDN_ERR_INVALID_ARG
    assert _extend(c, out=None) == gdn.GDN_ERR_INVALID_ARG
    assert _extend(c, cu=None) == gdn.GDN_ERR_INVALID_ARG
    assert _extend(c, ws=None) == gdn.GDN_ERR_INVALID_ARG
    assert _extend(c, x=FAKE_MIS) == gdn.GDN_ERR_INVALID_ARG
    assert _extend(c, params=_params(mis=True)) == gdn.GDN_ERR_INVALID_ARG
    assert _extend(c, ws_bytes=1024) == gdn.GDN_ERR_WORKSPACE
    assert _extend(cfg(num_v_heads=20)) == gdn.GDN_ERR_INVALID_ARG  # HV % HK != 0
    assert _extend(cfg(head_k_dim=96)) == gdn.GDN_ERR_UNSUPPORTED
    assert _extend(cfg(head_v_dim=256)) == gdn.GDN_ERR_UNSUPPORTED
    assert _extend(cfg(conv_kernel=3)) == gdn.GDN_ERR_UNSUPPORTED
    assert _extend(gdn.GdnConfig(16, 32, 128, 128, dtype=__import__("torch").float16)) == gdn.GDN_ERR_UNSUPPORTED
    assert B.lib().gdn_extend(None, _params(), FAKE, FAKE, FAKE, FAKE, 1, 1, FAKE, None, FAKE, FAKE, 4, FAKE, FAKE,
                              1 << 40, None) == gdn.GDN_ERR_INVALID_ARG
    assert B.lib().gdn_extend(ctypes.byref(cfg().c()), None, FAKE, FAKE, FAKE, FAKE, 1, 1, FAKE, None, FAKE, FAKE,
                              4, FAKE, FAKE, 1 << 40, None) == gdn.GDN_ERR_INVALID_ARG


def test_decode_and_verify_argument_validation():
    c = cfg()
    assert _decode(c, Bn=0) == gdn.GDN_OK  # IDLE
    assert _decode(c, Bn=-2) == gdn.GDN_ERR_INVALID_ARG
    assert _decode(c, ws=None) == gdn.GDN_ERR_INVALID_ARG
    assert _decode(c, slots=None) == gdn.GDN_ERR_INVALID_ARG
    assert _decode(c, ws_bytes=16) == gdn.GDN_ERR_WORKSPACE
    assert _decode(cfg(head_k_dim=32)) == gdn.GDN_ERR_UNSUPPORTED
    assert _verify(c, Bn=0) == gdn.GDN_OK
    assert _verify(c, D=0) == gdn.GDN_ERR_INVALID_ARG
    assert _verify(c, D=17) == gdn.GDN_ERR_INVALID_ARG
    assert _verify(c, ckpt=None) == gdn.GDN_ERR_INVALID_ARG


def _extend_ckpt(c, idx=FAKE, rows=FAKE, states=FAKE, cconv=None, num=4, x=FAKE):
    return B.lib().gdn_extend_checkpoints(ctypes.byref(c.c()), _params(), x, FAKE, FAKE, FAKE, 2, 100, FAKE, None,
                                          FAKE, FAKE, 4, FAKE, idx, rows, states, cconv, num, FAKE, 1 << 40, None)


def test_extend_checkpoints_argument_validation():
    c = cfg()
    assert _extend_ckpt(c, idx=None) == gdn.GDN_ERR_INVALID_ARG  # the three checkpoint arrays go together
    assert _extend_ckpt(c, rows=None) == gdn.GDN_ERR_INVALID_ARG
    assert _extend_ckpt(c, states=None) == gdn.GDN_ERR_INVALID_ARG
    assert _extend_ckpt(c, num=-1) == gdn.GDN_ERR_INVALID_ARG
    assert _extend_ckpt(c, idx=FAKE_MIS) == gdn.GDN_ERR_INVALID_ARG
    assert _extend_ckpt(c, cconv=FAKE_MIS) == gdn.GDN_ERR_INVALID_ARG
    assert _extend_ckpt(c, x=None) == gdn.GDN_ERR_INVALID_ARG  # and the extend's own checks still apply


def _commit(c, Bn=3, D=4, slots=FAKE, acc=FAKE, ckpt=FAKE, cck=None, cs=None, ss=FAKE, ws=FAKE, ws_bytes=256):
    return B.lib().gdn_commit(ctypes.byref(c.c()), slots, acc, Bn, D, ckpt, cck, cs, ss, 8, ws, ws_bytes, None)


def test_commit_argument_validation():
    c = cfg()
    assert gdn.gdn_commit_workspace_size(c, 256) == B.HEADER_BYTES
    assert gdn.gdn_commit_workspace_size(cfg(head_k_dim=96), 256) == 0
    assert _commit(c, Bn=0) == gdn.GDN_OK  # nothing to commit, nothing launched
    assert _commit(c, Bn=-1) == gdn.GDN_ERR_INVALID_ARG
    assert _commit(c, D=0) == gdn.GDN_ERR_INVALID_ARG
    assert _commit(c, D=17) == gdn.GDN_ERR_INVALID_ARG
    assert _commit(c, slots=None) == gdn.GDN_ERR_INVALID_ARG
    assert _commit(c, acc=None) == gdn.GDN_ERR_INVALID_ARG
    assert _commit(c, ckpt=None) == gdn.GDN_ERR_INVALID_ARG
    assert _commit(c, ss=None) == gdn.GDN_ERR_INVALID_ARG
    assert _commit(c, cck=FAKE, cs=None) == gdn.GDN_ERR_INVALID_ARG  # a conv checkpoint needs the conv pool
    assert _commit(c, cck=FAKE_MIS, cs=FAKE) == gdn.GDN_ERR_INVALID_ARG
    assert _commit(c, acc=FAKE_MIS) == gdn.GDN_ERR_INVALID_ARG
    assert _commit(c, ws=None) == gdn.GDN_ERR_INVALID_ARG
    assert _commit(c, ws_bytes=16) == gdn.GDN_ERR_WORKSPACE
    assert _commit(cfg(head_v_dim=256)) == gdn.GDN_ERR_UNSUPPORTED


def test_verify_tree_argument_validation():
    c = cfg()
    tree = lambda parents=FAKE, D=4: B.lib().gdn_verify_tree(ctypes.byref(c.c()), _params(), FAKE, FAKE, FAKE, FAKE,
                                                            parents, 3, D, FAKE, FAKE, 8, FAKE, None, FAKE, FAKE,
                                                            256, None)
    assert tree(parents=None) == gdn.GDN_ERR_INVALID_ARG  # a tree needs its parents
    assert tree(parents=FAKE_MIS) == gdn.GDN_ERR_INVALID_ARG
    assert tree(D=17) == gdn.GDN_ERR_INVALID_ARG


def test_error_helpers_reject_null():
    v = ctypes.c_int32(0)
    assert B.lib().gdn_get_device_error(None, ctypes.byref(v), None) == gdn.GDN_ERR_INVALID_ARG
    assert B.lib().gdn_reset_device_error(None, None) == gdn.GDN_ERR_INVALID_ARG


def test_binding_refuses_host_tensors():
    import torch

    c = gdn.GdnConfig(2, 2, 64, 64, dtype=torch.float32)
    t = torch.zeros(4)
    with pytest.raises(ValueError):
        gdn.gdn_decode(c, {"A_log": t, "dt_bias": t, "conv_w": t}, t, t, t, torch.zeros(1, dtype=torch.int32), t, t,
                       t, t)


def _ssd_call(c, x=FAKE, dt=FAKE, A=FAKE, Bm=FAKE, C=FAKE, D=None, z=None, bias=None, cu=FAKE, N=2, T=100,
              init=None, fin=None, ck=(None, None, None), num_ck=0, out=FAKE, ws=FAKE, wsb=4096):
    return B.lib().ssd_combined_fwd(ctypes.byref(c.c()), x, dt, A, Bm, C, D, z, bias, cu, N, T, init, fin, ck[0],
                                    ck[1], ck[2], num_ck, out, ws, wsb, None)


def test_ssd_workspace_and_argument_validation():
    c = gdn.SsdConfig(nheads=8, headdim=64, dstate=128, ngroups=2)
    assert gdn.ssd_workspace_size(c, 8, 32768) == B.HEADER_BYTES + 32
    assert gdn.ssd_workspace_size(c, 5, 100) == B.HEADER_BYTES + 32
    assert B.lib().ssd_workspace_size(None, 1, 1) == 0
    inv, uns, wsp = gdn.GDN_ERR_INVALID_ARG, gdn.GDN_ERR_UNSUPPORTED, gdn.GDN_ERR_WORKSPACE
    assert _ssd_call(gdn.SsdConfig(nheads=6, headdim=64, dstate=128, ngroups=4)) == inv   # H % G
    assert _ssd_call(gdn.SsdConfig(nheads=8, headdim=32, dstate=128, ngroups=2)) == uns   # headdim
    assert _ssd_call(gdn.SsdConfig(nheads=8, headdim=64, dstate=96, ngroups=2)) == uns    # dstate
    assert _ssd_call(gdn.SsdConfig(nheads=8, headdim=64, dstate=128, ngroups=2, dt_limit=(1.0, 0.5))) == inv
    assert _ssd_call(c, N=-1) == inv
    assert _ssd_call(c, x=None) == inv
    assert _ssd_call(c, cu=None) == inv
    assert _ssd_call(c, A=None) == inv
    assert _ssd_call(c, out=None) == inv
    assert _ssd_call(c, x=FAKE_MIS) == inv
    assert _ssd_call(c, z=FAKE_MIS) == inv
    assert _ssd_call(c, init=FAKE_MIS) == inv
    assert _ssd_call(c, ck=(FAKE, None, FAKE), num_ck=1) == inv           # checkpoint arguments in part
    assert _ssd_call(c, ck=(FAKE, FAKE, FAKE), num_ck=-1) == inv
    assert _ssd_call(c, ws=None) == inv
    assert _ssd_call(c, wsb=16) == wsp
    assert _ssd_call(c, N=2, wsb=B.HEADER_BYTES) == wsp                    # no room for the order
    assert _ssd_call(c, N=0, x=None, cu=None) == gdn.GDN_OK                # nothing to do
    bad = B.SsdConfigC(8, 64, 128, 2, 7, 1, 0, 0.0, float("inf"))          # state dtype
    assert B.lib().ssd_combined_fwd(ctypes.byref(bad), FAKE, FAKE, FAKE, FAKE, FAKE, None, None, None, FAKE, 2,
                                    100, None, None, None, None, None, 0, FAKE, FAKE, 4096, None) == uns


def test_ssd_workload_recipe_is_seeded_and_shaped():
    from hybrid_linear_attention_causal_b200 import workloads as W

    spec = W.SsdSpec(H=6, P=64, N=64, G=3, state_dtype=torch.float16)
    a = W.ssd_case(spec, [5, 0, 70], seed=3, d_per_dim=True)
    b = W.ssd_case(spec, [5, 0, 70], seed=3, d_per_dim=True)
    for name in ("x", "dt", "A", "B", "C", "D", "z", "dt_bias", "cu", "init"):
        assert torch.equal(getattr(a, name), getattr(b, name)), name
    assert a.x.shape == (75, 6, 64) and a.x.dtype == torch.bfloat16
    assert a.B.shape == (75, 3, 64) and a.C.shape == a.B.shape and a.dt.shape == (75, 6)
    assert a.D.shape == (6, 64) and a.init.shape == (3, 6, 64, 64) and a.init.dtype == torch.float16
    assert a.cu.tolist() == [0, 5, 5, 75]
    assert (a.A < 0).all() and a.A.dtype == torch.float32
    w = W.ssd_prefill()
    assert w.T == 32768 and len(w.lengths) == 8 and all(512 <= n <= 16384 for n in w.lengths)
    none = W.ssd_case(spec, [4], seed=1, with_D=False, with_z=False, with_bias=False, init_random=False)
    assert none.D is None and none.z is None and none.dt_bias is None and none.init is None


def test_bounded_wait_check_rejects_bad_arguments_before_launching():
    """gdn_check_bounded_wait validates on the host (no GPU needed): the time limit must lie in
    (0, 1e9] ns and the workspace must be a non-null, 16-byte aligned buffer of at least 512 bytes."""
    L = B.lib()
    assert L.gdn_check_bounded_wait(0, 0, FAKE, 512, None) == gdn.GDN_ERR_INVALID_ARG
    assert L.gdn_check_bounded_wait(0, -5, FAKE, 512, None) == gdn.GDN_ERR_INVALID_ARG
    assert L.gdn_check_bounded_wait(0, 1_000_000_001, FAKE, 512, None) == gdn.GDN_ERR_INVALID_ARG
    assert L.gdn_check_bounded_wait(0, 1000, None, 512, None) == gdn.GDN_ERR_INVALID_ARG
    assert L.gdn_check_bounded_wait(0, 1000, FAKE_MIS, 512, None) == gdn.GDN_ERR_INVALID_ARG
    assert L.gdn_check_bounded_wait(0, 1000, FAKE, 256, None) == gdn.GDN_ERR_WORKSPACE
