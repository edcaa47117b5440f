"""Helpers shared by the GPU parity tests: run a workload through the C ABI,
run the same inputs through the fp64 oracle, compare."""
from __future__ import annotations

import numpy as np
import torch

import hybrid_linear_attention_causal_b200 as gdn
from hybrid_linear_attention_causal_b200 import workloads as W
from oracle import oracle as O
from tests.tolerances import assert_out_close, assert_state_close


def ocfg(spec) -> O.OracleCfg:
    return O.OracleCfg(HK=spec.HK, HV=spec.HV, dk=spec.dk, dv=spec.dv, K=spec.K)


def gcfg(spec) -> gdn.GdnConfig:
    return gdn.GdnConfig.from_spec(spec)


def to_device(w: W.Workload, device="cuda") -> W.Workload:
    mv = lambda t: None if t is None else t.to(device)
    return W.Workload(
        w.name, w.spec, {k: mv(v) for k, v in w.params.items()}, mv(w.x), mv(w.a), mv(w.b), mv(w.cu_seqlens),
        mv(w.state_indices), mv(w.has_initial_state), mv(w.conv_state), mv(w.ssm_state), dict(w.extra),
    )


def gpu_extend(wd: W.Workload, conv_state=None, ssm_state=None, x=None, a=None, b=None, cu=None):
    """Runs gdn_extend on device copies of the pools; returns (out, conv, ssm, device_error)."""
    spec = wd.spec
    x = wd.x if x is None else x
    a = wd.a if a is None else a
    b = wd.b if b is None else b
    cu = wd.cu_seqlens if cu is None else cu
    cfg = gcfg(spec)
    T, N = int(x.shape[0]), int(wd.state_indices.shape[0])
    ws = gdn.alloc_workspace(gdn.gdn_extend_workspace_size(cfg, N, T), x.device)
    out = torch.full((T, spec.HV, spec.dv), float("nan"), dtype=spec.dtype, device=x.device)
    conv = (wd.conv_state if conv_state is None else conv_state).clone()
    ssm = (wd.ssm_state if ssm_state is None else ssm_state).clone()
    gdn.gdn_extend(cfg, wd.params, x, a, b, cu, wd.state_indices, wd.has_initial_state, conv, ssm, out, ws)
    torch.cuda.synchronize()
    return out, conv, ssm, gdn.gdn_get_device_error(ws)


def oracle_extend(w: W.Workload, conv_state=None, ssm_state=None, **kw):
    return O.extend(ocfg(w.spec), w.params, w.x, w.a, w.b, w.cu_seqlens, w.state_indices,
                    w.conv_state if conv_state is None else conv_state,
                    w.ssm_state if ssm_state is None else ssm_state, has_initial_state=w.has_initial_state, **kw)


def f64(t) -> np.ndarray:
    return t.detach().to("cpu").to(torch.float64).numpy()


def same_bits(a: torch.Tensor, b: torch.Tensor) -> bool:
    a, b = a.detach().cpu().contiguous(), b.detach().cpu().contiguous()
    if a.dtype != b.dtype or a.shape != b.shape:
        return False
    iv = torch.int32 if a.element_size() == 4 else torch.int16
    return bool(torch.equal(a.view(iv), b.view(iv)))


def live_slots(w: W.Workload) -> list[int]:
    P = w.P
    return sorted({int(s) for s in w.state_indices.tolist() if 0 <= s < P})


def check_extend(w: W.Workload, gpu, ref, touched_lens=None):
    """Compares GPU extend results with the oracle's: outputs and states within
    tolerance, conv slots bit-exact, untouched slots bit-identical to the input."""
    out, conv, ssm, err = gpu
    r_out, r_conv, r_ssm = ref
    assert err == 0, f"device error word {err:#x}"
    assert_out_close(f64(out), r_out)
    lens = (w.cu_seqlens[1:] - w.cu_seqlens[:-1]).tolist()
    touched = sorted({int(s) for s, L in zip(w.state_indices.tolist(), lens) if s >= 0 and L > 0})
    for s in touched:
        assert_state_close(f64(ssm[s]), r_ssm[s], what=f"ssm slot {s}")
        want = torch.from_numpy(r_conv[s]).to(w.spec.dtype)
        assert same_bits(conv[s], want), f"conv slot {s} not bit-exact"
    for s in range(w.P):
        if s not in touched:
            assert same_bits(ssm[s], w.ssm_state[s]), f"untouched ssm slot {s} changed"
            assert same_bits(conv[s], w.conv_state[s]), f"untouched conv slot {s} changed"


def restrict_to_group(w: W.Workload, hk: int) -> W.Workload:
    """The same inputs seen by qk head hk and its G value heads only, as a
    layer with one qk head (CPU tensors).  Value heads do not interact, so the
    restricted layer's outputs are the full layer's outputs of those heads."""
    s = w.spec
    G = s.HV // s.HK
    qk = s.HK * s.dk
    cols = torch.cat([
        torch.arange(hk * s.dk, (hk + 1) * s.dk),
        torch.arange(qk + hk * s.dk, qk + (hk + 1) * s.dk),
        torch.arange(2 * qk + hk * G * s.dv, 2 * qk + (hk + 1) * G * s.dv),
    ]).to(w.x.device)
    heads = torch.arange(hk * G, (hk + 1) * G, device=w.x.device)
    spec = W.LayerSpec(HK=1, HV=G, dk=s.dk, dv=s.dv, K=s.K, dtype=s.dtype)
    cpu = lambda t: None if t is None else t.to("cpu")
    params = {
        "A_log": cpu(w.params["A_log"][heads]),
        "dt_bias": cpu(w.params["dt_bias"][heads]),
        "conv_w": cpu(w.params["conv_w"][cols]),
        "conv_b": None if w.params.get("conv_b") is None else cpu(w.params["conv_b"][cols]),
    }
    slots = live_slots(w)
    slot_idx = torch.tensor(slots, dtype=torch.long, device=w.x.device)
    remap = {sl: i for i, sl in enumerate(slots)}
    new_slots = torch.tensor([remap.get(int(v), -1) for v in w.state_indices.tolist()], dtype=torch.int32)
    return W.Workload(
        f"{w.name}_group{hk}", spec, params, cpu(w.x[:, cols]), cpu(w.a[:, heads]), cpu(w.b[:, heads]),
        cpu(w.cu_seqlens), new_slots, cpu(w.has_initial_state), cpu(w.conv_state[slot_idx][:, cols]),
        cpu(w.ssm_state[slot_idx][:, heads]), extra={"slots": slots, "cols": cols, "heads": heads},
    )
