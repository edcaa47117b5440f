"""The library's two device-side guards, exercised on the GPU without faulting it.

1. Bounded waits.  Every tensor-core kernel waits on mbarrier phases with a
   time limit; a wait that runs out raises GDN_DEVERR_TIMEOUT, lets its copies
   land and returns, so a stuck kernel ends with an error status instead of
   hanging the GPU.  gdn_check_bounded_wait runs that same wait on a barrier
   that nothing completes, and the tests check that the bit is raised, that the
   kernel returned, and that the context keeps working.

2. The fp16 operand range.  The prefill rounds its tensor-core operands to
   fp16 (v, W, U, T's tiles, V' and the state's copy), whose largest finite
   magnitude is 65504, while its inputs are bf16 and its state fp32.  Inputs
   that stay inside that range must meet parity (the relative bounds; the
   absolute output bound scales with the inputs); inputs that leave it must
   raise GDN_DEVERR_FP16_RANGE, never return silently wrong results.
"""
import time

import numpy as np
import pytest
import torch

import hybrid_linear_attention_causal_b200 as gdn
from hybrid_linear_attention_causal_b200 import workloads as W
from tests.gpu_util import f64, gpu_extend, oracle_extend, same_bits, to_device
from tests.tolerances import OUT_MAX_ABS, OUT_REL_L2, STATE_REL_L2, rel_l2

pytestmark = pytest.mark.gpu

SPEC = W.LayerSpec(HK=2, HV=4, dk=128, dv=128, dtype=torch.bfloat16)


def test_bounded_wait_runs_out_raises_timeout_and_returns():
    ws = gdn.alloc_workspace(gdn.gdn_decode_workspace_size(gdn.GdnConfig(16, 32, 128, 128), 1), "cuda")
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    gdn.gdn_check_bounded_wait(False, 1_000_000, ws)  # nothing ever completes this barrier: 1 ms limit
    torch.cuda.synchronize()
    elapsed = time.perf_counter() - t0
    assert gdn.gdn_get_device_error(ws) & gdn.GDN_DEVERR_TIMEOUT
    assert elapsed < 1.0, f"the wait should give up after 1 ms, took {elapsed:.3f} s"
    # a barrier that completes: no bit on a fresh workspace
    ws2 = gdn.alloc_workspace(512, "cuda")
    gdn.gdn_check_bounded_wait(True, 1_000_000, ws2)
    assert gdn.gdn_get_device_error(ws2) == 0
    # the bit is sticky on the first workspace, and the context still runs real work correctly
    assert gdn.gdn_get_device_error(ws) & gdn.GDN_DEVERR_TIMEOUT
    w = W.random_case(W.LayerSpec(HK=2, HV=2, dk=64, dv=64, dtype=torch.bfloat16), [70], P=2, seed=11)
    out, conv, ssm, err = gpu_extend(to_device(w))
    assert err == 0
    r_out = oracle_extend(w)[0]
    assert rel_l2(f64(out), r_out) <= OUT_REL_L2


def _scaled_case(seed, v_scale=1.0, state_peak=None):
    w = W.random_case(SPEC, [200, 70], P=4, seed=seed)
    qk = 2 * SPEC.HK * SPEC.dk
    if v_scale != 1.0:
        x = w.x.float()
        x[:, qk:] *= v_scale
        w.x = x.to(SPEC.dtype)
    if state_peak is not None:
        for s in w.state_indices.tolist():
            w.ssm_state[s] *= state_peak / float(w.ssm_state[s].abs().max())
    return w


def _parity_or_flag(w, scale):
    """Either the range bit is raised, or outputs and states meet parity, the output's absolute bound
    scaled by `scale` (outputs grow with v and with the state)."""
    out, conv, ssm, err = gpu_extend(to_device(w))
    r_out, r_conv, r_ssm = oracle_extend(w)
    if err & gdn.GDN_DEVERR_FP16_RANGE:
        return "flagged"
    assert err == 0, f"device error word {err:#x}"
    got = f64(out)
    assert np.isfinite(got).all()
    assert rel_l2(got, r_out) <= OUT_REL_L2
    assert float(np.max(np.abs(got - r_out))) <= OUT_MAX_ABS * scale
    for s in w.state_indices.tolist():
        assert rel_l2(f64(ssm[s]), r_ssm[s]) <= STATE_REL_L2, f"slot {s}"
        assert same_bits(conv[s], torch.from_numpy(r_conv[s]).to(SPEC.dtype))
    return "parity"


def test_v_scaled_by_1e3_stays_in_range_and_meets_parity():
    """v about 1e3 times larger (still far below 65504 after the conv): no flag, parity holds."""
    assert _parity_or_flag(_scaled_case(21, v_scale=1e3), 1e3) == "parity"


def test_state_near_the_fp16_bound_meets_parity_or_flags():
    """Initial states scaled to a peak of 6e4, just under fp16's largest value: the state's fp16 copy
    and V' = U - W S approach the bound; the result is either within parity or flagged."""
    _parity_or_flag(_scaled_case(22, state_peak=6e4), 6e4 / 0.5)


def test_v_beyond_fp16_range_is_flagged():
    """v about 1e5 times larger: its fp16 copy would overflow, so the range bit must be raised."""
    w = _scaled_case(23, v_scale=1e5)
    _, _, _, err = gpu_extend(to_device(w))
    assert err & gdn.GDN_DEVERR_FP16_RANGE, f"device error word {err:#x}"
