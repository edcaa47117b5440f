"""gdn_extend_static_scratch: the EXTEND entry point for callers that cannot
allocate device memory (plugins whose enqueue step may not allocate, paths
that cannot take cudaMalloc's device synchronisation).  It must give the same
results as gdn_extend with a caller-allocated workspace, call after call,
although every call reuses the library's one fixed scratch array.

This file is collected last on purpose: if it fails, a run that stops at the
first failure has already run every other test."""
import ctypes

import pytest
import torch

import hybrid_linear_attention_causal_b200 as gdn
from hybrid_linear_attention_causal_b200 import binding as B
from hybrid_linear_attention_causal_b200 import workloads as W
from tests.gpu_util import gpu_extend, same_bits, to_device


def _static_call(wd):
    """One gdn_extend_static_scratch call through the C ABI on copies of the pools."""
    spec = wd.spec
    cfg = gdn.GdnConfig.from_spec(spec)
    out = torch.full((wd.T, spec.HV, spec.dv), float("nan"), dtype=spec.dtype, device="cuda")
    conv, ssm = wd.conv_state.clone(), wd.ssm_state.clone()
    params = B.GdnParamsC(wd.params["A_log"].data_ptr(), wd.params["dt_bias"].data_ptr(),
                          wd.params["conv_w"].data_ptr(), None)
    hi = wd.has_initial_state
    rc = B.lib().gdn_extend_static_scratch(
        ctypes.byref(cfg.c()), ctypes.byref(params), wd.x.data_ptr(), wd.a.data_ptr(), wd.b.data_ptr(),
        wd.cu_seqlens.data_ptr(), wd.N, wd.T, wd.state_indices.data_ptr(), None if hi is None else hi.data_ptr(),
        conv.data_ptr(), ssm.data_ptr(), wd.P, out.data_ptr(), torch.cuda.current_stream().cuda_stream)
    assert rc == gdn.GDN_OK, B.strerror(rc)
    torch.cuda.synchronize()
    return out, conv, ssm


def _compare(wd, got, ref):
    """The static path runs gdn_extend's kernels on the same (N, T), and extend is bit-reproducible, so
    the outputs and every slot of both pools must match gdn_extend's bit for bit; a scratch array that
    kept something stale from an earlier call would show here."""
    out, conv, ssm = got
    r_out, r_conv, r_ssm, err = ref
    assert err == 0
    assert same_bits(out, r_out), "outputs differ from gdn_extend's"
    for s in range(wd.P):
        assert same_bits(ssm[s], r_ssm[s]), f"ssm slot {s} differs from gdn_extend's"
        assert same_bits(conv[s], r_conv[s]), f"conv slot {s} differs from gdn_extend's"


@pytest.mark.gpu
def test_static_scratch_matches_workspace_entry_point_on_two_calls_in_a_row():
    spec = W.LayerSpec(HK=4, HV=8, dk=64, dv=64, dtype=torch.bfloat16)
    first = to_device(W.random_case(spec, [150, 1, 0, 64, 385], P=8, seed=101, has_init=[1, 0, 1, 1, 1]))
    second = to_device(W.random_case(spec, [70, 129], P=8, seed=102))
    for wd in (first, second):  # the second call reuses the scratch the first one left behind
        got = _static_call(wd)
        _compare(wd, got, gpu_extend(wd))
    # and once more on the first batch, after the second one overwrote the scratch
    _compare(first, _static_call(first), gpu_extend(first))


def test_static_scratch_rejects_sizes_beyond_its_maximum():
    """No GPU needed: the size check runs before anything touches the device."""
    cfg = gdn.GdnConfig(16, 32, 128, 128)
    lo, hi = 1, 1 << 20  # largest single-sequence batch that fits the fixed scratch
    while lo < hi:
        mid = (lo + hi + 1) // 2
        if gdn.gdn_extend_workspace_size(cfg, 1, mid) <= B.EXTEND_STATIC_SCRATCH_BYTES:
            lo = mid
        else:
            hi = mid - 1
    assert lo >= 256, "the fixed scratch should hold a useful batch of the large layer"
    too_big = lo + 1
    F = 0x10000
    params = B.GdnParamsC(F, F, F, None)
    rc = B.lib().gdn_extend_static_scratch(ctypes.byref(cfg.c()), ctypes.byref(params), F, F, F, F, 1, too_big, F,
                                           None, F, F, 4, F, None)
    assert rc == gdn.GDN_ERR_WORKSPACE
    bad = gdn.GdnConfig(16, 32, 96, 128)
    rc = B.lib().gdn_extend_static_scratch(ctypes.byref(bad.c()), ctypes.byref(params), F, F, F, F, 1, 8, F, None,
                                           F, F, 4, F, None)
    assert rc == gdn.GDN_ERR_UNSUPPORTED
