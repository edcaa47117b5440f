"""Mamba2 SSD scan parity: the CUDA path through the C ABI (ssd_combined_fwd)
against the fp64 oracle on the same seeded inputs."""
import math

import numpy as np
import pytest
import torch

import hybrid_linear_attention_causal_b200 as gdn
from hybrid_linear_attention_causal_b200 import workloads as W
from oracle import ssd as OS
from tests.tolerances import assert_ssd_out_close, assert_ssd_state_close

pytestmark = pytest.mark.gpu


def _dname(dt: torch.dtype) -> str:
    return str(dt).replace("torch.", "")


def _f64(t):
    return None if t is None else t.detach().cpu().to(torch.float64).numpy()


def gpu_ssd(w: W.SsdWorkload, d_per_dim=False, softplus=True, dt_limit=(0.0, math.inf), fin=True, ck=None,
            num_ck=0, cu=None):
    """Runs ssd_combined_fwd on device copies; returns (out, final, ckpt, device_error)."""
    s = w.spec
    wd = w.to("cuda")
    cu = wd.cu if cu is None else cu.cuda()
    cfg = gdn.SsdConfig(nheads=s.H, headdim=s.P, dstate=s.N, ngroups=s.G, state_dtype=s.state_dtype,
                        dt_softplus=softplus, d_per_dim=d_per_dim, dt_limit=dt_limit)
    Nseq = int(cu.shape[0]) - 1
    ws = gdn.alloc_workspace(gdn.ssd_workspace_size(cfg, Nseq, w.T), "cuda")
    out = torch.full((w.T, s.H, s.P), float("nan"), dtype=torch.bfloat16, device="cuda")
    final = torch.full((Nseq, s.H, s.P, s.N), float("nan"), dtype=s.state_dtype, device="cuda") if fin else None
    ck_idx = ck_row = ck_states = None
    if ck is not None:
        ck_idx = torch.tensor(ck[0], dtype=torch.int32, device="cuda")
        ck_row = torch.tensor(ck[1], dtype=torch.int32, device="cuda")
        ck_states = torch.zeros((num_ck, s.H, s.P, s.N), dtype=s.state_dtype, device="cuda")
    gdn.ssd_combined_fwd(cfg, wd.x, wd.dt, wd.A, wd.B, wd.C, cu, out, ws, D=wd.D, z=wd.z, dt_bias=wd.dt_bias,
                         initial_states=wd.init, final_states=final, ckpt_token_indices=ck_idx,
                         ckpt_state_slots=ck_row, ckpt_states=ck_states)
    torch.cuda.synchronize()
    return out, final, ck_states, gdn.gdn_get_device_error(ws)


def oracle_ssd(w: W.SsdWorkload, d_per_dim=False, softplus=True, dt_limit=(0.0, math.inf), ck=None, num_ck=0,
               heads=None):
    """The oracle on the same inputs; `heads` restricts it to a subset of heads (each keeping its group)."""
    s = w.spec
    x, dt, A, Bm, Cm, D, z, bias, init = w.x, w.dt, w.A, w.B, w.C, w.D, w.z, w.dt_bias, w.init
    H, G = s.H, s.G
    if heads is not None:
        hpg = s.H // s.G
        groups = [h // hpg for h in heads]
        x, dt, A, z = x[:, heads], dt[:, heads], A[heads], None if z is None else z[:, heads]
        Bm, Cm = Bm[:, groups], Cm[:, groups]
        D = None if D is None else D[heads]
        bias = None if bias is None else bias[heads]
        init = None if init is None else init[:, heads]
        H = G = len(heads)
    cfg = OS.SsdCfg(H=H, P=s.P, N=s.N, G=G, dt_softplus=softplus, dt_limit=dt_limit, d_per_dim=d_per_dim)
    kw = {}
    if ck is not None:
        kw = dict(ck_idx=ck[0], ck_row=ck[1], num_ck=num_ck)
    return OS.scan(cfg, x, dt, A, Bm, Cm, w.cu, D=D, z=z, dt_bias=bias, init=init, return_rc=True, **kw)


def check(w, gpu, ref, what=""):
    out, fin, _, err = gpu
    y, f, _, rc = ref
    assert err == 0 and rc == 0
    assert_ssd_out_close(_f64(out), y, what=f"{what} out")
    if fin is not None:
        assert_ssd_state_close(_f64(fin), f, _dname(w.spec.state_dtype), what=f"{what} final state")


@pytest.mark.parametrize("state_dtype", [torch.bfloat16, torch.float32, torch.float16])
def test_ragged_sequences_all_options(state_dtype):
    """Several sequences spanning 0 to 3 chunks with ragged tails, skip, gate, bias and initial states."""
    w = W.ssd_case(W.SsdSpec(H=4, P=64, N=128, G=2, state_dtype=state_dtype), [70, 1, 130, 0, 64, 200], seed=31)
    check(w, gpu_ssd(w), oracle_ssd(w), "ragged")


def test_state_dim_64_one_group_skip_per_dim():
    w = W.ssd_case(W.SsdSpec(H=6, P=64, N=64, G=1, state_dtype=torch.float32), [129, 63, 5], seed=32, d_per_dim=True)
    check(w, gpu_ssd(w, d_per_dim=True), oracle_ssd(w, d_per_dim=True), "n64")


def test_no_optional_inputs_raw_steps_with_limits():
    """No D, z, dt_bias or initial state; steps used raw and clamped to [0.01, 0.5]."""
    w = W.ssd_case(W.SsdSpec(H=4, P=64, N=128, G=4, state_dtype=torch.float32), [100, 257], seed=33, with_D=False,
                   with_z=False, with_bias=False, init_random=False)
    lim = (0.01, 0.5)
    check(w, gpu_ssd(w, softplus=False, dt_limit=lim), oracle_ssd(w, softplus=False, dt_limit=lim), "raw")


def test_slow_decay_long_sequence():
    """|A| in [0.01, 0.1]: the state keeps a long memory, so the carried fp32 state is what decides parity."""
    w = W.ssd_case(W.SsdSpec(H=4, P=64, N=128, G=2, state_dtype=torch.float32), [2000, 700], seed=34,
                   a_range=(0.01, 0.1))
    check(w, gpu_ssd(w), oracle_ssd(w), "slow decay")


def test_no_final_states_pointer():
    w = W.ssd_case(W.SsdSpec(H=2, P=64, N=128, G=1), [90], seed=35)
    gpu = gpu_ssd(w, fin=False)
    check(w, gpu, oracle_ssd(w), "no final")


def test_checkpoints():
    """Boundaries mid chunk, on a chunk edge, at the start and at the end of their sequences; one disabled."""
    lens = [150, 64, 70, 40, 9]
    w = W.ssd_case(W.SsdSpec(H=4, P=64, N=128, G=2, state_dtype=torch.float32), lens, seed=36)
    cu = np.concatenate([[0], np.cumsum(lens)])
    bounds = [int(cu[0] + 77), int(cu[1] + 64), int(cu[2]), int(cu[3] + 40), -1]
    rows = [3, 0, 1, 2, 0]
    gpu = gpu_ssd(w, ck=(bounds, rows), num_ck=4)
    ref = oracle_ssd(w, ck=(bounds, rows), num_ck=4)
    check(w, gpu, ref, "ckpt")
    assert_ssd_state_close(_f64(gpu[2]), ref[2], "float32", what="checkpoints")


def test_checkpoint_out_of_range_is_flagged():
    w = W.ssd_case(W.SsdSpec(H=2, P=64, N=128, G=1, state_dtype=torch.float32), [50, 30], seed=37)
    out, fin, cks, err = gpu_ssd(w, ck=([60, 20], [0, 5]), num_ck=1)   # outside its sequence; row >= num_ckpt
    assert err == gdn.GDN_DEVERR_CKPT_RANGE
    assert not cks.any()
    y, f, _, _ = oracle_ssd(w)
    assert_ssd_out_close(_f64(out), y)
    assert_ssd_state_close(_f64(fin), f, "float32")


def test_bad_seqlens_are_flagged_and_skipped():
    w = W.ssd_case(W.SsdSpec(H=2, P=64, N=128, G=1), [40, 30], seed=38)
    out, _, _, err = gpu_ssd(w, cu=torch.tensor([0, 40, 90], dtype=torch.int32))   # past T = 70
    assert err & gdn.GDN_DEVERR_SEQLENS
    assert torch.isnan(out[40:].float()).all()


def test_bench_workload_sampled_heads():
    """The bench's full-size workload (128 heads, 32768 rows in 8 sequences), launched as the bench
    launches it; the oracle checks a sample of heads, each with its own group, over every row."""
    w = W.ssd_prefill()
    out, fin, _, err = gpu_ssd(w)
    assert err == 0
    heads = [0, 37, 77, 127]
    y, f, _, rc = oracle_ssd(w, heads=heads)
    assert rc == 0
    assert_ssd_out_close(_f64(out[:, heads]), y, what="sampled heads out")
    assert_ssd_state_close(_f64(fin[:, heads]), f, "bfloat16", what="sampled heads final")
    assert torch.isfinite(out.float()).all()


def test_many_short_sequences():
    """1100 packed sequences of 0 to 9 rows: the longest-first order is ranked in tiles of 1024."""
    lens = [(7 * i) % 10 for i in range(1100)]
    w = W.ssd_case(W.SsdSpec(H=2, P=64, N=64, G=1, state_dtype=torch.float32), lens, seed=39)
    check(w, gpu_ssd(w), oracle_ssd(w), "many sequences")


def test_graph_capture_and_bit_reproducibility():
    """Two eager calls and a CUDA-graph replay of the same call give bit-identical outputs and states."""
    w = W.ssd_case(W.SsdSpec(H=4, P=64, N=128, G=2), [70, 1, 130], seed=40)
    s = w.spec
    wd = w.to("cuda")
    cfg = gdn.SsdConfig(nheads=s.H, headdim=s.P, dstate=s.N, ngroups=s.G, state_dtype=s.state_dtype)
    ws = gdn.alloc_workspace(gdn.ssd_workspace_size(cfg, 3, w.T), "cuda")
    outs = [torch.empty((w.T, s.H, s.P), dtype=torch.bfloat16, device="cuda") for _ in range(3)]
    fins = [torch.empty_like(wd.init) for _ in range(3)]

    def call(k):
        gdn.ssd_combined_fwd(cfg, wd.x, wd.dt, wd.A, wd.B, wd.C, wd.cu, outs[k], ws, D=wd.D, z=wd.z,
                             dt_bias=wd.dt_bias, initial_states=wd.init, final_states=fins[k])

    call(0)
    call(1)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        with torch.cuda.graph(g, stream=side):
            call(2)
    g.replay()
    torch.cuda.synchronize()
    assert gdn.gdn_get_device_error(ws) == 0
    for k in (1, 2):
        assert torch.equal(outs[k].view(torch.int16), outs[0].view(torch.int16))
        assert torch.equal(fins[k].view(torch.int16), fins[0].view(torch.int16))
