"""DECODE and TARGET_VERIFY parity: the CUDA path through the C ABI against
the fp64 oracle on the same seeded inputs."""
import numpy as np
import pytest
import torch

import hybrid_linear_attention_causal_b200 as gdn
from hybrid_linear_attention_causal_b200 import workloads as W
from oracle import oracle as O
from tests.gpu_util import f64, gcfg, ocfg, same_bits, to_device
from tests.tolerances import assert_out_close, assert_state_close

pytestmark = pytest.mark.gpu


def run_decode(wd, x, a, b, slots, conv, ssm):
    cfg = gcfg(wd.spec)
    ws = gdn.alloc_workspace(gdn.gdn_decode_workspace_size(cfg, int(slots.shape[0])), "cuda")
    out = torch.full((int(slots.shape[0]), wd.spec.HV, wd.spec.dv), float("nan"), dtype=wd.spec.dtype,
                     device="cuda")
    gdn.gdn_decode(cfg, wd.params, x, a, b, slots, conv, ssm, out, ws)
    torch.cuda.synchronize()
    return out, gdn.gdn_get_device_error(ws)


def run_verify(wd, x, a, b, slots, D, conv, ssm, want_conv_ckpt=True):
    cfg = gcfg(wd.spec)
    Bn = int(slots.shape[0])
    ws = gdn.alloc_workspace(gdn.gdn_verify_workspace_size(cfg, Bn, D), "cuda")
    out = torch.full((Bn * D, wd.spec.HV, wd.spec.dv), float("nan"), dtype=wd.spec.dtype, device="cuda")
    ck = W.sentinel_fill_(torch.empty(Bn, D, wd.spec.HV, wd.spec.dk, wd.spec.dv, device="cuda"))
    cck = (W.sentinel_fill_(torch.empty(Bn, D, wd.spec.conv_dim, 3, dtype=wd.spec.dtype, device="cuda"))
           if want_conv_ckpt else None)
    gdn.gdn_verify(cfg, wd.params, x, a, b, slots, D, conv, ssm, ck, cck, out, ws)
    torch.cuda.synchronize()
    return out, ck, cck, gdn.gdn_get_device_error(ws)


def _sample_oracle_decode(w, rows, pool_conv, pool_ssm):
    """Oracle decode of the requests in `rows` on a compact copy of their slots."""
    slots = [int(w.state_indices[r]) for r in rows]
    idx = torch.tensor(slots, dtype=torch.long)
    local = torch.arange(len(rows), dtype=torch.int32)
    ri = torch.tensor(rows, dtype=torch.long)
    return O.decode(ocfg(w.spec), w.params, w.x[ri], w.a[ri], w.b[ri], local, pool_conv[idx], pool_ssm[idx])


def test_decode_full_size_pool():
    """256 requests at random slots of a [1024, 32, 128, 128] pool, one token each
    (the benchmark's decode workload and launch configuration); 24 sampled
    requests checked against the oracle, the remaining slots checked untouched."""
    w = W.decode_verify(device="cpu")
    wd = to_device(w)
    conv, ssm = wd.conv_state.clone(), wd.ssm_state.clone()
    out, err = run_decode(wd, wd.x, wd.a, wd.b, wd.state_indices, conv, ssm)
    assert err == 0
    assert torch.isfinite(out.float()).all()
    rows = sorted(np.random.default_rng(0).choice(w.N, 24, replace=False).tolist())
    r_out, r_conv, r_ssm = _sample_oracle_decode(w, rows, w.conv_state, w.ssm_state)
    assert_out_close(f64(out[rows]), r_out)
    for i, r in enumerate(rows):
        s = int(w.state_indices[r])
        assert_state_close(f64(ssm[s]), r_ssm[i], what=f"slot {s}")
        assert same_bits(conv[s], torch.from_numpy(r_conv[i]).to(torch.bfloat16))
    named = torch.zeros(w.P, dtype=torch.bool)
    named[w.state_indices.long()] = True
    untouched = (~named).nonzero().flatten().cuda()
    assert same_bits(ssm[untouched], wd.ssm_state[untouched])
    assert same_bits(conv[untouched], wd.conv_state[untouched])


def test_verify_full_size_checkpoints():
    """The same pool, 4 draft tokens per request: checkpoints after every token,
    pools left bit-identical."""
    w = W.decode_verify(device="cpu")
    wd = to_device(w)
    D = w.extra["D"]
    xv, av, bv = w.extra["verify"]
    out, ck, cck, err = run_verify(wd, xv.cuda(), av.cuda(), bv.cuda(), wd.state_indices, D, wd.conv_state,
                                   wd.ssm_state)
    assert err == 0
    assert same_bits(wd.ssm_state, w.ssm_state.cuda()) and same_bits(wd.conv_state, w.conv_state.cuda())
    rows = sorted(np.random.default_rng(1).choice(w.N, 12, replace=False).tolist())
    slots = [int(w.state_indices[r]) for r in rows]
    idx = torch.tensor(slots, dtype=torch.long)
    tok = torch.tensor([r * D + t for r in rows for t in range(D)], dtype=torch.long)
    r_out, r_ck, r_cck = O.verify(ocfg(w.spec), w.params, xv[tok], av[tok], bv[tok],
                                  torch.arange(len(rows), dtype=torch.int32), D, w.conv_state[idx], w.ssm_state[idx])
    assert_out_close(f64(out[tok.cuda()]), r_out)
    for i, r in enumerate(rows):
        for t in range(D):
            assert_state_close(f64(ck[r, t]), r_ck[i, t], what=f"ckpt {r},{t}")
        assert same_bits(cck[r], torch.from_numpy(r_cck[i]).to(torch.bfloat16))


SHAPES = [
    (2, 2, 64, 64, torch.float32),
    (2, 4, 64, 64, torch.bfloat16),
    (1, 4, 128, 64, torch.bfloat16),
    (2, 2, 64, 128, torch.bfloat16),
    (4, 8, 128, 128, torch.bfloat16),
    (2, 8, 128, 128, torch.float32),
]


@pytest.mark.parametrize("HK,HV,dk,dv,dtype", SHAPES)
def test_decode_and_verify_shapes_with_padding(HK, HV, dk, dv, dtype):
    spec = W.LayerSpec(HK=HK, HV=HV, dk=dk, dv=dv, dtype=dtype)
    slots = [4, -1, 0, 6, 2]
    w = W.random_case(spec, [1] * len(slots), P=8, seed=dk + dv + HV, slots=slots)
    wd = to_device(w)
    conv, ssm = wd.conv_state.clone(), wd.ssm_state.clone()
    out, err = run_decode(wd, wd.x, wd.a, wd.b, wd.state_indices, conv, ssm)
    assert err == 0
    r_out, r_conv, r_ssm = O.decode(ocfg(spec), w.params, w.x, w.a, w.b, w.state_indices, w.conv_state,
                                    w.ssm_state)
    assert_out_close(f64(out), r_out)
    assert torch.all(out[1].float() == 0)
    for s in range(w.P):
        if s in slots:
            assert_state_close(f64(ssm[s]), r_ssm[s])
            assert same_bits(conv[s], torch.from_numpy(r_conv[s]).to(dtype))
        else:
            assert same_bits(ssm[s], w.ssm_state[s]) and same_bits(conv[s], w.conv_state[s])
    # verify, D = 3, from the original pools
    D = 3
    g = torch.Generator().manual_seed(5)
    xv = torch.randn(len(slots) * D, spec.conv_dim, generator=g).to(dtype)
    av = torch.randn(len(slots) * D, HV, generator=g).to(dtype)
    bv = torch.randn(len(slots) * D, HV, generator=g).to(dtype)
    out, ck, cck, err = run_verify(wd, xv.cuda(), av.cuda(), bv.cuda(), wd.state_indices, D, wd.conv_state,
                                   wd.ssm_state)
    assert err == 0
    r_out, r_ck, r_cck = O.verify(ocfg(spec), w.params, xv, av, bv, w.state_indices, D, w.conv_state, w.ssm_state)
    assert_out_close(f64(out), r_out)
    for i, s in enumerate(slots):
        if s < 0:
            assert torch.all(out[i * D:(i + 1) * D].float() == 0)
            continue
        for t in range(D):
            assert_state_close(f64(ck[i, t]), r_ck[i, t])
        assert same_bits(cck[i], torch.from_numpy(r_cck[i]).to(dtype))


def test_decode_slot_out_of_range_is_flagged_and_skipped():
    spec = W.LayerSpec(HK=2, HV=2, dk=64, dv=64, dtype=torch.bfloat16)
    w = W.random_case(spec, [1, 1], P=4, seed=9, slots=[2, 4])
    wd = to_device(w)
    conv, ssm = wd.conv_state.clone(), wd.ssm_state.clone()
    out, err = run_decode(wd, wd.x, wd.a, wd.b, wd.state_indices, conv, ssm)
    assert err & gdn.GDN_DEVERR_SLOT_RANGE
    assert torch.all(out[1].float() == 0)
    for s in (0, 1, 3):
        assert same_bits(ssm[s], w.ssm_state[s]) and same_bits(conv[s], w.conv_state[s])


def test_verify_long_draft_and_no_conv_checkpoint():
    spec = W.LayerSpec(HK=2, HV=4, dk=128, dv=128, dtype=torch.bfloat16)
    D = 16
    w = W.random_case(spec, [D, D], P=3, seed=12)
    wd = to_device(w)
    out, ck, cck, err = run_verify(wd, wd.x, wd.a, wd.b, wd.state_indices, D, wd.conv_state, wd.ssm_state,
                                   want_conv_ckpt=False)
    assert err == 0 and cck is None
    r_out, r_ck, _ = O.verify(ocfg(spec), w.params, w.x, w.a, w.b, w.state_indices, D, w.conv_state, w.ssm_state,
                              want_conv_ckpt=False)
    assert_out_close(f64(out), r_out)
    assert_state_close(f64(ck), r_ck)


def test_decode_and_verify_in_cuda_graph_with_padded_batch():
    """Capture with a fixed maximum batch whose tail is padding (-1), replay,
    and compare bit for bit with eager calls."""
    spec = W.LayerSpec(HK=4, HV=8, dk=128, dv=128, dtype=torch.bfloat16)
    slots = [3, 0, 5, -1, -1, -1]
    w = W.random_case(spec, [1] * len(slots), P=6, seed=40, slots=slots)
    wd = to_device(w)
    cfg = gcfg(spec)
    conv_e, ssm_e = wd.conv_state.clone(), wd.ssm_state.clone()
    out_e, _ = run_decode(wd, wd.x, wd.a, wd.b, wd.state_indices, conv_e, ssm_e)
    conv, ssm = wd.conv_state.clone(), wd.ssm_state.clone()
    out = torch.empty_like(out_e)
    ws = gdn.alloc_workspace(gdn.gdn_decode_workspace_size(cfg, len(slots)), "cuda")
    s = torch.cuda.Stream()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            gdn.gdn_decode(cfg, wd.params, wd.x, wd.a, wd.b, wd.state_indices, conv, ssm, out, ws)
    g.replay()
    torch.cuda.synchronize()
    assert same_bits(out, out_e) and same_bits(ssm, ssm_e) and same_bits(conv, conv_e)
    # verify graph
    D = 2
    xv = wd.x.repeat_interleave(D, 0).contiguous()
    av = wd.a.repeat_interleave(D, 0).contiguous()
    bv = wd.b.repeat_interleave(D, 0).contiguous()
    out_v, ck_v, cck_v, _ = run_verify(wd, xv, av, bv, wd.state_indices, D, wd.conv_state, wd.ssm_state)
    ws2 = gdn.alloc_workspace(gdn.gdn_verify_workspace_size(cfg, len(slots), D), "cuda")
    out2 = torch.empty_like(out_v)
    ck2 = ck_v.clone()
    cck2 = cck_v.clone()
    g2 = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        with torch.cuda.graph(g2, stream=s):
            gdn.gdn_verify(cfg, wd.params, xv, av, bv, wd.state_indices, D, wd.conv_state, wd.ssm_state, ck2, cck2,
                           out2, ws2)
    g2.replay()
    torch.cuda.synchronize()
    assert same_bits(out2, out_v) and same_bits(ck2, ck_v) and same_bits(cck2, cck_v)


def run_commit(wd, slots, accepted, D, ck, cck, conv, ssm):
    cfg = gcfg(wd.spec)
    ws = gdn.alloc_workspace(gdn.gdn_commit_workspace_size(cfg, int(slots.shape[0])), "cuda")
    gdn.gdn_commit(cfg, slots, accepted, D, ck, cck, conv, ssm, ws)
    torch.cuda.synchronize()
    return gdn.gdn_get_device_error(ws)


@pytest.mark.parametrize("HK,HV,dk,dv,dtype", [(2, 4, 64, 64, torch.float32), (4, 8, 128, 128, torch.bfloat16),
                                               (1, 4, 128, 64, torch.bfloat16)])
def test_commit_after_verify_equals_extend_of_accepted_prefix(HK, HV, dk, dv, dtype):
    """verify, then commit: each slot holds the checkpoint of its last accepted token (a copy, bit
    for bit) and matches the oracle's extend over the accepted prefix; zero accepted, padded and
    unnamed slots keep their bits."""
    spec = W.LayerSpec(HK=HK, HV=HV, dk=dk, dv=dv, dtype=dtype)
    D = 4
    slots = [5, -1, 0, 7, 2, 3]
    accepted = [1, 3, 0, 4, 2, 4]
    w = W.random_case(spec, [D] * len(slots), P=9, seed=dk + HV + 3, slots=slots)
    wd = to_device(w)
    out, ck, cck, err = run_verify(wd, wd.x, wd.a, wd.b, wd.state_indices, D, wd.conv_state, wd.ssm_state)
    assert err == 0
    conv, ssm = wd.conv_state.clone(), wd.ssm_state.clone()
    acc = torch.tensor(accepted, dtype=torch.int32, device="cuda")
    assert run_commit(wd, wd.state_indices, acc, D, ck, cck, conv, ssm) == 0
    touched = set()
    for i, (s, a) in enumerate(zip(slots, accepted)):
        if s < 0 or a == 0:
            continue
        touched.add(s)
        assert same_bits(ssm[s], ck[i, a - 1]) and same_bits(conv[s], cck[i, a - 1])
        rows = torch.arange(i * D, i * D + a)
        _, r_cs, r_ss = O.extend(ocfg(spec), w.params, w.x[rows], w.a[rows], w.b[rows],
                                 torch.tensor([0, a], dtype=torch.int32), torch.tensor([s], dtype=torch.int32),
                                 w.conv_state, w.ssm_state)
        assert_state_close(f64(ssm[s]), r_ss[s], what=f"slot {s}")
        assert same_bits(conv[s], torch.from_numpy(r_cs[s]).to(dtype))
    for s in range(9):
        if s not in touched:
            assert same_bits(ssm[s], wd.ssm_state[s]) and same_bits(conv[s], wd.conv_state[s])


def test_commit_full_size_pool_and_range_errors():
    """The decode-verify workload's pool: 256 requests commit 0..4 accepted tokens; then counts and
    slots out of range are flagged and skipped."""
    w = W.decode_verify(device="cpu")
    wd = to_device(w)
    D = w.extra["D"]
    xv, av, bv = w.extra["verify"]
    out, ck, cck, err = run_verify(wd, xv.cuda(), av.cuda(), bv.cuda(), wd.state_indices, D, wd.conv_state,
                                   wd.ssm_state)
    assert err == 0
    acc = torch.from_numpy(np.random.default_rng(3).integers(0, D + 1, w.N).astype(np.int32)).cuda()
    conv, ssm = wd.conv_state.clone(), wd.ssm_state.clone()
    assert run_commit(wd, wd.state_indices, acc, D, ck, cck, conv, ssm) == 0
    expect_ssm, expect_conv = wd.ssm_state.clone(), wd.conv_state.clone()
    for i in range(w.N):
        a = int(acc[i])
        if a > 0:
            s = int(w.state_indices[i])
            expect_ssm[s] = ck[i, a - 1]
            expect_conv[s] = cck[i, a - 1]
    assert same_bits(ssm, expect_ssm) and same_bits(conv, expect_conv)
    # an accepted count past D and a slot past the pool: both flagged, neither written
    bad_acc = acc.clone()
    bad_acc[0] = D + 1
    bad_slots = wd.state_indices.clone()
    bad_slots[1] = w.ssm_state.shape[0]
    conv2, ssm2 = wd.conv_state.clone(), wd.ssm_state.clone()
    err = run_commit(wd, bad_slots, bad_acc, D, ck, cck, conv2, ssm2)
    assert err == gdn.GDN_DEVERR_ACCEPT_RANGE | gdn.GDN_DEVERR_SLOT_RANGE
    s0 = int(w.state_indices[0])
    assert same_bits(ssm2[s0], wd.ssm_state[s0])


def run_verify_tree(wd, parents, D, want_conv_ckpt=True):
    cfg = gcfg(wd.spec)
    Bn = int(wd.state_indices.shape[0])
    ws = gdn.alloc_workspace(gdn.gdn_verify_workspace_size(cfg, Bn, D), "cuda")
    out = torch.full((Bn * D, wd.spec.HV, wd.spec.dv), float("nan"), dtype=wd.spec.dtype, device="cuda")
    ck = W.sentinel_fill_(torch.empty(Bn, D, wd.spec.HV, wd.spec.dk, wd.spec.dv, device="cuda"))
    cck = (W.sentinel_fill_(torch.empty(Bn, D, wd.spec.conv_dim, 3, dtype=wd.spec.dtype, device="cuda"))
           if want_conv_ckpt else None)
    gdn.gdn_verify_tree(cfg, wd.params, wd.x, wd.a, wd.b, wd.state_indices, parents.cuda(), D, wd.conv_state,
                        wd.ssm_state, ck, cck, out, ws)
    torch.cuda.synchronize()
    return out, ck, cck, gdn.gdn_get_device_error(ws)


@pytest.mark.parametrize("HK,HV,dk,dv,dtype", [(2, 4, 64, 64, torch.float32), (4, 8, 128, 128, torch.bfloat16),
                                               (1, 4, 128, 64, torch.bfloat16)])
def test_verify_tree_matches_oracle(HK, HV, dk, dv, dtype):
    """Branching draft trees (EAGLE topk 2 style) against the oracle's path replay; pools untouched."""
    spec = W.LayerSpec(HK=HK, HV=HV, dk=dk, dv=dv, dtype=dtype)
    D = 7
    slots = [2, -1, 0, 4]
    w = W.random_case(spec, [D] * 4, P=5, seed=dk + dv + 7, slots=slots)
    parents = torch.tensor([[-1, 0, 0, 1, 1, 2, 2], [-1, 0, 1, 2, 3, 4, 5], [-1, -1, 0, 1, 3, 4, 1],
                            [-1, 0, 1, 0, 3, -1, 5]], dtype=torch.int32)
    wd = to_device(w)
    out, ck, cck, err = run_verify_tree(wd, parents, D)
    assert err == 0
    assert same_bits(wd.ssm_state, w.ssm_state.cuda()) and same_bits(wd.conv_state, w.conv_state.cuda())
    r_out, r_ck, r_cck = O.verify_tree(ocfg(spec), w.params, w.x, w.a, w.b, w.state_indices, parents, D,
                                       w.conv_state, w.ssm_state)
    assert_out_close(f64(out), r_out)
    for i, s in enumerate(slots):
        if s < 0:
            continue
        for t in range(D):
            assert_state_close(f64(ck[i, t]), r_ck[i, t], what=f"ckpt {i},{t}")
            assert same_bits(cck[i, t], torch.from_numpy(r_cck[i, t]).to(dtype)), f"conv ckpt {i},{t}"


def test_verify_tree_chain_is_verify_bit_for_bit_and_bad_parent_flagged():
    spec = W.LayerSpec(HK=2, HV=4, dk=128, dv=128, dtype=torch.bfloat16)
    D = 6
    w = W.random_case(spec, [D] * 3, P=4, seed=33)
    wd = to_device(w)
    chain = torch.arange(-1, D - 1, dtype=torch.int32).repeat(3, 1)
    t_out, t_ck, t_cck, err = run_verify_tree(wd, chain, D)
    v_out, v_ck, v_cck, err2 = run_verify(wd, wd.x, wd.a, wd.b, wd.state_indices, D, wd.conv_state, wd.ssm_state)
    assert err == 0 and err2 == 0
    assert same_bits(t_out, v_out) and same_bits(t_ck, v_ck) and same_bits(t_cck, v_cck)
    bad = chain.clone()
    bad[1, 3] = 3  # a token cannot be its own parent
    b_out, b_ck, _, err = run_verify_tree(wd, bad, D)
    assert err == gdn.GDN_DEVERR_TREE
    assert torch.all(b_out[D:2 * D] == 0)  # that request is treated as padded
    assert same_bits(b_out[:D], v_out[:D]) and same_bits(b_ck[0], v_ck[0])
