"""EXTEND (prefill) parity: the CUDA path through the C ABI against the fp64
oracle on the same seeded inputs."""
import numpy as np
import pytest
import torch

import hybrid_linear_attention_causal_b200 as gdn
from hybrid_linear_attention_causal_b200 import workloads as W
from oracle import oracle as O
from tests.gpu_util import (check_extend, f64, gcfg, gpu_extend, ocfg, oracle_extend, restrict_to_group,
                            same_bits, to_device)
from tests.tolerances import assert_out_close, assert_state_close

pytestmark = pytest.mark.gpu


def test_tiny_fp32_extend_then_decode():
    """One sequence of 64 tokens from a zero state, then 8 decode steps (fp32)."""
    w = W.tiny_fp32()
    wd = to_device(w)
    gpu = gpu_extend(wd)
    ref = oracle_extend(w)
    check_extend(w, gpu, ref)
    _, conv, ssm, _ = gpu
    r_conv, r_ssm = ref[1], ref[2]
    xd, ad, bd = w.extra["decode"]
    cfg = gcfg(w.spec)
    ws = gdn.alloc_workspace(gdn.gdn_decode_workspace_size(cfg, 1), "cuda")
    for t in range(8):
        out = torch.empty(1, w.spec.HV, w.spec.dv, dtype=w.spec.dtype, device="cuda")
        gdn.gdn_decode(cfg, wd.params, xd[t:t + 1].cuda(), ad[t:t + 1].cuda(), bd[t:t + 1].cuda(),
                       wd.state_indices, conv, ssm, out, ws)
        r_out, r_conv, r_ssm = O.decode(ocfg(w.spec), w.params, xd[t:t + 1], ad[t:t + 1], bd[t:t + 1],
                                        w.state_indices, r_conv, r_ssm)
        torch.cuda.synchronize()
        assert_out_close(f64(out), r_out)
    assert gdn.gdn_get_device_error(ws) == 0
    assert_state_close(f64(ssm[3]), r_ssm[3])
    assert same_bits(conv[3], torch.from_numpy(r_conv[3]).float())


def _prefix_states(w: W.Workload):
    """Slot contents after running each request's prefix from zero (oracle)."""
    xp, ap, bp, cup = w.extra["prefix"]
    hi = torch.zeros(w.N, dtype=torch.int32)
    _, conv, ssm = O.extend(ocfg(w.spec), w.params, xp, ap, bp, cup, w.state_indices, w.conv_state, w.ssm_state,
                            has_initial_state=hi)
    conv_t = w.conv_state.clone()
    ssm_t = w.ssm_state.clone()
    for s, L in zip(w.state_indices.tolist(), w.extra["prefix_lens"]):
        if L > 0:
            conv_t[s] = torch.from_numpy(conv[s]).to(w.spec.dtype)
            ssm_t[s] = torch.from_numpy(ssm[s]).float()
    return conv_t, ssm_t


def test_ragged_varlen_bf16_with_real_prefix_states():
    """6 requests, prefixes U{0..300} run through the oracle into their slots,
    extends U{1..200}, 4/8 heads, dk = dv = 64, bf16 in / fp32 state."""
    w = W.ragged_varlen()
    conv_t, ssm_t = _prefix_states(w)
    w.conv_state, w.ssm_state = conv_t, ssm_t
    check_extend(w, gpu_extend(to_device(w)), oracle_extend(w))


def test_ragged_prefix_then_extend_on_gpu_equals_whole_sequence():
    """The GPU runs the prefixes, then the extends from the slots it wrote; the
    oracle runs each whole sequence from zero."""
    w = W.ragged_varlen()
    xp, ap, bp, cup = w.extra["prefix"]
    wd = to_device(w)
    hi0 = torch.zeros(w.N, dtype=torch.int32, device="cuda")
    wd_pref = to_device(w)
    wd_pref.has_initial_state = hi0
    _, conv1, ssm1, err = gpu_extend(wd_pref, x=xp.cuda(), a=ap.cuda(), b=bp.cuda(), cu=cup.cuda())
    assert err == 0
    out2, conv2, ssm2, err = gpu_extend(wd, conv_state=conv1, ssm_state=ssm1)
    assert err == 0
    # whole sequences for the oracle: prefix rows then extend rows, per request
    pl, el = w.extra["prefix_lens"], w.extra["extend_lens"]
    xs, as_, bs, lens, rows_ext = [], [], [], [], []
    pc, ec, off = 0, 0, 0
    for L0, L1 in zip(pl, el):
        xs += [xp[pc:pc + L0], w.x[ec:ec + L1]]
        as_ += [ap[pc:pc + L0], w.a[ec:ec + L1]]
        bs += [bp[pc:pc + L0], w.b[ec:ec + L1]]
        rows_ext.append(np.arange(off + L0, off + L0 + L1))
        lens.append(L0 + L1)
        pc, ec, off = pc + L0, ec + L1, off + L0 + L1
    cu = W.cu_from_lengths(lens, "cpu")
    r_out, r_conv, r_ssm = O.extend(ocfg(w.spec), w.params, torch.cat(xs), torch.cat(as_), torch.cat(bs), cu,
                                    w.state_indices, w.conv_state, w.ssm_state,
                                    has_initial_state=torch.zeros(w.N, dtype=torch.int32))
    assert_out_close(f64(out2), r_out[np.concatenate(rows_ext)])
    for s in w.state_indices.tolist():
        assert_state_close(f64(ssm2[s]), r_ssm[s])
        assert same_bits(conv2[s], torch.from_numpy(r_conv[s]).to(w.spec.dtype))


SHAPES = [
    (2, 2, 64, 64, torch.float32),
    (2, 4, 64, 64, torch.bfloat16),
    (1, 4, 128, 64, torch.bfloat16),
    (2, 2, 64, 128, torch.bfloat16),
    (2, 4, 128, 128, torch.bfloat16),
    (3, 3, 128, 128, torch.float32),
]


@pytest.mark.parametrize("HK,HV,dk,dv,dtype", SHAPES)
def test_edge_lengths_and_shapes(HK, HV, dk, dv, dtype):
    """Empty, single-row, chunk-boundary and multi-chunk sequences, a padded
    request and a request without initial state, on every supported (dk, dv)."""
    spec = W.LayerSpec(HK=HK, HV=HV, dk=dk, dv=dv, dtype=dtype)
    lengths = [1, 0, 63, 64, 65, 130, 3, 200]
    slots = [5, 7, -1, 0, 9, 2, 11, 3]
    hi = [1, 1, 1, 0, 1, 1, 0, 1]
    w = W.random_case(spec, lengths, P=12, seed=HK * 100 + dk + dv, has_init=hi, slots=slots)
    check_extend(w, gpu_extend(to_device(w)), oracle_extend(w))


@pytest.mark.parametrize("HK,HV,dk,dv,dtype", SHAPES)
def test_many_sequences(HK, HV, dk, dv, dtype):
    """More (sequence, head) state-pass CTAs than one wave of the SMs, with
    ragged lengths, padded and fresh requests: the longest-first launch order
    and the CTAs that start late."""
    spec = W.LayerSpec(HK=HK, HV=HV, dk=dk, dv=dv, dtype=dtype)
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    pattern = [1, 0, 63, 64, 65, 130, 3, 200, 17, 128, 5, 70]
    n = sms // (4 * HV) + 1
    lengths = (pattern * (n // len(pattern) + 1))[:n]
    hi = [(i % 3) != 1 for i in range(n)]
    slots = list(range(n))
    slots[2] = -1
    w = W.random_case(spec, lengths, P=n + 2, seed=HV * 10 + dk + dv, has_init=hi, slots=slots)
    check_extend(w, gpu_extend(to_device(w)), oracle_extend(w))


@pytest.mark.parametrize("lengths,slots,hi", [
    # 33000 packed rows -> 2 segments: long, medium, short, single-row, empty and padded requests
    ([16000, 12000, 4000, 1, 0, 999], [3, 0, 5, 1, 2, -1], [1, 0, 1, 1, 1, 1]),
    # one sequence of 49152 rows -> 3 segments, each continuing from the previous one's state
    ([49152], [2], [1]),
])
def test_segmented_batches(lengths, slots, hi):
    """Batches of 32768 packed rows or more run as several segments (the state
    pass of segment k alongside the per-chunk step of segment k+1, each segment a piece of
    the chunks listed longest sequence first); every sequence's chain must
    continue across the segment boundaries."""
    spec = W.LayerSpec(HK=2, HV=4, dk=128, dv=128, dtype=torch.bfloat16)
    w = W.random_case(spec, lengths, P=6, seed=sum(lengths), has_init=hi, slots=slots, a_mean=-2.0)
    check_extend(w, gpu_extend(to_device(w)), oracle_extend(w))


def test_page_shapes_with_nonzero_prefix_state():
    """The ragged page-boundary, exact-page and checkpoint-boundary shapes of the
    SGLang GDN test matrix (prefix (0,8,16) / extend (15,8,1); extend (16,);
    prefix (0,64,128) / extend (64,65,129)), here continuing from real states."""
    spec = W.LayerSpec(HK=2, HV=2, dk=128, dv=128, dtype=torch.bfloat16)
    for pref, ext in [((0, 8, 16), (15, 8, 1)), ((0,), (16,)), ((0, 64, 128), (64, 65, 129))]:
        base = W.random_case(spec, list(pref), P=6, seed=sum(ext), init_random=False,
                             has_init=[0] * len(pref))
        _, conv, ssm = oracle_extend(base)
        w = W.random_case(spec, list(ext), P=6, seed=sum(ext) + 1, init_random=False,
                          has_init=[1 if p > 0 else 0 for p in pref], slots=base.state_indices.tolist())
        w.params = base.params
        w.conv_state = base.conv_state.clone()
        w.ssm_state = base.ssm_state.clone()
        for s, p in zip(base.state_indices.tolist(), pref):
            if p > 0:
                w.conv_state[s] = torch.from_numpy(conv[s]).to(spec.dtype)
                w.ssm_state[s] = torch.from_numpy(ssm[s]).float()
        check_extend(w, gpu_extend(to_device(w)), oracle_extend(w))


def test_strong_decay_and_saturated_gates():
    """a ~ N(4, 1) drives g to about -20 per token; b large drives beta to 1."""
    spec = W.LayerSpec(HK=2, HV=4, dk=64, dv=64, dtype=torch.bfloat16)
    w = W.random_case(spec, [150, 70], P=4, seed=77, a_mean=4.0)
    w.b = (w.b.float() * 6.0).to(spec.dtype)
    check_extend(w, gpu_extend(to_device(w)), oracle_extend(w))


def test_large_prefill_full_size_sampled_groups():
    """32768 packed tokens, 8 sequences, 16/32 heads, d = 128 (the benchmark's
    prefill workload and launch configuration), checked on two qk-head groups
    (each with its 2 value heads) against the oracle, the rest by properties."""
    w = W.large_prefill(device="cuda")
    out, conv, ssm, err = gpu_extend(w)
    assert err == 0
    assert torch.isfinite(out.float()).all()
    G = w.spec.HV // w.spec.HK
    for hk in (0, 11):
        sub = restrict_to_group(w, hk)
        r_out, r_conv, r_ssm = oracle_extend(sub)
        assert_out_close(f64(out[:, hk * G:(hk + 1) * G]), r_out)
        for i, s in enumerate(sub.extra["slots"]):
            assert_state_close(f64(ssm[s, hk * G:(hk + 1) * G]), r_ssm[i], what=f"slot {s} group {hk}")
            want = torch.from_numpy(r_conv[i]).to(w.spec.dtype)
            assert same_bits(conv[s][sub.extra["cols"]].cpu(), want)
    # untouched pool slots keep the sentinel
    live = set(w.state_indices.tolist())
    for s in range(w.P):
        if s not in live:
            assert same_bits(ssm[s], w.ssm_state[s]) and same_bits(conv[s], w.conv_state[s])


def test_long_prefill_full_size_sampled_group():
    """One sequence of 262144 tokens continuing from a random state, checked on
    one qk-head group against the oracle."""
    w = W.long_prefill(device="cuda")
    out, conv, ssm, err = gpu_extend(w)
    assert err == 0
    hk, G = 5, w.spec.HV // w.spec.HK
    sub = restrict_to_group(w, hk)
    del w
    r_out, r_conv, r_ssm = oracle_extend(sub)
    assert_out_close(f64(out[:, hk * G:(hk + 1) * G]), r_out)
    assert_state_close(f64(ssm[1, hk * G:(hk + 1) * G]), r_ssm[0])
    assert same_bits(conv[1][sub.extra["cols"]].cpu(), torch.from_numpy(r_conv[0]).to(torch.bfloat16))


def test_device_error_flags():
    spec = W.LayerSpec(HK=2, HV=2, dk=64, dv=64, dtype=torch.bfloat16)
    w = W.random_case(spec, [10, 20], P=4, seed=3, slots=[1, 9])  # slot 9 >= P
    wd = to_device(w)
    out, conv, ssm, err = gpu_extend(wd)
    assert err & gdn.GDN_DEVERR_SLOT_RANGE
    assert torch.all(out[10:].float() == 0)
    ref = oracle_extend(W.random_case(spec, [10, 20], P=4, seed=3, slots=[1, -1]))
    assert_out_close(f64(out), ref[0])
    # malformed cu_seqlens: the batch is skipped and flagged, the pools untouched
    bad = torch.tensor([0, 25, 20], dtype=torch.int32, device="cuda")
    out, conv, ssm, err = gpu_extend(wd, cu=bad)
    assert err & gdn.GDN_DEVERR_SEQLENS
    assert same_bits(ssm, w.ssm_state) and same_bits(conv, w.conv_state)


def test_run_to_run_bit_reproducible():
    spec = W.LayerSpec(HK=2, HV=4, dk=128, dv=128, dtype=torch.bfloat16)
    wd = to_device(W.random_case(spec, [300, 5, 129], P=5, seed=21))
    a = gpu_extend(wd)
    b = gpu_extend(wd)
    assert same_bits(a[0], b[0]) and same_bits(a[1], b[1]) and same_bits(a[2], b[2])


def test_extend_captured_in_cuda_graph_matches_eager():
    spec = W.LayerSpec(HK=2, HV=4, dk=64, dv=128, dtype=torch.bfloat16)
    wd = to_device(W.random_case(spec, [100, 37, 64], P=6, seed=31))
    eager = gpu_extend(wd)
    cfg = gcfg(spec)
    ws = gdn.alloc_workspace(gdn.gdn_extend_workspace_size(cfg, wd.N, wd.T), "cuda")
    out = torch.empty(wd.T, spec.HV, spec.dv, dtype=spec.dtype, device="cuda")
    conv, ssm = wd.conv_state.clone(), wd.ssm_state.clone()
    s = torch.cuda.Stream()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            gdn.gdn_extend(cfg, wd.params, wd.x, wd.a, wd.b, wd.cu_seqlens, wd.state_indices, wd.has_initial_state,
                           conv, ssm, out, ws)
    conv.copy_(wd.conv_state)
    ssm.copy_(wd.ssm_state)
    g.replay()
    torch.cuda.synchronize()
    assert same_bits(out, eager[0]) and same_bits(conv, eager[1]) and same_bits(ssm, eager[2])


def gpu_extend_ckpt(wd, idx, rows, num):
    spec = wd.spec
    cfg = gcfg(spec)
    T, N = int(wd.x.shape[0]), int(wd.state_indices.shape[0])
    ws = gdn.alloc_workspace(gdn.gdn_extend_workspace_size(cfg, N, T), "cuda")
    out = torch.full((T, spec.HV, spec.dv), float("nan"), dtype=spec.dtype, device="cuda")
    conv, ssm = wd.conv_state.clone(), wd.ssm_state.clone()
    cks = W.sentinel_fill_(torch.empty(num, spec.HV, spec.dk, spec.dv, device="cuda"))
    ckc = W.sentinel_fill_(torch.empty(num, spec.conv_dim, spec.K - 1, dtype=spec.dtype, device="cuda"))
    gdn.gdn_extend_checkpoints(cfg, wd.params, wd.x, wd.a, wd.b, wd.cu_seqlens, wd.state_indices,
                               wd.has_initial_state, conv, ssm, out, idx.cuda(), rows.cuda(), cks, ckc, ws)
    torch.cuda.synchronize()
    return out, conv, ssm, cks, ckc, gdn.gdn_get_device_error(ws)


CKPT_SHAPES = [(2, 2, 64, 64, torch.float32), (4, 8, 128, 128, torch.bfloat16), (2, 4, 128, 64, torch.bfloat16),
               (1, 2, 64, 128, torch.bfloat16)]


@pytest.mark.parametrize("HK,HV,dk,dv,dtype", CKPT_SHAPES)
def test_extend_checkpoints_match_oracle(HK, HV, dk, dv, dtype):
    """Boundaries at a sequence's start, mid chunk (first and later chunks), on a chunk edge, at the
    end of a ragged sequence, on an empty sequence, disabled, and on a padded request: checkpoint
    states within the state tolerance of the oracle's, conv windows bit-exact, and the extend's own
    outputs and pools bit-identical to gdn_extend's."""
    spec = W.LayerSpec(HK=HK, HV=HV, dk=dk, dv=dv, dtype=dtype)
    lens = [130, 70, 0, 64, 200, 9, 100]
    slots = [3, 0, 6, 1, -1, 4, 2]
    w = W.random_case(spec, lens, P=8, seed=dk + 2 * dv + HV, slots=slots)
    w.has_initial_state = torch.tensor([1, 0, 1, 1, 1, 0, 1], dtype=torch.int32)
    cu = [int(v) for v in w.cu_seqlens]
    offs = [37, 70, 0, 64, 100, 0, -1]  # boundary inside each sequence; -1 disables
    idx = torch.tensor([cu[n] + o if o >= 0 else -1 for n, o in enumerate(offs)], dtype=torch.int32)
    rows = torch.tensor([1, 0, 2, 5, 3, 4, 6], dtype=torch.int32)
    wd = to_device(w)
    out, conv, ssm, cks, ckc, err = gpu_extend_ckpt(wd, idx, rows, 7)
    assert err == 0, f"device error word {err:#x}"
    b_out, b_conv, b_ssm, _ = gpu_extend(wd)
    assert same_bits(out, b_out) and same_bits(ssm, b_ssm) and same_bits(conv, b_conv)
    r_out, r_cs, r_ss, r_ck, r_ckc, code = O.extend_ckpt(ocfg(spec), w.params, w.x, w.a, w.b, w.cu_seqlens,
                                                         w.state_indices, w.conv_state, w.ssm_state, idx, rows, 7,
                                                         has_initial_state=w.has_initial_state)
    assert code == 0
    for n, o in enumerate(offs):
        r = int(rows[n])
        if o < 0 or slots[n] < 0:  # nothing captured: the sentinel is still there
            assert same_bits(cks[r], W.sentinel_fill_(torch.empty_like(cks[r])))
            continue
        assert_state_close(f64(cks[r]), r_ck[r], what=f"checkpoint of sequence {n}")
        assert same_bits(ckc[r], torch.from_numpy(r_ckc[r]).to(dtype)), f"conv checkpoint of sequence {n}"


def test_extend_checkpoints_cached_prefix_case():
    """Cached prefixes (0, 64, 128) extended by (64, 65, 129) rows, head dim 128, checkpoints on the
    last chunk edge and mid chunk: against the oracle's checkpoints of the whole sequences."""
    spec = W.LayerSpec(HK=2, HV=4, dk=128, dv=128, dtype=torch.bfloat16)
    prefix, ext = [0, 64, 128], [64, 65, 129]
    full = W.random_case(spec, [p + e for p, e in zip(prefix, ext)], P=4, seed=31)
    full.has_initial_state = torch.zeros(3, dtype=torch.int32)
    cu_f = [int(v) for v in full.cu_seqlens]
    pre_rows = [r for n in range(3) for r in range(cu_f[n], cu_f[n] + prefix[n])]
    ext_rows = [r for n in range(3) for r in range(cu_f[n] + prefix[n], cu_f[n + 1])]
    pr, er = torch.tensor(pre_rows, dtype=torch.long), torch.tensor(ext_rows, dtype=torch.long)
    # the prefixes' states (oracle) in the slots, then the extends on the GPU from them
    _, cs1, ss1 = O.extend(ocfg(spec), full.params, full.x[pr], full.a[pr], full.b[pr],
                           torch.tensor(np.cumsum([0] + prefix), dtype=torch.int32), full.state_indices,
                           full.conv_state, full.ssm_state, has_initial_state=full.has_initial_state)
    w = W.Workload(full.name, spec, full.params, full.x[er], full.a[er], full.b[er],
                   torch.tensor(np.cumsum([0] + ext), dtype=torch.int32), full.state_indices,
                   torch.tensor([1 if p > 0 else 0 for p in prefix], dtype=torch.int32),
                   torch.from_numpy(cs1).to(spec.dtype), torch.from_numpy(ss1).float(), {})
    cu_e = [int(v) for v in w.cu_seqlens]
    for offs in ([64, 64, 128], [13, 65, 100]):
        idx = torch.tensor([cu_e[n] + offs[n] for n in range(3)], dtype=torch.int32)
        out, conv, ssm, cks, ckc, err = gpu_extend_ckpt(to_device(w), idx, torch.arange(3, dtype=torch.int32), 3)
        assert err == 0
        for n in range(3):
            upto = prefix[n] + offs[n]
            rows = torch.arange(cu_f[n], cu_f[n] + upto)
            _, c_w, s_w = O.extend(ocfg(spec), full.params, full.x[rows], full.a[rows], full.b[rows],
                                   torch.tensor([0, upto], dtype=torch.int32), full.state_indices[n:n + 1],
                                   full.conv_state, full.ssm_state, has_initial_state=full.has_initial_state[n:n + 1])
            slot = int(full.state_indices[n])
            assert_state_close(f64(cks[n]), s_w[slot], what=f"checkpoint {n} at {offs[n]}")
            assert same_bits(ckc[n], torch.from_numpy(c_w[slot]).to(spec.dtype))


def test_extend_checkpoint_range_errors_flagged():
    spec = W.LayerSpec(HK=2, HV=4, dk=64, dv=64, dtype=torch.bfloat16)
    w = W.random_case(spec, [20, 30], P=4, seed=32)
    cu = [int(v) for v in w.cu_seqlens]
    idx = torch.tensor([cu[1] + 1, cu[1] + 5], dtype=torch.int32)  # the first lies in the second sequence
    out, conv, ssm, cks, ckc, err = gpu_extend_ckpt(to_device(w), idx, torch.tensor([0, 1], dtype=torch.int32), 2)
    assert err == gdn.GDN_DEVERR_CKPT_RANGE
    assert same_bits(cks[0], W.sentinel_fill_(torch.empty_like(cks[0])))
    r = O.extend_ckpt(ocfg(spec), w.params, w.x, w.a, w.b, w.cu_seqlens, w.state_indices, w.conv_state,
                      w.ssm_state, idx, torch.tensor([0, 1], dtype=torch.int32), 2)
    assert_state_close(f64(cks[1]), r[3][1])
