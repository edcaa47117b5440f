"""Pins for the fp64 oracle: closed forms, invariants, library routines and
brute force, chosen so that a dropped term, a wrong sign or index, or a
transposed operand in the oracle fails at least one of them.  CPU only."""
from fractions import Fraction

import numpy as np
import pytest
import torch

from oracle import oracle as O

RNG = np.random.default_rng(1234)


def _unit_rows(L, d, rng=RNG):
    x = rng.standard_normal((L, d))
    return x / np.linalg.norm(x, axis=1, keepdims=True)


def _rand_case(L, dk, dv, rng=RNG, g_scale=0.5):
    q = _unit_rows(L, dk, rng)
    k = _unit_rows(L, dk, rng)
    v = rng.standard_normal((L, dv))
    g = -g_scale * rng.random(L)
    beta = rng.random(L)
    S0 = rng.standard_normal((dk, dv)) * 0.3
    return q, k, v, g, beta, S0


# ---------------------------------------------------------------- gates


def test_softplus_and_gates_spot_values():
    assert O.softplus(0.0) == pytest.approx(np.log(2.0), rel=1e-15)
    assert O.softplus(30.0) == 30.0  # linear branch above 20
    assert O.softplus(-30.0) == pytest.approx(np.exp(-30.0), rel=1e-12)
    assert O.softplus(1.5) == pytest.approx(np.logaddexp(0.0, 1.5), rel=1e-15)
    assert O.gate_beta(0.0) == 0.5
    assert O.gate_beta(2.0) == pytest.approx(1.0 / (1.0 + np.exp(-2.0)), rel=1e-15)
    # g = -exp(A_log) softplus(a + dt_bias)
    assert O.gate_g(0.0, 0.0, 0.0) == pytest.approx(-np.log(2.0), rel=1e-15)
    assert O.gate_g(np.log(3.0), 0.7, -0.2) == pytest.approx(-3.0 * np.logaddexp(0.0, 0.5), rel=1e-14)
    assert O.gate_g(-np.inf, 1.0, 0.0) == 0.0  # exp(-inf) = 0 removes the decay
    assert O.gate_beta(-np.inf) == 0.0


def test_l2norm_against_numpy():
    x = RNG.standard_normal(128) * 3.0
    y = O.l2norm(x, eps=0.0)
    np.testing.assert_allclose(y, x / np.linalg.norm(x), rtol=1e-15, atol=1e-16)
    # with eps the norm is sqrt(ss / (ss + eps))
    ss = float(np.dot(x, x))
    y = O.l2norm(x, eps=1e-6)
    assert np.linalg.norm(y) == pytest.approx(np.sqrt(ss / (ss + 1e-6)), rel=1e-14)


# ---------------------------------------------------------------- conv


def _silu(z):
    return z / (1.0 + np.exp(-z))


def test_conv_identity_and_shift():
    L, C, K = 9, 5, 4
    x = RNG.standard_normal((L, C))
    hist = RNG.standard_normal((C, K - 1))
    w_id = np.zeros((C, K)); w_id[:, K - 1] = 1.0
    np.testing.assert_allclose(O.conv_silu(x, w_id, hist), _silu(x), rtol=1e-15)
    # weight on the oldest tap: y_t = SiLU(x_{t-3}), reaching into the history for t < 3
    w_old = np.zeros((C, K)); w_old[:, 0] = 1.0
    full = np.concatenate([hist.T, x], axis=0)  # rows -3..L-1
    np.testing.assert_allclose(O.conv_silu(x, w_old, hist), _silu(full[:L]), rtol=1e-15)
    # no history means zeros
    y0 = O.conv_silu(x, w_old, None)
    np.testing.assert_allclose(y0[:3], _silu(np.zeros((3, C))), rtol=0, atol=0)


def test_conv_matches_numpy_convolve():
    L, C, K = 17, 6, 4
    x = RNG.standard_normal((L, C))
    hist = RNG.standard_normal((C, K - 1))
    w = RNG.standard_normal((C, K))
    bias = RNG.standard_normal(C)
    y = O.conv_silu(x, w, hist, bias)
    for c in range(C):
        seq = np.concatenate([hist[c], x[:, c]])
        # cross-correlation == convolution with the reversed kernel
        ref = np.convolve(seq, w[c, ::-1], mode="valid") + bias[c]
        np.testing.assert_allclose(y[:, c], _silu(ref), rtol=1e-13, atol=1e-14)


# ---------------------------------------------------------------- core recurrence


def test_beta0_g0_leaves_state_and_reads_it():
    L, dk, dv = 7, 5, 3
    q, k, v, _, _, S0 = _rand_case(L, dk, dv)
    g = np.zeros(L); beta = np.zeros(L)
    o, S = O.core_recurrent(q, k, v, g, beta, S0, scale=0.37)
    np.testing.assert_array_equal(S, S0)
    np.testing.assert_allclose(o, 0.37 * q @ S0, rtol=1e-14, atol=1e-15)


def test_beta0_pure_decay():
    L, dk, dv = 6, 4, 3
    q, k, v, g, _, S0 = _rand_case(L, dk, dv)
    beta = np.zeros(L)
    o, S = O.core_recurrent(q, k, v, g, beta, S0, scale=1.0)
    np.testing.assert_allclose(S, np.exp(g.sum()) * S0, rtol=1e-14)
    gam = np.cumsum(g)
    np.testing.assert_allclose(o, np.exp(gam)[:, None] * (q @ S0), rtol=1e-13)


def test_strong_decay_resets_state():
    L, dk, dv = 4, 5, 3
    q, k, v, _, beta, S0 = _rand_case(L, dk, dv)
    S0 = S0 * 1e3
    g = np.full(L, -1e4)  # exp(-1e4) underflows to exactly 0
    o, S, st = O.core_recurrent(q, k, v, g, beta, S0, scale=0.5, return_states=True)
    for t in range(L):
        np.testing.assert_allclose(st[t], beta[t] * np.outer(k[t], v[t]), rtol=1e-14, atol=1e-300)
        np.testing.assert_allclose(o[t], 0.5 * beta[t] * np.dot(q[t], k[t]) * v[t], rtol=1e-13)


@pytest.mark.parametrize("nkeys", [3, 8])
def test_associative_recall_with_orthonormal_keys(nkeys):
    dk, dv = 8, 5
    Qm, _ = np.linalg.qr(RNG.standard_normal((dk, dk)))
    k = Qm[:, :nkeys].T.copy()  # orthonormal rows
    v = RNG.standard_normal((nkeys, dv))
    S0 = RNG.standard_normal((dk, dv))
    g = np.zeros(nkeys); beta = np.ones(nkeys)
    _, S = O.core_recurrent(k, k, v, g, beta, S0, scale=1.0)
    np.testing.assert_allclose(k @ S, v, rtol=1e-12, atol=1e-12)
    # directions orthogonal to every written key keep the old content
    if nkeys < dk:
        rest = Qm[:, nkeys:].T
        np.testing.assert_allclose(rest @ S, rest @ S0, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("L,dk,dv", [(1, 3, 2), (5, 4, 3), (8, 6, 7)])
def test_bruteforce_product_form(L, dk, dv):
    q, k, v, g, beta, S0 = _rand_case(L, dk, dv)
    o_bf, S_step, S_sum = O.core_bruteforce(q, k, v, g, beta, S0, scale=0.3)
    o, S = O.core_recurrent(q, k, v, g, beta, S0, scale=0.3)
    np.testing.assert_allclose(S_step, S_sum, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(S, S_step, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(o, o_bf, rtol=1e-12, atol=1e-13)


def test_exact_rational_tiny_case():
    """dk = dv = 2, beta = 1/2, g = 0, unit keys with rational entries: the
    defining product S_t = (I - b k k^T) S_{t-1} + b k v^T in exact arithmetic."""
    F = Fraction
    ks = [(F(3, 5), F(4, 5)), (F(1), F(0)), (F(-4, 5), F(3, 5))]
    vs = [(F(1), F(-2)), (F(1, 2), F(3)), (F(-1), F(1, 4))]
    qs = [(F(0), F(1)), (F(3, 5), F(-4, 5)), (F(1), F(0))]
    b = F(1, 2)
    S = [[F(1, 3), F(0)], [F(-1), F(2)]]
    outs = []
    for kt, vt, qt in zip(ks, vs, qs):
        A = [[(1 if r == c else 0) - b * kt[r] * kt[c] for c in range(2)] for r in range(2)]
        S = [[sum(A[r][m] * S[m][j] for m in range(2)) + b * kt[r] * vt[j] for j in range(2)] for r in range(2)]
        outs.append([sum(qt[r] * S[r][j] for r in range(2)) for j in range(2)])
    f = lambda m: np.array([[float(e) for e in row] for row in m])
    o, Sf = O.core_recurrent(f(qs), f(ks), f(vs), np.zeros(3), np.full(3, 0.5), np.array([[1 / 3, 0], [-1, 2]]), 1.0)
    np.testing.assert_allclose(Sf, f(S), rtol=1e-15, atol=1e-15)
    np.testing.assert_allclose(o, f(outs), rtol=1e-15, atol=1e-15)


@pytest.mark.parametrize("C", [1, 3, 16, 64])
@pytest.mark.parametrize("L", [1, 63, 64, 65, 200])
def test_chunked_equals_recurrent(C, L):
    dk, dv = 8, 6
    q, k, v, g, beta, S0 = _rand_case(L, dk, dv, g_scale=3.0)
    o1, S1 = O.core_recurrent(q, k, v, g, beta, S0, scale=0.25)
    o2, S2 = O.core_chunked(q, k, v, g, beta, S0, scale=0.25, chunk=C)
    np.testing.assert_allclose(o2, o1, rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(S2, S1, rtol=1e-10, atol=1e-12)


def test_chunked_strong_decay_is_finite():
    # g down to about -20 per token: exp(gamma_r - gamma_s) is formed from differences
    L, dk, dv = 130, 8, 4
    q, k, v, _, beta, S0 = _rand_case(L, dk, dv)
    g = -RNG.random(L) * 20.0
    o1, S1 = O.core_recurrent(q, k, v, g, beta, S0, scale=1.0)
    o2, S2 = O.core_chunked(q, k, v, g, beta, S0, scale=1.0, chunk=64)
    assert np.isfinite(o2).all() and np.isfinite(S2).all()
    np.testing.assert_allclose(o2, o1, rtol=1e-9, atol=1e-12)


# ---------------------------------------------------------------- the layer

CFG = O.OracleCfg(HK=2, HV=4, dk=8, dv=6)


def _layer_case(lengths, P=6, seed=0, cfg=CFG, dtype=torch.float32):
    from hybrid_linear_attention_causal_b200.workloads import LayerSpec, random_case

    spec = LayerSpec(HK=cfg.HK, HV=cfg.HV, dk=cfg.dk, dv=cfg.dv, dtype=dtype)
    return random_case(spec, lengths, P=P, seed=seed)


def _run(w, **kw):
    return O.extend(CFG if "cfg" not in kw else kw.pop("cfg"), w.params, w.x, w.a, w.b, w.cu_seqlens,
                    w.state_indices, w.conv_state, w.ssm_state, has_initial_state=w.has_initial_state, **kw)


def test_layer_chunked_equals_recurrent():
    w = _layer_case([70, 1, 0, 130], seed=3)
    o1, c1, s1 = _run(w)
    o2, c2, s2 = _run(w, chunk=64)
    np.testing.assert_allclose(o2, o1, rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(s2, s1, rtol=1e-10, atol=1e-12)
    np.testing.assert_array_equal(c2, c1)


@pytest.mark.parametrize("split", [1, 2, 3, 40])
def test_prefix_then_extend_equals_whole(split):
    w = _layer_case([57], seed=5)
    out, cs, ss = _run(w)
    cu1 = torch.tensor([0, split], dtype=torch.int32)
    cu2 = torch.tensor([0, 57 - split], dtype=torch.int32)
    o1, cs1, ss1 = O.extend(CFG, w.params, w.x[:split], w.a[:split], w.b[:split], cu1, w.state_indices,
                            w.conv_state, w.ssm_state)
    o2, cs2, ss2 = O.extend(CFG, w.params, w.x[split:], w.a[split:], w.b[split:], cu2, w.state_indices, cs1, ss1)
    np.testing.assert_allclose(np.concatenate([o1, o2]), out, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(ss2, ss, rtol=1e-12, atol=1e-13)
    np.testing.assert_array_equal(cs2, cs)


def test_decode_steps_equal_extend():
    w = _layer_case([8], seed=6)
    out, cs, ss = _run(w)
    c, s = w.conv_state, w.ssm_state
    for t in range(8):
        o, c, s = O.decode(CFG, w.params, w.x[t:t + 1], w.a[t:t + 1], w.b[t:t + 1], w.state_indices, c, s)
        np.testing.assert_allclose(o[0], out[t], rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(s, ss, rtol=1e-12, atol=1e-13)
    np.testing.assert_array_equal(c, cs)


def test_verify_checkpoints_and_read_only_pools():
    D = 5
    w = _layer_case([D, D, D], seed=7)
    slots = w.state_indices.clone()
    slots[1] = -1  # a padded request
    out, ck, cck = O.verify(CFG, w.params, w.x, w.a, w.b, slots, D, w.conv_state, w.ssm_state)
    assert np.all(out[D:2 * D] == 0)
    for i in (0, 2):
        for t in range(D):
            cu = torch.tensor([0, t + 1], dtype=torch.int32)
            rows = slice(i * D, i * D + t + 1)
            o_e, c_e, s_e = O.extend(CFG, w.params, w.x[rows], w.a[rows], w.b[rows], cu, slots[i:i + 1],
                                     w.conv_state, w.ssm_state)
            slot = int(slots[i])
            np.testing.assert_allclose(ck[i, t], s_e[slot], rtol=1e-12, atol=1e-13)
            np.testing.assert_array_equal(cck[i, t], c_e[slot])
            np.testing.assert_allclose(out[i * D + t], o_e[t], rtol=1e-12, atol=1e-13)


def test_commit_equals_extend_of_the_accepted_prefix():
    """verify, then commit(a), leaves each slot as an extend over the request's first a draft
    tokens would; a = 0 and padded requests leave their slots alone."""
    D = 4
    w = _layer_case([D] * 5, P=8, seed=11)
    slots = w.state_indices.clone()
    slots[3] = -1  # padding
    accepted = np.array([1, 4, 0, 2, 3], dtype=np.int32)
    out, ck, cck = O.verify(CFG, w.params, w.x, w.a, w.b, slots, D, w.conv_state, w.ssm_state)
    cs, ss, code = O.commit(CFG, slots, accepted, D, ck, cck, w.conv_state, w.ssm_state)
    assert code == 0
    for i in range(5):
        slot = int(slots[i])
        if slot < 0:
            continue
        if accepted[i] == 0:
            np.testing.assert_array_equal(ss[slot], O._f64(w.ssm_state)[slot])
            np.testing.assert_array_equal(cs[slot], O._f64(w.conv_state)[slot])
            continue
        rows = slice(i * D, i * D + int(accepted[i]))
        cu = torch.tensor([0, int(accepted[i])], dtype=torch.int32)
        _, c_e, s_e = O.extend(CFG, w.params, w.x[rows], w.a[rows], w.b[rows], cu, slots[i:i + 1], w.conv_state,
                               w.ssm_state)
        np.testing.assert_allclose(ss[slot], s_e[slot], rtol=1e-12, atol=1e-13)
        np.testing.assert_array_equal(cs[slot], c_e[slot])
    # slots no request names are untouched
    named = {int(x) for x in slots if int(x) >= 0}
    for sl in range(8):
        if sl not in named:
            np.testing.assert_array_equal(ss[sl], O._f64(w.ssm_state)[sl])


def test_commit_rejects_out_of_range_counts():
    D = 3
    w = _layer_case([D, D], P=4, seed=12)
    out, ck, cck = O.verify(CFG, w.params, w.x, w.a, w.b, w.state_indices, D, w.conv_state, w.ssm_state)
    cs, ss, code = O.commit(CFG, w.state_indices, np.array([D + 1, 2], dtype=np.int32), D, ck, cck, w.conv_state,
                            w.ssm_state)
    assert code == 3
    s0 = int(w.state_indices[0])
    np.testing.assert_array_equal(ss[s0], O._f64(w.ssm_state)[s0])  # the bad request wrote nothing
    np.testing.assert_array_equal(ss[int(w.state_indices[1])], ck[1, 1])


def test_extend_checkpoints_equal_extends_of_the_prefixes():
    """A checkpoint at boundary b of sequence n is the slot state (and conv window) that extending
    only rows cu[n] .. b-1 leaves; the boundary may sit at the start, mid chunk, on a chunk edge or at
    the end; checkpointing leaves the outputs and pools of the extend unchanged."""
    lens = [70, 130, 5, 64, 40]
    w = _layer_case(lens, P=8, seed=13)
    w.has_initial_state = torch.tensor([1, 0, 0, 1, 1], dtype=torch.int32)
    cu = [int(v) for v in w.cu_seqlens]
    offs = [37, 64, 0, 64, -1]  # boundary offsets inside each sequence; -1 disables
    idx = torch.tensor([cu[n] + o if o >= 0 else -1 for n, o in enumerate(offs)], dtype=torch.int32)
    rows_of = torch.tensor([2, 0, 3, 1, 4], dtype=torch.int32)
    out, cs, ss, ck, ckc, code = O.extend_ckpt(CFG, w.params, w.x, w.a, w.b, w.cu_seqlens, w.state_indices,
                                               w.conv_state, w.ssm_state, idx, rows_of, 5,
                                               has_initial_state=w.has_initial_state)
    assert code == 0
    o_ref, cs_ref, ss_ref = _run(w)
    np.testing.assert_array_equal(out, o_ref)
    np.testing.assert_array_equal(ss, ss_ref)
    np.testing.assert_array_equal(cs, cs_ref)
    for n, o in enumerate(offs):
        r = int(rows_of[n])
        if o < 0:
            assert not ck[r].any() and not ckc[r].any()
            continue
        sl = w.state_indices[n:n + 1]
        rows = slice(cu[n], cu[n] + o)
        _, c_p, s_p = O.extend(CFG, w.params, w.x[rows], w.a[rows], w.b[rows],
                               torch.tensor([0, o], dtype=torch.int32), sl, w.conv_state, w.ssm_state,
                               has_initial_state=w.has_initial_state[n:n + 1])
        slot = int(sl[0])
        if o == 0:  # nothing run: the slot as the sequence found it (zeros without an initial state)
            init = bool(w.has_initial_state[n])
            np.testing.assert_array_equal(ck[r], O._f64(w.ssm_state)[slot] * init)
            np.testing.assert_array_equal(ckc[r], O._f64(w.conv_state)[slot] * init)
        else:
            np.testing.assert_allclose(ck[r], s_p[slot], rtol=1e-12, atol=1e-13)
            np.testing.assert_array_equal(ckc[r], c_p[slot])
    # the end of a sequence is its final state
    n = 1
    _, _, _, ck2, _, _ = O.extend_ckpt(CFG, w.params, w.x, w.a, w.b, w.cu_seqlens, w.state_indices, w.conv_state,
                                       w.ssm_state, torch.tensor([-1, cu[2], -1, -1, -1], dtype=torch.int32),
                                       torch.tensor([-1, 0, -1, -1, -1], dtype=torch.int32), 1,
                                       has_initial_state=w.has_initial_state)
    np.testing.assert_allclose(ck2[0], ss_ref[int(w.state_indices[n])], rtol=1e-12, atol=1e-13)


def test_extend_checkpoints_prefix_cache_case():
    """Cached prefixes (0, 64, 128) continued by extends (64, 65, 129) with a checkpoint on the last
    chunk edge of each extend: the checkpoint equals the state after the whole-sequence prefix."""
    prefix, ext = [0, 64, 128], [64, 65, 129]
    full = _layer_case([p + e for p, e in zip(prefix, ext)], P=4, seed=14)
    full.has_initial_state = torch.tensor([0, 1, 1], dtype=torch.int32)
    xs, a_s, bs, pre_rows, ext_rows = [], [], [], [], []
    cu_full = [int(v) for v in full.cu_seqlens]
    for n in range(3):
        pre_rows += list(range(cu_full[n], cu_full[n] + prefix[n]))
        ext_rows += list(range(cu_full[n] + prefix[n], cu_full[n + 1]))
    pr, er = torch.tensor(pre_rows, dtype=torch.long), torch.tensor(ext_rows, dtype=torch.long)
    cu_pre = torch.tensor(np.cumsum([0] + prefix), dtype=torch.int32)
    cu_ext = torch.tensor(np.cumsum([0] + ext), dtype=torch.int32)
    _, cs1, ss1 = O.extend(CFG, full.params, full.x[pr], full.a[pr], full.b[pr], cu_pre, full.state_indices,
                           full.conv_state, full.ssm_state, has_initial_state=full.has_initial_state)
    # after the prefix the slots hold the prefix state; the extend starts from it
    hi = torch.ones(3, dtype=torch.int32)
    bnd = [int(cu_ext[n]) + (ext[n] // 64) * 64 for n in range(3)]
    out, cs2, ss2, ck, ckc, code = O.extend_ckpt(CFG, full.params, full.x[er], full.a[er], full.b[er], cu_ext,
                                                 full.state_indices, cs1, ss1, torch.tensor(bnd, dtype=torch.int32),
                                                 torch.arange(3, dtype=torch.int32), 3, has_initial_state=hi)
    assert code == 0
    for n in range(3):
        upto = prefix[n] + (ext[n] // 64) * 64
        rows = slice(cu_full[n], cu_full[n] + upto)
        _, c_w, s_w = O.extend(CFG, full.params, full.x[rows], full.a[rows], full.b[rows],
                               torch.tensor([0, upto], dtype=torch.int32), full.state_indices[n:n + 1],
                               full.conv_state, full.ssm_state, has_initial_state=full.has_initial_state[n:n + 1])
        slot = int(full.state_indices[n])
        np.testing.assert_allclose(ck[n], s_w[slot], rtol=1e-11, atol=1e-12)
        np.testing.assert_array_equal(ckc[n], c_w[slot])


def test_extend_checkpoint_ranges():
    w = _layer_case([20, 30], P=4, seed=15)
    cu = [int(v) for v in w.cu_seqlens]
    assert w.has_initial_state is None  # every slot holds a starting state
    *_, code = O.extend_ckpt(CFG, w.params, w.x, w.a, w.b, w.cu_seqlens, w.state_indices, w.conv_state,
                             w.ssm_state, torch.tensor([cu[1] + 1, cu[1]], dtype=torch.int32),
                             torch.tensor([0, 1], dtype=torch.int32), 2, has_initial_state=w.has_initial_state)
    assert code == 4  # the first boundary lies in the second sequence
    *_, ck, _, code = O.extend_ckpt(CFG, w.params, w.x, w.a, w.b, w.cu_seqlens, w.state_indices, w.conv_state,
                                    w.ssm_state, torch.tensor([5, cu[1] + 3], dtype=torch.int32),
                                    torch.tensor([0, 2], dtype=torch.int32), 2, has_initial_state=w.has_initial_state)
    assert code == 4 and ck[0].any() and not ck[1].any()  # row 2 >= 2 rows: skipped


def test_verify_tree_chain_equals_verify_and_star_equals_decodes():
    """A chain tree (parent t-1) is verify; a star (every parent the slot) is D independent decodes
    from the slot."""
    D = 5
    w = _layer_case([D, D, D], P=5, seed=16)
    slots = w.state_indices.clone()
    slots[1] = -1
    chain = np.tile(np.arange(-1, D - 1, dtype=np.int32), (3, 1))
    o_t, ck_t, cc_t = O.verify_tree(CFG, w.params, w.x, w.a, w.b, slots, chain, D, w.conv_state, w.ssm_state)
    o_v, ck_v, cc_v = O.verify(CFG, w.params, w.x, w.a, w.b, slots, D, w.conv_state, w.ssm_state)
    np.testing.assert_allclose(o_t, o_v, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(ck_t[[0, 2]], ck_v[[0, 2]], rtol=1e-12, atol=1e-13)
    np.testing.assert_array_equal(cc_t[[0, 2]], cc_v[[0, 2]])
    star = np.full((3, D), -1, dtype=np.int32)
    o_s, ck_s, cc_s = O.verify_tree(CFG, w.params, w.x, w.a, w.b, slots, star, D, w.conv_state, w.ssm_state)
    for i in (0, 2):
        for t in range(D):
            r = slice(i * D + t, i * D + t + 1)
            o_d, c_d, s_d = O.decode(CFG, w.params, w.x[r], w.a[r], w.b[r], slots[i:i + 1], w.conv_state,
                                     w.ssm_state)
            sl = int(slots[i])
            np.testing.assert_allclose(o_s[i * D + t], o_d[0], rtol=1e-12, atol=1e-13)
            np.testing.assert_allclose(ck_s[i, t], s_d[sl], rtol=1e-12, atol=1e-13)
            np.testing.assert_array_equal(cc_s[i, t], c_d[sl])


def test_verify_tree_node_is_one_step_from_its_parent():
    """In a branching tree every node's state is one decode step, with its own token, from its
    parent's checkpoint (the slot for the root's children)."""
    D = 7
    w = _layer_case([D, D], P=3, seed=17)
    parents = np.array([[-1, 0, 0, 1, 1, 2, -1], [-1, -1, 1, 2, 0, 4, 3]], dtype=np.int32)
    o, ck, cc = O.verify_tree(CFG, w.params, w.x, w.a, w.b, w.state_indices, parents, D, w.conv_state,
                              w.ssm_state)
    for i in range(2):
        sl = int(w.state_indices[i])
        for t in range(D):
            pool_s, pool_c = O._f64(w.ssm_state).copy(), O._f64(w.conv_state).copy()
            pt = int(parents[i, t])
            if pt >= 0:
                pool_s[sl], pool_c[sl] = ck[i, pt], cc[i, pt]
            r = slice(i * D + t, i * D + t + 1)
            o_d, c_d, s_d = O.decode(CFG, w.params, w.x[r], w.a[r], w.b[r], w.state_indices[i:i + 1], pool_c, pool_s)
            np.testing.assert_allclose(ck[i, t], s_d[sl], rtol=1e-11, atol=1e-12)
            np.testing.assert_allclose(o[i * D + t], o_d[0], rtol=1e-11, atol=1e-12)
            np.testing.assert_array_equal(cc[i, t], c_d[sl])


def test_head_independence_and_gqa_mapping():
    w = _layer_case([23, 9], seed=8)
    base, _, _ = _run(w)
    G = CFG.HV // CFG.HK
    qk = CFG.HK * CFG.dk
    # perturb the v channels of value head 3: only head 3 moves
    x = w.x.clone(); x[:, 2 * qk + 3 * CFG.dv: 2 * qk + 4 * CFG.dv] += 0.5
    w2 = _layer_case([23, 9], seed=8); w2.x = x
    o, _, _ = _run(w2)
    moved = [h for h in range(CFG.HV) if not np.allclose(o[:, h], base[:, h], rtol=0, atol=0)]
    assert moved == [3]
    # perturb the k channels of qk head 1: exactly the value heads h with h // G == 1 move
    x = w.x.clone(); x[:, qk + 1 * CFG.dk: qk + 2 * CFG.dk] += 0.5
    w2.x = x
    o, _, _ = _run(w2)
    moved = [h for h in range(CFG.HV) if not np.allclose(o[:, h], base[:, h], rtol=0, atol=0)]
    assert moved == [h for h in range(CFG.HV) if h // G == 1]
    # perturb a of head 0: only head 0 moves
    a = w.a.clone(); a[:, 0] += 1.0
    w3 = _layer_case([23, 9], seed=8); w3.a = a
    o, _, _ = _run(w3)
    moved = [h for h in range(CFG.HV) if not np.allclose(o[:, h], base[:, h], rtol=0, atol=0)]
    assert moved == [0]


def test_gqa_equals_mha_with_duplicated_qk_heads():
    """A G=2 layer equals a G=1 layer whose qk heads are the G=2 layer's qk
    heads repeated per value head (q/k channels and conv weights copied)."""
    w = _layer_case([31], seed=9)
    out, _, ss = _run(w)
    mha = O.OracleCfg(HK=CFG.HV, HV=CFG.HV, dk=CFG.dk, dv=CFG.dv)
    G = CFG.HV // CFG.HK
    qk = CFG.HK * CFG.dk

    def remap(rows):  # rows: [..., conv_dim] for the G=2 layout -> MHA layout
        q = [rows[..., (h // G) * CFG.dk:(h // G + 1) * CFG.dk] for h in range(CFG.HV)]
        k = [rows[..., qk + (h // G) * CFG.dk: qk + (h // G + 1) * CFG.dk] for h in range(CFG.HV)]
        return torch.cat(q + k + [rows[..., 2 * qk:]], dim=-1)

    params = dict(w.params)
    params["conv_w"] = remap(w.params["conv_w"].T).T.contiguous()
    cs = remap(w.conv_state.transpose(1, 2)).transpose(1, 2).contiguous()
    o2, _, ss2 = O.extend(mha, params, remap(w.x), w.a, w.b, w.cu_seqlens, w.state_indices, cs, w.ssm_state,
                          has_initial_state=w.has_initial_state)
    np.testing.assert_allclose(o2, out, rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(ss2, ss, rtol=1e-13, atol=1e-14)


def test_permuting_value_columns_permutes_state_and_output():
    w = _layer_case([19], seed=10)
    out, _, ss = _run(w)
    perm = torch.from_numpy(RNG.permutation(CFG.dv))
    qk = 2 * CFG.HK * CFG.dk
    cols = torch.arange(CFG.conv_dim)
    for h in range(CFG.HV):
        cols[qk + h * CFG.dv: qk + (h + 1) * CFG.dv] = qk + h * CFG.dv + perm
    w2 = _layer_case([19], seed=10)
    w2.x = w.x[:, cols]
    w2.params = dict(w.params); w2.params["conv_w"] = w.params["conv_w"][cols]
    w2.conv_state = w.conv_state[:, cols]
    w2.ssm_state = w.ssm_state[..., perm]
    o2, _, ss2 = _run(w2)
    np.testing.assert_allclose(o2, out[..., perm.numpy()], rtol=1e-13, atol=1e-14)
    slot = int(w.state_indices[0])
    np.testing.assert_allclose(ss2[slot], ss[slot][..., perm.numpy()], rtol=1e-13, atol=1e-14)


@pytest.mark.parametrize("L", [1, 2, 3, 4, 9])
def test_conv_state_carry_is_exact_copy(L):
    w = _layer_case([L], seed=11)
    _, cs, _ = _run(w)
    slot = int(w.state_indices[0])
    old = w.conv_state[slot].double().numpy()  # [conv_dim, 3]
    full = np.concatenate([old.T, w.x.double().numpy()], axis=0)  # rows -3..L-1
    np.testing.assert_array_equal(cs[slot], full[-3:].T)


def test_has_initial_state_zero_equals_zeroed_slot():
    w = _layer_case([12, 5], seed=12)
    w.has_initial_state = torch.tensor([0, 1], dtype=torch.int32)
    o1, c1, s1 = _run(w)
    w2 = _layer_case([12, 5], seed=12)
    slot = int(w2.state_indices[0])
    w2.conv_state[slot] = 0
    w2.ssm_state[slot] = 0
    o2, c2, s2 = _run(w2)
    np.testing.assert_array_equal(o1, o2)
    np.testing.assert_array_equal(s1, s2)
    np.testing.assert_array_equal(c1, c2)


def test_padded_request_touches_nothing():
    w = _layer_case([6, 4], seed=13)
    w.state_indices = torch.tensor([-1, int(w.state_indices[1])], dtype=torch.int32)
    out, cs, ss = _run(w)
    assert np.all(out[:6] == 0)
    untouched = [p for p in range(w.P) if p != int(w.state_indices[1])]
    np.testing.assert_array_equal(ss[untouched], w.ssm_state[untouched].double().numpy())
    np.testing.assert_array_equal(cs[untouched], w.conv_state[untouched].double().numpy())
