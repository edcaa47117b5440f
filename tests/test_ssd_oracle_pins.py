"""Pins of the Mamba2 SSD oracle against what the mathematics fixes on its own.

Every expected value here comes from a computation that shares nothing with
``oracle/ssd_oracle.c``: the unrolled (quadratic, attention-like) form of the
scan written with explicit decay matrices in numpy, closed forms of special
cases (no decay, zero step, one scalar token, a state reset), and identities
between runs (prefix then continuation, checkpoints, group mapping, gate).
"""
import math

import numpy as np
import pytest

from oracle import ssd as S

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")


def _case(rng, T, H, P, N, G, with_init=True):
    x = rng.standard_normal((T, H, P))
    dt = rng.standard_normal((T, H))
    A = -rng.uniform(0.5, 4.0, H)
    B = rng.standard_normal((T, G, N))
    C = rng.standard_normal((T, G, N))
    D = rng.standard_normal(H)
    z = rng.standard_normal((T, H, P))
    bias = rng.uniform(-2.0, 0.5, H)
    init = 0.3 * rng.standard_normal((1, H, P, N)) if with_init else None
    return x, dt, A, B, C, D, z, bias, init


def _steps(dt, bias, softplus=True, lo=0.0, hi=math.inf):
    v = dt + bias[None, :]
    if softplus:
        v = np.where(v > 20.0, v, np.log1p(np.exp(np.minimum(v, 20.0))))
    return np.clip(v, lo, hi)


def _dual(x, d, A, B, C, D, z, h0, G):
    """The scan unrolled: y_t = sum_{s<=t} e^{Gam_t - Gam_s} d_s (C_t.B_s) x_s + e^{Gam_t} h0 C_t."""
    T, H, P = x.shape
    N = B.shape[2]
    y = np.zeros((T, H, P))
    fin = np.zeros((H, P, N))
    for h in range(H):
        g = h // (H // G)
        gam = np.cumsum(d[:, h] * A[h])
        Lm = np.tril(np.exp(gam[:, None] - gam[None, :]))
        M = Lm * (C[:, g, :] @ B[:, g, :].T) * d[None, :, h]
        y[:, h, :] = M @ x[:, h, :] + np.exp(gam)[:, None] * (C[:, g, :] @ h0[h].T)
        w = np.exp(gam[-1] - gam) * d[:, h]
        fin[h] = np.exp(gam[-1]) * h0[h] + (x[:, h, :] * w[:, None]).T @ B[:, g, :]
        if D is not None:
            y[:, h, :] += D[h] * x[:, h, :]
        if z is not None:
            y[:, h, :] *= z[:, h, :] / (1.0 + np.exp(-z[:, h, :]))
    return y, fin


def _rel(a, b):
    return np.linalg.norm((a - b).ravel()) / max(np.linalg.norm(b.ravel()), 1e-300)


@pytest.mark.parametrize("G", [1, 2, 4])
def test_scan_equals_unrolled_form(G):
    rng = np.random.default_rng(10 + G)
    T, H, P, N = 23, 4, 6, 5
    x, dt, A, B, C, D, z, bias, init = _case(rng, T, H, P, N, G)
    cfg = S.SsdCfg(H=H, P=P, N=N, G=G)
    y, fin, _ = S.scan(cfg, x, dt, A, B, C, [0, T], D=D, z=z, dt_bias=bias, init=init)
    ye, fe = _dual(x, _steps(dt, bias), A, B, C, D, z, init[0], G)
    assert _rel(y, ye) < 1e-12 and _rel(fin[0], fe) < 1e-12


def test_no_decay_is_a_running_sum():
    rng = np.random.default_rng(1)
    T, H, P, N, G = 17, 2, 3, 4, 1
    x, dt, _, B, C, _, _, bias, init = _case(rng, T, H, P, N, G)
    A = np.zeros(H)
    cfg = S.SsdCfg(H=H, P=P, N=N, G=G)
    y, fin, _ = S.scan(cfg, x, dt, A, B, C, [0, T], dt_bias=bias, init=init)
    d = _steps(dt, bias)
    for h in range(H):
        inc = np.cumsum(d[:, h, None, None] * x[:, h, :, None] * B[:, 0, None, :], axis=0) + init[0, h]
        assert np.allclose(fin[0, h], inc[-1], rtol=1e-13, atol=1e-13)
        assert np.allclose(y[:, h, :], np.einsum("tpn,tn->tp", inc, C[:, 0, :]), rtol=1e-12, atol=1e-12)


def test_zero_step_keeps_the_state():
    rng = np.random.default_rng(2)
    T, H, P, N, G = 9, 2, 3, 4, 2
    x, _, A, B, C, D, _, _, init = _case(rng, T, H, P, N, G)
    cfg = S.SsdCfg(H=H, P=P, N=N, G=G, dt_softplus=False)
    y, fin, _ = S.scan(cfg, x, np.zeros((T, H)), A, B, C, [0, T], D=D, init=init)
    assert np.array_equal(fin, init)
    for h in range(H):
        expect = C[:, h, :] @ init[0, h].T + D[h] * x[:, h, :]
        assert np.allclose(y[:, h, :], expect, rtol=1e-13, atol=1e-13)


def test_one_scalar_token_by_hand():
    cfg = S.SsdCfg(H=1, P=1, N=1, G=1)
    x, dt, A, B, C, D, z, bias, h0 = 0.7, 0.3, -1.5, 1.2, -0.8, 0.25, 0.9, -0.4, 0.6
    d = math.log1p(math.exp(dt + bias))
    h1 = math.exp(d * A) * h0 + d * x * B
    yv = (h1 * C + D * x) * z / (1.0 + math.exp(-z))
    y, fin, _ = S.scan(cfg, [[[x]]], [[dt]], [A], [[[B]]], [[[C]]], [0, 1], D=[D], z=[[[z]]], dt_bias=[bias],
                       init=[[[[h0]]]])
    assert abs(y[0, 0, 0] - yv) < 1e-15 and abs(fin[0, 0, 0, 0] - h1) < 1e-15


def test_step_size_processing():
    base = S.SsdCfg(H=1, P=1, N=1, G=1)
    assert abs(S.step_size(base, 0.3, -0.1) - math.log1p(math.exp(0.2))) < 1e-15
    assert S.step_size(base, 25.0, 0.0) == 25.0
    raw = S.SsdCfg(H=1, P=1, N=1, G=1, dt_softplus=False)
    assert S.step_size(raw, -0.5, 0.2) == 0.0          # the default lower limit 0
    assert abs(S.step_size(raw, 0.5, 0.2) - 0.7) < 1e-15
    lim = S.SsdCfg(H=1, P=1, N=1, G=1, dt_limit=(0.01, 0.1))
    assert S.step_size(lim, 5.0, 0.0) == 0.1 and S.step_size(lim, -30.0, 0.0) == 0.01


def test_strong_decay_resets_the_state():
    rng = np.random.default_rng(3)
    T, H, P, N, G = 6, 2, 3, 4, 1
    x, _, _, B, C, D, _, _, init = _case(rng, T, H, P, N, G)
    A = np.full(H, -1e4)
    dt = np.full((T, H), 3.0)
    cfg = S.SsdCfg(H=H, P=P, N=N, G=G, dt_softplus=False)
    y, fin, _ = S.scan(cfg, x, dt, A, B, C, [0, T], D=D, init=init)
    for h in range(H):
        last = 3.0 * np.outer(x[-1, h], B[-1, 0])
        assert np.allclose(fin[0, h], last, rtol=1e-14, atol=0)
        cb = np.sum(C[:, 0, :] * B[:, 0, :], axis=1)
        assert np.allclose(y[:, h, :], (3.0 * cb)[:, None] * x[:, h, :] + D[h] * x[:, h, :], rtol=1e-13, atol=1e-13)


def test_prefix_then_continuation_equals_whole():
    rng = np.random.default_rng(4)
    T, H, P, N, G, a = 40, 4, 5, 3, 2, 17
    x, dt, A, B, C, D, z, bias, init = _case(rng, T, H, P, N, G)
    cfg = S.SsdCfg(H=H, P=P, N=N, G=G)
    kw = dict(D=D, dt_bias=bias)
    y, fin, _ = S.scan(cfg, x, dt, A, B, C, [0, T], z=z, init=init, **kw)
    y1, f1, _ = S.scan(cfg, x[:a], dt[:a], A, B[:a], C[:a], [0, a], z=z[:a], init=init, **kw)
    y2, f2, _ = S.scan(cfg, x[a:], dt[a:], A, B[a:], C[a:], [0, T - a], z=z[a:], init=f1, **kw)
    assert _rel(np.concatenate([y1, y2]), y) < 1e-13 and _rel(f2, fin) < 1e-13


def test_packed_sequences_are_independent():
    rng = np.random.default_rng(5)
    lens = [5, 0, 12, 1, 9]
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    T, H, P, N, G = int(cu[-1]), 2, 3, 4, 1
    x, dt, A, B, C, D, z, bias, _ = _case(rng, T, H, P, N, G, with_init=False)
    init = 0.3 * rng.standard_normal((len(lens), H, P, N))
    cfg = S.SsdCfg(H=H, P=P, N=N, G=G)
    y, fin, _ = S.scan(cfg, x, dt, A, B, C, cu, D=D, z=z, dt_bias=bias, init=init)
    for n, (a, b) in enumerate(zip(cu[:-1], cu[1:])):
        if b == a:
            assert np.array_equal(fin[n], init[n])
            continue
        ye, fe = _dual(x[a:b], _steps(dt[a:b], bias), A, B[a:b], C[a:b], D, z[a:b], init[n], G)
        assert _rel(y[a:b], ye) < 1e-12 and _rel(fin[n], fe) < 1e-12


def test_checkpoint_is_the_final_state_of_the_prefix():
    rng = np.random.default_rng(6)
    lens = [30, 7, 64]
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    T, H, P, N, G = int(cu[-1]), 2, 3, 4, 2
    x, dt, A, B, C, D, z, bias, _ = _case(rng, T, H, P, N, G, with_init=False)
    init = 0.3 * rng.standard_normal((3, H, P, N))
    cfg = S.SsdCfg(H=H, P=P, N=N, G=G)
    bounds = [cu[0] + 13, cu[1], cu[2] + 64]  # mid sequence, at the start (the initial state), at the end
    rows = [2, 0, 1]
    _, fin, ck, rc = S.scan(cfg, x, dt, A, B, C, cu, D=D, z=z, dt_bias=bias, init=init, ck_idx=bounds, ck_row=rows,
                            num_ck=3, return_rc=True)
    assert rc == 0
    for n in range(3):
        a, b = int(cu[n]), int(bounds[n])
        if b == a:
            expect = init[n]
        else:
            _, f, _ = S.scan(cfg, x[a:b], dt[a:b], A, B[a:b], C[a:b], [0, b - a], dt_bias=bias, init=init[n:n + 1])
            expect = f[0]
        assert _rel(ck[rows[n]], expect) < 1e-13
    assert _rel(ck[1], fin[2]) < 1e-13


def test_checkpoint_out_of_range_is_flagged_and_skipped():
    rng = np.random.default_rng(7)
    T, H, P, N, G = 10, 1, 2, 2, 1
    x, dt, A, B, C, _, _, bias, init = _case(rng, T, H, P, N, G)
    cfg = S.SsdCfg(H=H, P=P, N=N, G=G)
    _, _, ck, rc = S.scan(cfg, x, dt, A, B, C, [0, T], dt_bias=bias, init=init, ck_idx=[T + 1], ck_row=[0],
                          num_ck=1, return_rc=True)
    assert rc == 4 and not ck.any()
    _, _, ck, rc = S.scan(cfg, x, dt, A, B, C, [0, T], dt_bias=bias, init=init, ck_idx=[-1], ck_row=[0],
                          num_ck=1, return_rc=True)
    assert rc == 0 and not ck.any()


def test_head_reads_its_group():
    rng = np.random.default_rng(8)
    T, H, P, N, G = 11, 4, 3, 5, 2
    x, dt, A, B, C, D, z, bias, init = _case(rng, T, H, P, N, G)
    cfg = S.SsdCfg(H=H, P=P, N=N, G=G)
    y, fin, _ = S.scan(cfg, x, dt, A, B, C, [0, T], D=D, z=z, dt_bias=bias, init=init)
    one = S.SsdCfg(H=1, P=P, N=N, G=1)
    for h in range(H):
        g = h // (H // G)
        yh, fh, _ = S.scan(one, x[:, h:h + 1], dt[:, h:h + 1], A[h:h + 1], B[:, g:g + 1], C[:, g:g + 1], [0, T],
                           D=D[h:h + 1], z=z[:, h:h + 1], dt_bias=bias[h:h + 1], init=init[:, h:h + 1])
        assert np.array_equal(yh[:, 0], y[:, h]) and np.array_equal(fh[:, 0], fin[:, h])


def test_gate_and_skip():
    rng = np.random.default_rng(9)
    T, H, P, N, G = 8, 2, 4, 3, 1
    x, dt, A, B, C, D, z, bias, init = _case(rng, T, H, P, N, G)
    cfg = S.SsdCfg(H=H, P=P, N=N, G=G)
    y0, _, _ = S.scan(cfg, x, dt, A, B, C, [0, T], dt_bias=bias, init=init)
    yd, _, _ = S.scan(cfg, x, dt, A, B, C, [0, T], D=D, dt_bias=bias, init=init)
    yz, _, _ = S.scan(cfg, x, dt, A, B, C, [0, T], D=D, z=z, dt_bias=bias, init=init)
    assert np.allclose(yd, y0 + D[None, :, None] * x, rtol=1e-14, atol=1e-14)
    assert np.allclose(yz, yd * z / (1.0 + np.exp(-z)), rtol=1e-14, atol=1e-14)
    per = S.SsdCfg(H=H, P=P, N=N, G=G, d_per_dim=True)
    ypd, _, _ = S.scan(per, x, dt, A, B, C, [0, T], D=np.repeat(D[:, None], P, axis=1), dt_bias=bias, init=init)
    assert np.array_equal(ypd, yd)


@pytest.mark.parametrize("chunk", [1, 3, 64])
def test_chunked_form_equals_the_scan(chunk):
    rng = np.random.default_rng(20 + chunk)
    lens = [70, 0, 1, 130, 64]
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    T, H, P, N, G = int(cu[-1]), 4, 4, 6, 2
    x, dt, A, B, C, D, z, bias, _ = _case(rng, T, H, P, N, G, with_init=False)
    init = 0.3 * rng.standard_normal((len(lens), H, P, N))
    cfg = S.SsdCfg(H=H, P=P, N=N, G=G)
    y, fin, _ = S.scan(cfg, x, dt, A, B, C, cu, D=D, z=z, dt_bias=bias, init=init)
    yc, fc = S.scan_chunked(cfg, x, dt, A, B, C, cu, chunk, D=D, z=z, dt_bias=bias, init=init)
    assert _rel(yc, y) < 1e-12 and _rel(fc, fin) < 1e-12
