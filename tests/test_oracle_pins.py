"""Pins for the fp64 attention oracle (CPU only).

Each pin checks the oracle against something other than itself: a hand-derived
example, closed forms, finite differences, invariants the mathematics fixes, or
the online recurrence stated on the pages.  A plausible slip anywhere in the
oracle (a dropped term, a wrong sign, a transposed operand, a wrong mask
direction, a missing dropout rescale) fails at least one of them.
"""

import os

import numpy as np
import pytest

from oracle import attention, online, philox

HERE = os.path.dirname(os.path.abspath(__file__))
RTOL_FD = 1e-6


def _rand(rng, n, d, std=1.0):
    return rng.standard_normal((n, d)) * std


def _load_golden():
    vals = {}
    with open(os.path.join(HERE, "golden", "two_token_closed_form.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            name, *xs = line.split()
            vals[name] = np.array([float(x) for x in xs])
    return vals


# --------------------------------------------------------------------- golden

def test_two_token_hand_derived_example():
    g = _load_golden()
    q, k, v, do = (g[n].reshape(2, 1) for n in ("Q", "K", "V", "dO"))
    o, lse = attention.forward(q, k, v, causal=False, scale=1.0)
    np.testing.assert_allclose(o[:, 0], g["noncausal_O"], rtol=0, atol=1e-14)
    np.testing.assert_allclose(lse, g["noncausal_LSE"], rtol=0, atol=1e-14)
    o, lse = attention.forward(q, k, v, causal=True, scale=1.0)
    np.testing.assert_allclose(o[:, 0], g["causal_O"], rtol=0, atol=1e-14)
    np.testing.assert_allclose(lse, g["causal_LSE"], rtol=0, atol=1e-14)
    dq, dk, dv, _ = attention.backward(q, k, v, do, causal=False, scale=1.0)
    np.testing.assert_allclose(dq[:, 0], g["noncausal_dQ"], rtol=0, atol=1e-14)
    np.testing.assert_allclose(dk[:, 0], g["noncausal_dK"], rtol=0, atol=1e-14)
    np.testing.assert_allclose(dv[:, 0], g["noncausal_dV"], rtol=0, atol=1e-14)


# --------------------------------------------------------------- rows sum to 1

@pytest.mark.parametrize("n,d,causal", [(128, 64, False), (256, 64, True), (256, 128, True)])
def test_softmax_rows_sum_to_one(n, d, causal):
    rng = np.random.default_rng(n + d)
    q, k, v = (_rand(rng, n, d) for _ in range(3))
    _, _, p, _ = attention.forward(q, k, v, causal=causal, scale=d ** -0.5, return_p=True)
    np.testing.assert_allclose(p.sum(axis=1), 1.0, rtol=0, atol=1e-12)
    if causal:
        assert np.all(p[np.triu_indices(n, 1)] == 0.0)


# --------------------------------------------------------------- Q = 0 closed forms

@pytest.mark.parametrize("causal", [False, True])
def test_zero_q_gives_mean_of_v(causal):
    rng = np.random.default_rng(3)
    n, d = 200, 16
    q = np.zeros((n, d))
    k, v = _rand(rng, n, d), _rand(rng, n, d)
    o, lse = attention.forward(q, k, v, causal=causal, scale=0.25)
    if causal:
        want = np.cumsum(v, axis=0) / np.arange(1, n + 1)[:, None]
        want_lse = np.log(np.arange(1, n + 1))
    else:
        want = np.broadcast_to(v.mean(axis=0), (n, d))
        want_lse = np.full(n, np.log(n))
    np.testing.assert_allclose(o, want, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, want_lse, rtol=0, atol=1e-12)


def test_zero_q_with_dropout_gives_masked_mean():
    rng = np.random.default_rng(4)
    n, d, p = 64, 8, 0.25
    q = np.zeros((n, d))
    k, v = _rand(rng, n, d), _rand(rng, n, d)
    o, lse = attention.forward(q, k, v, causal=True, scale=0.3, p_drop=p, seed=11, b=1, h=2)
    z = philox.keep_mask(11, 1, 2, np.arange(n), np.arange(n), p).astype(float)
    z = np.tril(z)
    want = (z @ v) / (np.arange(1, n + 1)[:, None] * (1 - p))
    np.testing.assert_allclose(o, want, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, np.log(np.arange(1, n + 1)), rtol=0, atol=1e-12)


# ------------------------------------------------- online recurrence == two-pass

@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("std", [1.0, 4.0])
@pytest.mark.parametrize("p_drop", [0.0, 0.2])
def test_online_recurrence_equals_two_pass(causal, std, p_drop):
    rng = np.random.default_rng(int(std * 10) + causal)
    n, d = 64, 16
    q, k = _rand(rng, n, d, std), _rand(rng, n, d, std)
    v = _rand(rng, n, d)
    o2, l2 = attention.forward(q, k, v, causal=causal, scale=d ** -0.5, p_drop=p_drop, seed=5)
    for tile in (1, 3, 16, n):
        o1, l1 = online.forward_online(q, k, v, causal=causal, scale=d ** -0.5, tile=tile, p_drop=p_drop, seed=5)
        np.testing.assert_allclose(o1, o2, rtol=0, atol=1e-12)
        np.testing.assert_allclose(l1, l2, rtol=0, atol=1e-12)


# ------------------------------------------------------ finite-difference grads

def _loss(q, k, v, do, **kw):
    o, _ = attention.forward(q, k, v, **kw)
    return float((o * do).sum())


def _fd_grad(x_index, args, kw, h=1e-6):
    args = [a.copy() for a in args]
    x = args[x_index]
    g = np.zeros_like(x)
    for idx in np.ndindex(x.shape):
        old = x[idx]
        x[idx] = old + h
        fp = _loss(*args, **kw)
        x[idx] = old - h
        fm = _loss(*args, **kw)
        x[idx] = old
        g[idx] = (fp - fm) / (2 * h)
    return g


@pytest.mark.parametrize("n,d", [(16, 4), (12, 8)])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("p_drop", [0.0, 0.3])
def test_gradients_match_finite_differences(n, d, causal, p_drop):
    rng = np.random.default_rng(n * 100 + d + causal)
    q, k, v, do = (_rand(rng, n, d) for _ in range(4))
    kw = dict(causal=causal, scale=d ** -0.5, p_drop=p_drop, seed=21, b=1, h=3)
    dq, dk, dv, _ = attention.backward(q, k, v, do, **kw)
    for i, g in enumerate((dq, dk, dv)):
        fd = _fd_grad(i, (q, k, v, do), kw)
        rel = np.linalg.norm(g - fd) / np.linalg.norm(fd)
        assert rel <= RTOL_FD, (i, rel)


# --------------------------------------------------------------------- invariants

@pytest.mark.parametrize("causal", [False, True])
def test_key_shift_invariance(causal):
    rng = np.random.default_rng(8)
    n, d, scale = 96, 16, 0.25
    q, k, v = (_rand(rng, n, d) for _ in range(3))
    c = rng.standard_normal(d)
    o1, l1 = attention.forward(q, k, v, causal=causal, scale=scale)
    o2, l2 = attention.forward(q, k + c, v, causal=causal, scale=scale)
    np.testing.assert_allclose(o2, o1, rtol=0, atol=1e-12)
    np.testing.assert_allclose(l2, l1 + scale * (q @ c), rtol=0, atol=1e-12)


def test_joint_kv_permutation_invariance():
    rng = np.random.default_rng(9)
    n, d = 80, 16
    q, k, v = (_rand(rng, n, d) for _ in range(3))
    perm = rng.permutation(n)
    o1, l1 = attention.forward(q, k, v, causal=False, scale=0.25)
    o2, l2 = attention.forward(q, k[perm], v[perm], causal=False, scale=0.25)
    np.testing.assert_allclose(o2, o1, rtol=0, atol=1e-12)
    np.testing.assert_allclose(l2, l1, rtol=0, atol=1e-12)


def test_single_token_returns_v():
    rng = np.random.default_rng(10)
    q, k, v = (_rand(rng, 1, 8) for _ in range(3))
    o, lse = attention.forward(q, k, v, causal=True, scale=0.5)
    np.testing.assert_allclose(o, v, rtol=0, atol=0)
    np.testing.assert_allclose(lse, 0.5 * (q @ k.T)[0], rtol=0, atol=1e-15)


def test_p_zero_is_no_dropout():
    rng = np.random.default_rng(12)
    q, k, v, do = (_rand(rng, 40, 8) for _ in range(4))
    a = attention.forward(q, k, v, causal=True, scale=0.3)
    b = attention.forward(q, k, v, causal=True, scale=0.3, p_drop=0.0, seed=1234)
    np.testing.assert_array_equal(a[0], b[0])
    np.testing.assert_array_equal(a[1], b[1])


@pytest.mark.parametrize("p_drop", [0.0, 0.2])
def test_d_equals_rowsum_do_times_o(p_drop):
    rng = np.random.default_rng(13)
    n, d = 64, 16
    q, k, v, do = (_rand(rng, n, d) for _ in range(4))
    kw = dict(causal=True, scale=0.25, p_drop=p_drop, seed=3, b=0, h=1)
    o, _ = attention.forward(q, k, v, **kw)
    _, _, _, d_row = attention.backward(q, k, v, do, **kw)
    np.testing.assert_allclose(d_row, (do * o).sum(axis=1), rtol=0, atol=1e-12)


# ----------------------------------------------- sampled evaluation == full

@pytest.mark.parametrize("p_drop", [0.0, 0.1])
def test_row_and_column_sampling_matches_full(p_drop):
    rng = np.random.default_rng(14)
    n, d = 192, 32
    q, k, v, do = (_rand(rng, n, d) for _ in range(4))
    kw = dict(causal=True, scale=d ** -0.5, p_drop=p_drop, seed=4, b=0, h=2)
    o, lse = attention.forward(q, k, v, **kw)
    dq, dk, dv, d_row = attention.backward(q, k, v, do, **kw)
    rows = np.array([0, 5, 63, 64, 100, 191])
    lse_s, o_s, d_s = attention.row_stats(q, k, v, do, rows=rows, block=4, **kw)
    np.testing.assert_allclose(lse_s, lse[rows], rtol=0, atol=1e-12)
    np.testing.assert_allclose(o_s, o[rows], rtol=0, atol=1e-12)
    np.testing.assert_allclose(d_s, d_row[rows], rtol=0, atol=1e-12)
    dq_s = attention.grad_rows(q, k, v, do, rows=rows, block=4, **kw)
    np.testing.assert_allclose(dq_s, dq[rows], rtol=0, atol=1e-12)
    lse_all, _, d_all = attention.row_stats(q, k, v, do, block=50, **kw)
    cols = np.array([0, 1, 77, 128, 191])
    dk_s, dv_s = attention.grad_cols(q, k, v, do, lse_all, d_all, cols=cols, block=50, **kw)
    np.testing.assert_allclose(dk_s, dk[cols], rtol=0, atol=1e-12)
    np.testing.assert_allclose(dv_s, dv[cols], rtol=0, atol=1e-12)
