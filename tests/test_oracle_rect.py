"""Pins for the oracle on rectangular problems (Nq != Nk) and on query rows that
see no key (CPU only).

Causal alignment is bottom-right: query i sits at key position i + Nk - Nq.
The pins are closed forms (Q = 0 gives prefix means of V whose lengths fix
the alignment, and -inf / 0 for rows that see nothing), central finite
differences of the gradients, the online recurrence, and the row / column
sampled evaluators against the full materialisation.
"""

import numpy as np
import pytest

from oracle import attention, online

RTOL_FD = 1e-6


def _rand(rng, n, d):
    return rng.standard_normal((n, d))


@pytest.mark.parametrize("nq,nk", [(5, 12), (12, 12), (12, 5), (1, 9), (9, 1)])
def test_zero_q_causal_closed_form(nq, nk):
    """Q = 0: row i averages V over keys 0 .. i + nk - nq; with no such key,
    O_i = 0 and LSE_i = -inf."""
    rng = np.random.default_rng(nq * 31 + nk)
    d = 6
    q = np.zeros((nq, d))
    k, v = _rand(rng, nk, d), _rand(rng, nk, d)
    o, lse = attention.forward(q, k, v, causal=True, scale=0.7)
    for i in range(nq):
        last = i + nk - nq  # last visible key
        if last < 0:
            assert np.all(o[i] == 0.0) and lse[i] == -np.inf
        else:
            np.testing.assert_allclose(o[i], v[:last + 1].mean(axis=0), rtol=0, atol=1e-12)
            assert abs(lse[i] - np.log(last + 1)) < 1e-12


@pytest.mark.parametrize("nq,nk", [(5, 12), (12, 5)])
def test_zero_q_non_causal_closed_form(nq, nk):
    rng = np.random.default_rng(7)
    q = np.zeros((nq, 4))
    k, v = _rand(rng, nk, 4), _rand(rng, nk, 4)
    o, lse = attention.forward(q, k, v, causal=False, scale=1.3)
    np.testing.assert_allclose(o, np.broadcast_to(v.mean(axis=0), (nq, 4)), rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, np.full(nq, np.log(nk)), rtol=0, atol=1e-12)


def test_bottom_right_rows_equal_the_tail_of_the_square_problem():
    """Without dropout, the rectangular causal problem is the last nq rows of the
    square causal problem over all nk positions."""
    rng = np.random.default_rng(11)
    nk, nq, d = 20, 7, 5
    q_full, k, v = _rand(rng, nk, d), _rand(rng, nk, d), _rand(rng, nk, d)
    o_sq, l_sq = attention.forward(q_full, k, v, causal=True, scale=0.5)
    o, lse = attention.forward(q_full[nk - nq:], k, v, causal=True, scale=0.5)
    np.testing.assert_allclose(o, o_sq[nk - nq:], rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, l_sq[nk - nq:], rtol=0, atol=1e-12)


def _loss(q, k, v, do, **kw):
    o, _ = attention.forward(q, k, v, **kw)
    return float((o * do).sum())


def _fd(idx, args, kw, h=1e-6):
    args = [a.copy() for a in args]
    x = args[idx]
    g = np.zeros_like(x)
    for pos in np.ndindex(x.shape):
        old = x[pos]
        x[pos] = old + h
        fp = _loss(*args, **kw)
        x[pos] = old - h
        fm = _loss(*args, **kw)
        x[pos] = old
        g[pos] = (fp - fm) / (2 * h)
    return g


@pytest.mark.parametrize("nq,nk", [(6, 10), (10, 6)])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("p_drop", [0.0, 0.3])
def test_rectangular_gradients_match_finite_differences(nq, nk, causal, p_drop):
    rng = np.random.default_rng(nq * 10 + nk + causal)
    d = 4
    q, do = _rand(rng, nq, d), _rand(rng, nq, d)
    k, v = _rand(rng, nk, d), _rand(rng, nk, d)
    kw = dict(causal=causal, scale=0.5, p_drop=p_drop, seed=9, b=2, h=1)
    dq, dk, dv, _ = attention.backward(q, k, v, do, **kw)
    for i, g in enumerate((dq, dk, dv)):
        fd = _fd(i, (q, k, v, do), kw)
        assert np.linalg.norm(g - fd) <= RTOL_FD * max(np.linalg.norm(fd), 1e-300), (i,)
    if causal and nk < nq:
        # rows that see no key get no gradient
        assert np.all(dq[:nq - nk] == 0.0)


@pytest.mark.parametrize("nq,nk", [(24, 40), (40, 24)])
@pytest.mark.parametrize("p_drop", [0.0, 0.2])
def test_online_recurrence_equals_two_pass_rectangular(nq, nk, p_drop):
    rng = np.random.default_rng(nq + nk)
    d = 8
    q, k, v = _rand(rng, nq, d) * 3, _rand(rng, nk, d) * 3, _rand(rng, nk, d)
    o2, l2 = attention.forward(q, k, v, causal=True, scale=d ** -0.5, p_drop=p_drop, seed=4)
    for tile in (1, 5, 16, nk):
        o1, l1 = online.forward_online(q, k, v, causal=True, scale=d ** -0.5, tile=tile, p_drop=p_drop, seed=4)
        np.testing.assert_allclose(o1, o2, rtol=0, atol=1e-12)
        assert np.array_equal(np.isneginf(l1), np.isneginf(l2))
        fin = np.isfinite(l2)
        np.testing.assert_allclose(l1[fin], l2[fin], rtol=0, atol=1e-12)


@pytest.mark.parametrize("nq,nk", [(30, 50), (50, 30)])
def test_sampled_evaluators_match_full_rectangular(nq, nk):
    rng = np.random.default_rng(3)
    d = 8
    q, do = _rand(rng, nq, d), _rand(rng, nq, d)
    k, v = _rand(rng, nk, d), _rand(rng, nk, d)
    kw = dict(causal=True, scale=0.4, p_drop=0.1, seed=12, b=0, h=2)
    o, lse = attention.forward(q, k, v, **kw)
    dq, dk, dv, d_row = attention.backward(q, k, v, do, **kw)
    rows = np.array([0, 3, nq // 2, nq - 1])
    lse_s, o_s, d_s = attention.row_stats(q, k, v, do, rows=rows, block=3, **kw)
    np.testing.assert_allclose(o_s, o[rows], rtol=0, atol=1e-12)
    assert np.array_equal(np.isneginf(lse_s), np.isneginf(lse[rows]))
    np.testing.assert_allclose(d_s, d_row[rows], rtol=0, atol=1e-12)
    np.testing.assert_allclose(attention.grad_rows(q, k, v, do, rows=rows, block=3, **kw), dq[rows],
                               rtol=0, atol=1e-12)
    lse_all, _, d_all = attention.row_stats(q, k, v, do, **kw)
    cols = np.array([0, 7, nk - 1])
    dk_s, dv_s = attention.grad_cols(q, k, v, do, lse_all, d_all, cols=cols, block=7, **kw)
    np.testing.assert_allclose(dk_s, dk[cols], rtol=0, atol=1e-12)
    np.testing.assert_allclose(dv_s, dv[cols], rtol=0, atol=1e-12)
