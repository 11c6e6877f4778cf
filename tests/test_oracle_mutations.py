"""Planted mistakes: each plausible slip in the oracle's arithmetic must make at
least one of the pins fail.  The mutants are local copies written here; the
oracle itself is not modified."""

import numpy as np
import pytest

from oracle import attention, philox


def _closed_form_zero_q(forward, causal):
    rng = np.random.default_rng(3)
    n, d = 64, 8
    q = np.zeros((n, d))
    k, v = rng.standard_normal((n, d)), rng.standard_normal((n, d))
    o, _ = forward(q, k, v, causal=causal, scale=0.25)
    want = (np.cumsum(v, axis=0) / np.arange(1, n + 1)[:, None]) if causal else np.broadcast_to(v.mean(0), (n, d))
    return np.abs(o - want).max() < 1e-12


def _fd_ok(backward, causal=True, p_drop=0.0):
    rng = np.random.default_rng(7)
    n, d = 10, 4
    q, k, v, do = (rng.standard_normal((n, d)) for _ in range(4))
    kw = dict(causal=causal, scale=0.5, p_drop=p_drop, seed=3, b=0, h=1)
    grads = backward(q, k, v, do, **kw)[:3]
    h = 1e-6
    for idx, g in enumerate(grads):
        args = [q, k, v]
        fd = np.zeros_like(g)
        for pos in np.ndindex(g.shape):
            a = [x.copy() for x in args]
            a[idx][pos] += h
            fp = (attention.forward(*a, **kw)[0] * do).sum()
            a[idx][pos] -= 2 * h
            fm = (attention.forward(*a, **kw)[0] * do).sum()
            fd[pos] = (fp - fm) / (2 * h)
        if np.linalg.norm(g - fd) / np.linalg.norm(fd) > 1e-6:
            return False
    return True


def test_unmutated_oracle_passes_the_same_checks():
    assert _closed_form_zero_q(attention.forward, True)
    assert _closed_form_zero_q(attention.forward, False)
    assert _fd_ok(attention.backward)
    assert _fd_ok(attention.backward, p_drop=0.3)


def test_flipped_causal_mask_is_caught():
    def fwd(q, k, v, *, causal, scale, **kw):
        n = k.shape[0]
        s = scale * q @ k.T
        if causal:
            s = np.where(np.arange(n)[None, :] < np.arange(n)[:, None], -np.inf, s)  # wrong direction
        p = np.exp(s - s.max(1, keepdims=True))
        p /= p.sum(1, keepdims=True)
        return p @ v, None
    assert not _closed_form_zero_q(fwd, True)


def test_missing_dropout_rescale_is_caught():
    rng = np.random.default_rng(4)
    n, d, p = 64, 8, 0.25
    q = np.zeros((n, d))
    k, v = rng.standard_normal((n, d)), rng.standard_normal((n, d))
    z = np.tril(philox.keep_mask(11, 1, 2, np.arange(n), np.arange(n), p).astype(float))
    want = (z @ v) / (np.arange(1, n + 1)[:, None] * (1 - p))
    s = np.where(np.triu(np.ones((n, n)), 1) > 0, -np.inf, 0.3 * q @ k.T)
    pm = np.exp(s - s.max(1, keepdims=True))
    pm /= pm.sum(1, keepdims=True)
    mutant = (pm * z) @ v  # forgot the 1/(1-p)
    assert np.abs(mutant - want).max() > 1e-3
    got, _ = attention.forward(q, k, v, causal=True, scale=0.3, p_drop=p, seed=11, b=1, h=2)
    assert np.abs(got - want).max() < 1e-12


def _backward_mutant(kind):
    def bwd(q, k, v, do, *, causal, scale, p_drop=0.0, seed=0, b=0, h=0):
        n = q.shape[0]
        rows = np.arange(n)
        s = attention.scores(q, k, scale, causal, rows, rows)
        p = np.exp(s - s.max(1, keepdims=True))
        p /= p.sum(1, keepdims=True)
        f = attention.dropout_factor(seed, b, h, rows, rows, p_drop)
        dv = (p * f).T @ do
        dp = (do @ v.T) * f
        dd = (p * dp).sum(1)
        ds = p * (dp + dd[:, None]) if kind == "sign" else p * (dp - dd[:, None])
        dq = scale * ds @ k
        dk = scale * (ds @ q if kind == "transpose" else ds.T @ q)
        return dq, dk, dv, dd
    return bwd


@pytest.mark.parametrize("kind", ["sign", "transpose"])
def test_backward_slips_are_caught_by_finite_differences(kind):
    assert not _fd_ok(_backward_mutant(kind))


def test_missing_philox_key_bump_is_caught_by_library_cross_check():
    def mutant(c0, c1, c2, c3, k0, k1):
        m32 = 0xFFFFFFFF
        for _ in range(10):  # the key is never advanced
            p0 = c0 * philox.PHILOX_M0
            p1 = c2 * philox.PHILOX_M1
            c0, c1, c2, c3 = ((p1 >> 32) ^ c1 ^ k0) & m32, p1 & m32, ((p0 >> 32) ^ c3 ^ k1) & m32, p0 & m32
        return c0, c1, c2, c3
    ref = tuple(int(x) for x in philox.philox4x32(1, 2, 3, 4, 5, 6))
    assert mutant(1, 2, 3, 4, 5, 6) != ref


@pytest.mark.parametrize("slip", ["none", "no_key_bump", "swapped_multipliers", "nine_rounds"])
def test_philox_slips_fail_the_known_answer_vectors(slip):
    import os
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "philox4x32_10_kat.txt")
    rows = []
    with open(path) as f:
        for line in f:
            if line.strip() and not line.startswith("#"):
                lhs, rhs = line.split("->")
                rows.append(([int(x, 16) for x in lhs.split()], [int(x, 16) for x in rhs.split()]))
    m0, m1 = philox.PHILOX_M0, philox.PHILOX_M1
    if slip == "swapped_multipliers":
        m0, m1 = m1, m0
    rounds = 9 if slip == "nine_rounds" else 10
    bump = slip != "no_key_bump"

    def mutant(c0, c1, c2, c3, k0, k1):
        m32 = 0xFFFFFFFF
        for r in range(rounds):
            if r and bump:
                k0, k1 = (k0 + 0x9E3779B9) & m32, (k1 + 0xBB67AE85) & m32
            p0, p1 = c0 * m0, c2 * m1
            c0, c1, c2, c3 = ((p1 >> 32) ^ c1 ^ k0) & m32, p1 & m32, ((p0 >> 32) ^ c3 ^ k1) & m32, p0 & m32
        return [c0, c1, c2, c3]

    if slip == "none":  # the restatement itself reproduces the vectors, so each mutant differs only by its slip
        assert all(mutant(*ins) == want for ins, want in rows)
    else:
        assert any(mutant(*ins) != want for ins, want in rows)


def test_keep_tie_break_at_threshold():
    """u16 == t is kept (keep <=> u16 >= t): find such draws and check them."""
    t = philox.keep_threshold(0.1)
    rows, cols = np.arange(64), np.arange(4096)
    u = philox.uniform16(5, 0, 0, rows, cols)
    z = philox.keep_mask(5, 0, 0, rows, cols, 0.1)
    eq = u == t
    assert eq.any()
    assert z[eq].all()
    assert not z[u == t - 1].any()


def test_top_left_alignment_for_rectangular_is_caught():
    """With Nq < Nk a mask that ignores the offset (top-left alignment) gives
    prefix means that are too short: the bottom-right closed form rejects it."""
    rng = np.random.default_rng(8)
    nq, nk, d = 4, 10, 3
    q = np.zeros((nq, d))
    k, v = rng.standard_normal((nk, d)), rng.standard_normal((nk, d))
    s = np.where(np.arange(nk)[None, :] > np.arange(nq)[:, None], -np.inf, 0.2 * q @ k.T)  # no offset
    p = np.exp(s - s.max(1, keepdims=True))
    p /= p.sum(1, keepdims=True)
    mutant = p @ v
    want = np.stack([v[:i + nk - nq + 1].mean(0) for i in range(nq)])
    assert np.abs(mutant - want).max() > 1e-3
    got, _ = attention.forward(q, k, v, causal=True, scale=0.2)
    assert np.abs(got - want).max() < 1e-12


def test_interleaved_gqa_head_mapping_is_caught():
    """Query head h reads key/value head h // (H / H_kv); a mutant that reads
    h % H_kv gives the wrong mean of V for the Q = 0 closed form."""
    rng = np.random.default_rng(12)
    H, H_kv, L, d = 6, 2, 9, 3
    v = rng.standard_normal((L, H_kv, d))
    want = [v[:, h // 3].mean(0) for h in range(H)]
    mutant = [v[:, h % H_kv].mean(0) for h in range(H)]
    assert max(np.abs(a - b).max() for a, b in zip(mutant, want)) > 1e-3
    from oracle import paged
    cache = v[None]  # one page holding all L positions
    o, _ = paged.decode_forward(np.zeros((1, H, 1, d)), cache, cache, np.zeros((1, 1), dtype=np.int32),
                                np.array([L]), causal=False, scale=1.0)
    for h in range(H):
        assert np.abs(o[0, h, 0] - want[h]).max() < 1e-12
