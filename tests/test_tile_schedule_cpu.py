"""CPU replay of the CUDA kernels' work assignment and mask limits (no GPU).

The forward kernel (fa_fwd.cu) and the backward kernel (fa_bwd.cu) each
decode a 1-D grid into (unit group, tile, unit), pick the key tiles (forward)
or query tiles (backward) a CTA visits, and skip the per-element mask on
tiles that need none.  This file restates that index arithmetic, as the
kernels write it, and checks over ragged lengths, Nq != Nk (bottom-right
causal), packed sequences (empty ones included), grids whose unit count is not
a multiple of the group size and the deterministic backward order that every
(query, key) pair the method keeps is visited unmasked exactly once and that
no other pair is left unmasked.  A change to those formulas in the kernels is
to be mirrored here."""

import itertools

import numpy as np
import pytest


def floor_div(a, b):
    """floor(a / b) for b > 0 (Python's // on integers)."""
    return a // b


def _units(B, H, Nq, Nk, cu_q, cu_k):
    """(unit, queries, keys) of every (b, h) unit, as the kernels resolve them."""
    out = []
    for unit in range(B * H):
        b = unit // H
        if cu_q is None:
            out.append((unit, Nq, Nk))
        else:
            out.append((unit, min(cu_q[b + 1] - cu_q[b], Nq), min(cu_k[b + 1] - cu_k[b], Nk)))
    return out


def _want(nq, nk, causal):
    i = np.arange(nq)[:, None]
    j = np.arange(nk)[None, :]
    return ((j <= i + nk - nq) if causal else np.ones((nq, nk), bool)).astype(np.int32)


def fwd(B, H, Nq, Nk, causal, cu_q=None, cu_k=None):
    """Forward: CTAs of two 128-row query tiles over 128-key tiles."""
    BH = B * H
    n_qb = ((Nq + 127) // 128 + 1) // 2
    group = min(max((256 + n_qb // 2) // n_qb, 1), BH)
    U = {u: (nq, nk) for u, nq, nk in _units(B, H, Nq, Nk, cu_q, cu_k)}
    seen = {u: np.zeros((max(nq, 1), max(nk, 1)), np.int32) for u, (nq, nk) in U.items()}
    per_group = group * n_qb
    for bid in range(BH * n_qb):
        grp = bid // per_group
        rr = bid - grp * per_group
        gsz = min(group, BH - grp * group)
        qb_lin = rr // gsz
        unit = grp * group + (rr - qb_lin * gsz)
        N, nk = U[unit]
        n_qt = (N + 127) // 128
        qt0 = 2 * ((n_qb - 1 - qb_lin) if causal else qb_lin)
        if qt0 >= n_qt:
            continue
        n_kt = (nk + 127) // 128
        delta = nk - N
        for q in range(min(2, n_qt - qt0)):
            last_row = min(N - 1, (qt0 + q) * 128 + 127)
            ntq = min(n_kt, max(0, floor_div(last_row + delta, 128) + 1)) if causal else n_kt
            rows = (qt0 + q) * 128 + np.arange(128)
            lim0 = np.minimum(nk - 1, rows + delta) if causal else np.full(128, nk - 1)
            t_mask = nk // 128
            if causal:
                t_mask = min(t_mask, max(0, floor_div((qt0 + q) * 128 + delta - 127, 128) + 1))
            stored = (rows < N)[:, None]  # rows of a partial last tile are not stored
            for t in range(ntq):
                cols = t * 128 + np.arange(128)
                vis = (cols[None, :] <= lim0[:, None]) if t >= t_mask else np.ones((128, 128), bool)
                keep = (cols[None, :] < nk) & ((cols[None, :] <= rows[:, None] + delta) if causal else True)
                assert not (vis & ~keep & stored).any(), ("forward leaves a pair unmasked", Nq, Nk, unit, t)
                r, c = np.nonzero(vis & keep & stored)
                np.add.at(seen[unit], (rows[r], cols[c]), 1)
    for u, (nq, nk) in U.items():
        if nq and nk:
            assert (seen[u][:nq, :nk] == _want(nq, nk, causal)).all(), ("forward coverage", Nq, Nk, u)


def bwd(B, H, Nq, Nk, causal, cu_q=None, cu_k=None, det=False):
    """Backward: CTAs of one 128-key tile over 128-row query tiles."""
    BH = B * H
    n_kt_grid = (Nk + 127) // 128
    group = min(max((512 + n_kt_grid // 2) // n_kt_grid, 1), BH)
    U = {u: (nq, nk) for u, nq, nk in _units(B, H, Nq, Nk, cu_q, cu_k)}
    seen = {u: np.zeros((max(nq, 1), max(nk, 1)), np.int32) for u, (nq, nk) in U.items()}
    per_group = group * n_kt_grid
    r = np.arange(128)
    c = np.arange(128)
    for bid in range(BH * n_kt_grid):
        grp = bid // per_group
        rr = bid - grp * per_group
        gsz = min(group, BH - grp * group)
        kj = rr // gsz
        unit = grp * group + (rr - kj * gsz)
        nqu, nk = U[unit]
        if kj * 128 >= nk:
            continue
        n_qt = (nqu + 127) // 128
        delta = nk - nqu
        q_first = max(0, floor_div(kj * 128 - delta, 128)) if causal else 0
        if n_qt - q_first <= 0:
            continue
        keys = kj * 128 + r
        key_valid = keys < nk
        lo0 = kj * 128 + r - delta if causal else np.full(128, -(1 << 30))
        qi_mask = floor_div(kj * 128 + 126 - delta, 128) if causal else -1
        tile_past_keys = kj * 128 + 128 > nk
        for it in range(n_qt - q_first):
            qi = (n_qt - 1 - it) if det else (q_first + it)
            qrows = qi * 128 + c
            vis = np.broadcast_to(qrows[None, :] < nqu, (128, 128)).copy()  # LSE2 = +inf past the unit
            if qi <= qi_mask or tile_past_keys:
                lo = np.where(key_valid, lo0 - qi * 128, 128)
                vis &= ~(c[None, :] < lo[:, None])
            keep = key_valid[:, None] & (qrows[None, :] < nqu) & \
                ((qrows[None, :] + delta >= keys[:, None]) if causal else True)
            assert not (vis & ~keep).any(), ("backward leaves a pair unmasked", Nq, Nk, unit, kj, qi)
            k, q = np.nonzero(vis)
            np.add.at(seen[unit], (qrows[q], keys[k]), 1)
    for u, (nq, nk) in U.items():
        if nq and nk:
            assert (seen[u][:nq, :nk] == _want(nq, nk, causal)).all(), ("backward coverage", Nq, Nk, u, det)


LENS = [1, 64, 127, 128, 129, 255, 257, 383, 513]


@pytest.mark.parametrize("causal", [False, True])
def test_ragged_and_rectangular(causal):
    for Nq, Nk in itertools.product(LENS, LENS):
        fwd(1, 2, Nq, Nk, causal)
        bwd(1, 2, Nq, Nk, causal)
        bwd(1, 2, Nq, Nk, causal, det=True)


@pytest.mark.parametrize("B,H,N", [(3, 37, 300), (2, 300, 128), (1, 700, 257)])
def test_group_boundaries(B, H, N):
    for causal in (False, True):
        fwd(B, H, N, N, causal)
        bwd(B, H, N, N, causal)


def test_packed_sequences():
    rng = np.random.default_rng(0)
    for _ in range(20):
        B, H = int(rng.integers(1, 6)), int(rng.integers(1, 3))
        lq, lk = rng.integers(0, 600, size=B), rng.integers(0, 600, size=B)
        if rng.random() < 0.3:
            lk = lq.copy()
        lq[0] = 0  # an empty sequence in every draw
        cu_q = np.concatenate([[0], np.cumsum(lq)]).astype(int)
        cu_k = np.concatenate([[0], np.cumsum(lk)]).astype(int)
        mq, mk = max(1, int(lq.max())), max(1, int(lk.max()))
        for causal in (False, True):
            fwd(B, H, mq, mk, causal, cu_q, cu_k)
            bwd(B, H, mq, mk, causal, cu_q, cu_k)
            bwd(B, H, mq, mk, causal, cu_q, cu_k, det=True)
