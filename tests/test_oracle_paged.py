"""Pins for the paged-cache oracle (CPU only): page gathering is pure
indexing, checked against contiguous storage; grouped-query heads read the
right key/value head (closed form with Q = 0); the decode rows equal the last
rows of the full causal problem; sequences without keys give O = 0, LSE = -inf."""

import numpy as np
import pytest

from oracle import attention, paged


def _paged_copy(k_contig, page, rng, extra_pages=3):
    """Scatter contiguous [B, L, H_kv, d] keys into shuffled pages; returns cache, table."""
    B, L, H_kv, d = k_contig.shape
    n = (L + page - 1) // page
    total = B * n + extra_pages
    perm = rng.permutation(total)
    cache = rng.standard_normal((total, page, H_kv, d))  # unused slots hold noise
    table = np.zeros((B, n), dtype=np.int32)
    for b in range(B):
        for j in range(n):
            p = perm[b * n + j]
            table[b, j] = p
            rows = k_contig[b, j * page:(j + 1) * page]
            cache[p, :len(rows)] = rows
    return cache, table


@pytest.mark.parametrize("page", [1, 4, 16])
def test_gather_inverts_the_page_scatter(page):
    rng = np.random.default_rng(page)
    k = rng.standard_normal((2, 37, 3, 5))
    cache, table = _paged_copy(k, page, rng)
    for b in range(2):
        for L in (0, 1, 16, 37):
            np.testing.assert_array_equal(paged.gather_pages(cache, table[b], L), k[b, :L])


def test_gqa_heads_read_their_group_closed_form():
    """Q = 0, no mask: O[b, h] = mean over positions of V[:, h // group]."""
    rng = np.random.default_rng(2)
    B, H, H_kv, Nq, L, d, page = 2, 6, 2, 3, 29, 4, 8
    k = rng.standard_normal((B, L, H_kv, d))
    v = rng.standard_normal((B, L, H_kv, d))
    kc, table = _paged_copy(k, page, np.random.default_rng(9))
    vc, _ = _paged_copy(v, page, np.random.default_rng(9))
    q = np.zeros((B, H, Nq, d))
    o, lse = paged.decode_forward(q, kc, vc, table, np.full(B, L), causal=False, scale=0.3)
    for b in range(B):
        for h in range(H):
            np.testing.assert_allclose(o[b, h], np.broadcast_to(v[b, :, h // 3].mean(0), (Nq, d)), atol=1e-12)
            np.testing.assert_allclose(lse[b, h], np.log(L), atol=1e-12)


def test_decode_rows_are_the_tail_of_the_full_causal_problem():
    rng = np.random.default_rng(4)
    B, H, Nq, d, page = 3, 2, 4, 8, 16
    lens = [50, 4, 77]
    Lmax = max(lens)
    k = rng.standard_normal((B, Lmax, H, d))
    v = rng.standard_normal((B, Lmax, H, d))
    q_full = rng.standard_normal((B, H, Lmax, d))
    kc, table = _paged_copy(k, page, np.random.default_rng(1))
    vc, _ = _paged_copy(v, page, np.random.default_rng(1))
    q = np.stack([q_full[b, :, lens[b] - Nq:lens[b]] for b in range(B)])
    o, lse = paged.decode_forward(q, kc, vc, table, np.array(lens), causal=True, scale=0.35)
    for b in range(B):
        for h in range(H):
            L = lens[b]
            o_sq, l_sq = attention.forward(q_full[b, h, :L], k[b, :L, h], v[b, :L, h], causal=True, scale=0.35)
            np.testing.assert_allclose(o[b, h], o_sq[L - Nq:], atol=1e-12)
            np.testing.assert_allclose(lse[b, h], l_sq[L - Nq:], atol=1e-12)


def test_sequence_without_keys():
    rng = np.random.default_rng(6)
    kc = rng.standard_normal((4, 8, 1, 4))
    q = rng.standard_normal((2, 1, 2, 4))
    table = np.array([[0, 1], [2, 3]], dtype=np.int32)
    o, lse = paged.decode_forward(q, kc, kc, table, np.array([0, 9]), causal=True, scale=0.5)
    assert np.all(o[0] == 0.0) and np.all(np.isneginf(lse[0]))
    assert np.all(np.isfinite(lse[1]))
