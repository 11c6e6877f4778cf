"""Attention over a paged key/value cache (decode), by gathering the pages back
into contiguous keys and applying the plain definition.

TEST INFRASTRUCTURE ONLY -- see ``oracle/__init__.py``.

The "FlashAttention" glossary (inferensys.com: the inference-server bullets
on vLLM and the PagedAttention entry) describes serving systems that keep the
key/value cache in non-contiguous fixed-size blocks and run FlashAttention-
style kernels over it while decoding; the computation is still exact
attention, only the storage of K and V changes.  Layout read here (the
plainest one that fits):

* k_cache, v_cache: [num_pages, page_size, H_kv, d]; page p holds page_size
  consecutive token positions of one sequence, for every key/value head;
* block_table[b, n] = the page that holds positions n*page_size ..
  (n+1)*page_size - 1 of sequence b;
* seqlens_k[b] = number of cached positions of sequence b;
* q: [B, H, Nq, d] with H a multiple of H_kv; query head h reads key/value
  head h // (H / H_kv) (grouped-query attention; H_kv = H is plain multi-head);
* the Nq queries of sequence b are its last Nq positions, so under the causal
  mask query i sees positions j <= seqlens_k[b] - Nq + i (the bottom-right
  alignment of ``attention.scores``).
"""

import numpy as np

from . import attention


def gather_pages(cache, block_table_row, seqlen):
    """Contiguous [seqlen, H_kv, d] keys (or values) of one sequence."""
    cache = np.asarray(cache)
    page = cache.shape[1]
    n_pages = (seqlen + page - 1) // page
    rows = [cache[int(block_table_row[n])] for n in range(n_pages)]
    if not rows:
        return cache[:0].reshape(0, cache.shape[2], cache.shape[3])
    return np.concatenate(rows, axis=0)[:seqlen]


def decode_forward(q, k_cache, v_cache, block_table, seqlens_k, *, causal, scale):
    """(O [B, H, Nq, d], LSE [B, H, Nq]) over the paged cache, fp64."""
    q = np.asarray(q, dtype=np.float64)
    B, H, Nq, d = q.shape
    H_kv = k_cache.shape[2]
    group = H // H_kv
    o = np.zeros((B, H, Nq, d))
    lse = np.full((B, H, Nq), -np.inf)
    for b in range(B):
        L = int(seqlens_k[b])
        k = gather_pages(k_cache, block_table[b], L).astype(np.float64)
        v = gather_pages(v_cache, block_table[b], L).astype(np.float64)
        for h in range(H):
            g = h // group
            if L == 0:
                continue  # no key at all: O = 0, LSE = -inf
            o[b, h], lse[b, h] = attention.forward(q[b, h], k[:, g], v[:, g], causal=causal, scale=scale)
    return o, lse
