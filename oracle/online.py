"""The online-softmax recurrence, written out tile by tile (oracle self-check only).

TEST INFRASTRUCTURE ONLY -- see ``oracle/__init__.py``.

"DL0056 FlashAttention", Mathematical Formulation: for key/value tiles
t = 1..T and query row i,
    m_i^(t) = max(m_i^(t-1), max_j S_ij^(t)),
    l_i^(t) = exp(m_i^(t-1) - m_i^(t)) * l_i^(t-1) + sum_j exp(S_ij^(t) - m_i^(t)),
with m_i^(0) = -inf and l_i^(0) = 0.  The output accumulator is given there
only in words ("the exponential factors rescale earlier partial sums when the
maximum changes"; "Flash Attention" glossary, How Flash Attention Works,
step 4: accumulate each output tile as further key/value tiles arrive).  Its
plainest reading, used here:
    O_i^(t) = exp(m_i^(t-1) - m_i^(t)) * O_i^(t-1) + sum_j exp(S_ij^(t) - m_i^(t)) * F_ij V_j,
with O_i^(0) = 0, F = Z/(1-p) the dropout factor, and the result
O_i = O_i^(T) / l_i^(T), LSE_i = m_i^(T) + ln l_i^(T).

This module is never used to produce an expected value for the CUDA path; the
tests use it only to show it equals ``attention.forward`` (two-pass softmax).
"""

import numpy as np

from .attention import scores, dropout_factor


def forward_online(q, k, v, *, causal, scale, tile, p_drop=0.0, seed=0, b=0, h=0):
    q, k, v = (np.asarray(x, dtype=np.float64) for x in (q, k, v))
    n_q, n = q.shape[0], k.shape[0]
    rows = np.arange(n_q)
    m = np.full(n_q, -np.inf)
    l = np.zeros(n_q)
    acc = np.zeros((n_q, v.shape[1]))
    for start in range(0, n, tile):
        cols = np.arange(start, min(n, start + tile))
        s_t = scores(q, k, scale, causal, rows, cols)
        m_new = np.maximum(m, s_t.max(axis=1))
        # exp(m^(t-1) - m^(t)); a row whose max is still -inf has nothing to rescale
        alpha = np.where(np.isneginf(m_new), 0.0, np.exp(m - np.where(np.isneginf(m_new), 0.0, m_new)))
        e = np.where(np.isneginf(s_t), 0.0, np.exp(s_t - np.where(np.isneginf(m_new), 0.0, m_new)[:, None]))
        l = alpha * l + e.sum(axis=1)
        acc = alpha[:, None] * acc + (e * dropout_factor(seed, b, h, rows, cols, p_drop)) @ v[cols]
        m = m_new
    # a row that saw no key keeps l = 0: O = 0 and LSE = ln 0 = -inf (empty softmax)
    seen = l > 0
    with np.errstate(divide="ignore"):
        return (np.where(seen[:, None], acc / np.where(seen, l, 1.0)[:, None], 0.0),
                np.where(seen, m + np.log(np.where(seen, l, 1.0)), -np.inf))
