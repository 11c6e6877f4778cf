"""Materialising fp64 attention: the plain definition the fused kernels must equal.

TEST INFRASTRUCTURE ONLY -- see ``oracle/__init__.py``.

Definition followed (per head):

* S_ij = scale * Q_i . K_j  ("DL0056 FlashAttention", "Where:" after the
  Mathematical Formulation, with scale = 1/sqrt(d) there; here ``scale`` is an
  argument and the workloads pass 1/sqrt(d)).
* causal: S_ij = -inf for j > i + (Nk - Nq) ("FlashAttention" glossary,
  Causal Masking bullet: no token attends to a future token).  For Nq = Nk
  this is the square, top-left aligned mask; for Nq != Nk the queries are the
  LAST Nq positions of the key sequence (bottom-right alignment), the reading
  under which query i sits at position i + Nk - Nq.
* a query row that sees no key at all (only possible when Nk < Nq under the
  causal mask) has an empty softmax: its sum l_i is the empty sum 0, so
  LSE_i = ln 0 = -inf, O_i = 0, and it contributes nothing to any gradient.
* P = softmax over each row of S ("Flash Attention" glossary, "Why Regular
  Attention Becomes a Bottleneck": scores, softmax weights, combine values).
* stored statistic LSE_i = m_i + ln(l_i) with m_i = max_j S_ij and
  l_i = sum_j exp(S_ij - m_i): the per-row output the backward pass recomputes
  P from ("FlashAttention" glossary, Recomputation: gradients are recomputed
  from the stored outputs).  Natural-log units of the scaled scores; not
  affected by dropout.
* dropout: Z from ``oracle.philox.keep_mask``; P_d = P * Z / (1 - p), applied to
  the normalised probabilities after the softmax ("FlashAttention" glossary,
  Dropout bullet; reading recorded in the design notes).
* O = P_d V.

Q and dO are [Nq, d]; K and V are [Nk, d].

Backward: the analytic gradient of O = P_d V for an upstream gradient dO,
    dV = P_d^T dO,   dP_d = dO V^T,   dP = dP_d * Z / (1 - p),
    D_i = sum_j P_ij dP_ij,   dS = P * (dP - D),
    dQ = scale * dS K,   dK = scale * dS^T Q.
Pinned against central finite differences in tests/test_oracle_pins.py.

Every function takes float64 arrays and returns float64 arrays.  ``rows``
selects which query rows to evaluate: each row of the definition depends only
on its own row of S, so evaluating a subset of rows is the same definition,
not a reordering of it.
"""

import numpy as np

from .philox import keep_mask


def _as64(x):
    x = np.asarray(x)
    if x.dtype != np.float64:
        x = x.astype(np.float64)
    return x


def scores(q, k, scale, causal, rows=None, cols=None):
    """S[rows, cols] = scale * Q[rows] K[cols]^T with the causal mask: -inf where
    key j lies after query i's position i + Nk - Nq."""
    q, k = _as64(q), _as64(k)
    n = k.shape[0]
    offset = n - q.shape[0]
    rows = np.arange(q.shape[0]) if rows is None else np.asarray(rows, dtype=np.int64)
    cols = np.arange(n) if cols is None else np.asarray(cols, dtype=np.int64)
    s = scale * (q[rows] @ k[cols].T)
    if causal:
        s = np.where(cols[None, :] > rows[:, None] + offset, -np.inf, s)
    return s


def softmax_rows(s):
    """(P, LSE) of each row of S.  A row with no finite entry (no visible key)
    gets P = 0 and LSE = -inf: the empty sum is 0 and ln 0 = -inf."""
    m = s.max(axis=1)
    seen = np.isfinite(m)
    m_safe = np.where(seen, m, 0.0)
    e = np.exp(s - m_safe[:, None])
    l = e.sum(axis=1)
    p = e / np.where(seen, l, 1.0)[:, None]
    with np.errstate(divide="ignore"):
        lse = np.where(seen, m_safe + np.log(np.where(seen, l, 1.0)), -np.inf)
    return p, lse


def dropout_factor(seed, b, h, rows, cols, p_drop):
    """Z / (1 - p) for the given rows/cols (all ones when p = 0)."""
    if p_drop == 0.0:
        return np.ones((len(rows), len(cols)))
    z = keep_mask(seed, b, h, rows, cols, p_drop).astype(np.float64)
    return z / (1.0 - p_drop)


def forward(q, k, v, *, causal, scale, p_drop=0.0, seed=0, b=0, h=0, rows=None, return_p=False):
    """O[rows], LSE[rows] of one head by the materialising definition.

    q, k, v: [N, d] (bf16-rounded values as float64).  Returns (O, LSE) or
    (O, LSE, P, Pd) with ``return_p``.
    """
    q, k, v = _as64(q), _as64(k), _as64(v)
    n = k.shape[0]
    rows = np.arange(q.shape[0]) if rows is None else np.asarray(rows, dtype=np.int64)
    cols = np.arange(n)
    s = scores(q, k, scale, causal, rows, cols)
    p, lse = softmax_rows(s)
    pd = p * dropout_factor(seed, b, h, rows, cols, p_drop)
    o = pd @ v
    if return_p:
        return o, lse, p, pd
    return o, lse


def backward(q, k, v, do, *, causal, scale, p_drop=0.0, seed=0, b=0, h=0):
    """(dQ, dK, dV, D) of one head for the loss gradient dO, full materialisation."""
    q, k, v, do = _as64(q), _as64(k), _as64(v), _as64(do)
    rows = np.arange(q.shape[0])
    cols = np.arange(k.shape[0])
    s = scores(q, k, scale, causal, rows, cols)
    p, _ = softmax_rows(s)
    f = dropout_factor(seed, b, h, rows, cols, p_drop)
    pd = p * f
    dv = pd.T @ do
    dpd = do @ v.T
    dp = dpd * f
    d_row = (p * dp).sum(axis=1)
    ds = p * (dp - d_row[:, None])
    dq = scale * (ds @ k)
    dk = scale * (ds.T @ q)
    return dq, dk, dv, d_row


# ---------------------------------------------------------------------------
# Row-sampled evaluation for heads too large to materialise at once.  Same
# definition; only which entries are evaluated changes.
# ---------------------------------------------------------------------------

def row_stats(q, k, v, do, *, causal, scale, p_drop=0.0, seed=0, b=0, h=0, rows=None, block=512):
    """LSE_i, O_i and D_i = sum_j P_ij dP_ij for ``rows`` (default: all), evaluated in row blocks."""
    q, k, v, do = _as64(q), _as64(k), _as64(v), _as64(do)
    n = k.shape[0]
    rows = np.arange(q.shape[0]) if rows is None else np.asarray(rows, dtype=np.int64)
    cols = np.arange(n)
    lse = np.empty(len(rows))
    o = np.empty((len(rows), v.shape[1]))
    d_row = np.empty(len(rows))
    for a in range(0, len(rows), block):
        rb = rows[a:a + block]
        s = scores(q, k, scale, causal, rb, cols)
        p, lse[a:a + block] = softmax_rows(s)
        f = dropout_factor(seed, b, h, rb, cols, p_drop)
        o[a:a + block] = (p * f) @ v
        dp = (do[rb] @ v.T) * f
        d_row[a:a + block] = (p * dp).sum(axis=1)
    return lse, o, d_row


def grad_rows(q, k, v, do, *, causal, scale, p_drop=0.0, seed=0, b=0, h=0, rows, block=512):
    """dQ[rows]: dQ_i = scale * sum_j P_ij (dP_ij - D_i) K_j (needs only row i of S)."""
    q, k, v, do = _as64(q), _as64(k), _as64(v), _as64(do)
    n = k.shape[0]
    rows = np.asarray(rows, dtype=np.int64)
    cols = np.arange(n)
    dq = np.empty((len(rows), q.shape[1]))
    for a in range(0, len(rows), block):
        rb = rows[a:a + block]
        s = scores(q, k, scale, causal, rb, cols)
        p, _ = softmax_rows(s)
        f = dropout_factor(seed, b, h, rb, cols, p_drop)
        dp = (do[rb] @ v.T) * f
        d_row = (p * dp).sum(axis=1)
        dq[a:a + block] = scale * ((p * (dp - d_row[:, None])) @ k)
    return dq


def grad_cols(q, k, v, do, lse_all, d_all, *, causal, scale, p_drop=0.0, seed=0, b=0, h=0, cols, block=4096):
    """dK[cols], dV[cols] given LSE_i and D_i of every query row of the head.

    dV_j = sum_i P_d,ij dO_i and dK_j = scale * sum_i P_ij (dP_ij - D_i) Q_i with
    P_ij = exp(S_ij - LSE_i) (0 for a row with LSE_i = -inf, which sees no key).
    """
    q, k, v, do = _as64(q), _as64(k), _as64(v), _as64(do)
    n = q.shape[0]
    cols = np.asarray(cols, dtype=np.int64)
    dk = np.zeros((len(cols), k.shape[1]))
    dv = np.zeros((len(cols), v.shape[1]))
    for a in range(0, n, block):
        rb = np.arange(a, min(n, a + block))
        s = scores(q, k, scale, causal, rb, cols)
        lse_rb = lse_all[rb]
        p = np.where(np.isfinite(lse_rb)[:, None], np.exp(s - np.where(np.isfinite(lse_rb), lse_rb, 0.0)[:, None]), 0.0)
        f = dropout_factor(seed, b, h, rb, cols, p_drop)
        dv += (p * f).T @ do[rb]
        dp = (do[rb] @ v[cols].T) * f
        ds = p * (dp - d_all[rb][:, None])
        dk += scale * (ds.T @ q[rb])
    return dk, dv
