"""Philox4x32-10 and the attention-dropout keep mask (oracle side).

TEST INFRASTRUCTURE ONLY -- see ``oracle/__init__.py``.

The pages say only that attention dropout is Bernoulli per attention score,
applied block-wise inside the softmax ("FlashAttention" glossary, Dropout
bullet) and that training kernels regenerate the same random pattern during
recomputation instead of storing a mask ("Flash Attention" glossary, Key
Components).  The mask is therefore a pure function of (seed, b, h, i, j).
The generator and the bit layout below are this library's fixed reading of
that requirement:

* generator: Philox4x32 with 10 rounds, as defined by Salmon, Moraes, Dror
  and Shaw, "Parallel Random Numbers: As Easy as 1, 2, 3" (SC'11): the two
  multipliers and the two Weyl key increments are the ones that paper
  publishes;
* key   (k0, k1)         = (seed mod 2^32, seed >> 32);
* counter (c0, c1, c2, c3) = (j >> 3, i, h, b);
* the four output words r0..r3 of one call serve the eight keys
  j = 8*(j>>3) .. 8*(j>>3)+7: key j uses word r[(j >> 1) & 3], its low 16
  bits when j is even and its high 16 bits when j is odd;
* keep(i, j)  <=>  u16(i, j) >= t,  t = round-half-even(p * 65536) in double.
  p = 0 gives t = 0 (keep everything).

All arithmetic is on NumPy uint64 arrays masked to 32 bits, vectorised over
counters.
"""

import numpy as np

# Philox4x32 round multipliers and key (Weyl) increments, SC'11 paper.
PHILOX_M0 = 0xD2511F53
PHILOX_M1 = 0xCD9E8D57
PHILOX_W0 = 0x9E3779B9
PHILOX_W1 = 0xBB67AE85
ROUNDS = 10

_MASK32 = np.uint64(0xFFFFFFFF)


def _mulhilo(a, m):
    """(hi, lo) 32-bit halves of the 64-bit product a*m (a: uint64 array < 2^32)."""
    prod = a * np.uint64(m)  # < 2^64, exact in uint64
    return prod >> np.uint64(32), prod & _MASK32


def philox4x32(c0, c1, c2, c3, k0, k1, rounds=ROUNDS):
    """Philox4x32-R bijection of the 128-bit counter under the 64-bit key.

    Arguments are integers or integer arrays (broadcast together), each in
    [0, 2^32).  Returns four uint64 arrays holding the 32-bit output words.
    One round maps (c0, c1, c2, c3) to
        (hi(M1*c2) ^ c1 ^ k0,  lo(M1*c2),  hi(M0*c0) ^ c3 ^ k1,  lo(M0*c0))
    and the key is advanced by the Weyl increments between rounds.
    """
    c0, c1, c2, c3 = (np.asarray(x, dtype=np.uint64) & _MASK32 for x in (c0, c1, c2, c3))
    c0, c1, c2, c3 = np.broadcast_arrays(c0, c1, c2, c3)
    k0 = np.uint64(int(k0) & 0xFFFFFFFF)
    k1 = np.uint64(int(k1) & 0xFFFFFFFF)
    for r in range(rounds):
        if r:
            k0 = np.uint64((int(k0) + PHILOX_W0) & 0xFFFFFFFF)
            k1 = np.uint64((int(k1) + PHILOX_W1) & 0xFFFFFFFF)
        hi0, lo0 = _mulhilo(c0, PHILOX_M0)
        hi1, lo1 = _mulhilo(c2, PHILOX_M1)
        c0, c1, c2, c3 = (hi1 ^ c1 ^ k0) & _MASK32, lo1, (hi0 ^ c3 ^ k1) & _MASK32, lo0
    return c0, c1, c2, c3


def keep_threshold(p_drop):
    """t = round-half-even(p * 65536), computed in double precision."""
    p = float(p_drop)
    if not (0.0 <= p < 1.0):
        raise ValueError("p_drop must lie in [0, 1)")
    return int(np.round(p * 65536.0))  # np.round rounds half to even


def uniform16(seed, b, h, rows, cols):
    """u16(i, j) for every i in ``rows`` and j in ``cols`` -> uint32 array [len(rows), len(cols)]."""
    rows = np.asarray(rows, dtype=np.uint64).reshape(-1)
    cols = np.asarray(cols, dtype=np.int64).reshape(-1)
    seed = int(seed)
    k0, k1 = seed & 0xFFFFFFFF, (seed >> 32) & 0xFFFFFFFF
    groups, inv = np.unique(cols >> 3, return_inverse=True)
    r = philox4x32(groups[None, :].astype(np.uint64), rows[:, None], np.uint64(h), np.uint64(b), k0, k1)
    words = np.stack(r, axis=-1)  # [R, G, 4]
    word_idx = (cols >> 1) & 3
    w = words[:, inv, word_idx]  # [R, C]
    shift = np.where((cols & 1) == 1, 16, 0).astype(np.uint64)
    return ((w >> shift[None, :]) & np.uint64(0xFFFF)).astype(np.uint32)


def keep_mask(seed, b, h, rows, cols, p_drop):
    """Bernoulli keep mask Z[i, j] in {0, 1} (bool) for the given rows and columns."""
    t = keep_threshold(p_drop)
    if t == 0:
        return np.ones((len(np.atleast_1d(rows)), len(np.atleast_1d(cols))), dtype=bool)
    return uniform16(seed, b, h, rows, cols) >= np.uint32(t)
