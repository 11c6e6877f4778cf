"""Dropout mask parity: the device Philox (fa_dropout_mask) and the masks the
forward and backward kernels actually apply must equal the oracle's mask bit
for bit."""

import numpy as np
import pytest
import torch

from oracle import philox
from tests import parity_util as pu

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("B,H,N,p,seed", [
    (1, 1, 128, 0.1, 2), (2, 3, 200, 0.1, 0xFFFFFFFF00000001), (1, 2, 1000, 0.5, 4), (1, 1, 256, 0.7, 9),
    (1, 1, 64, 0.0, 3),
])
def test_device_mask_matches_oracle(B, H, N, p, seed):
    from exact_io_aware_49_b200 import fa_dropout_mask
    m = fa_dropout_mask(B, H, N, p, seed).cpu().numpy()
    for b in range(B):
        for h in range(H):
            want = philox.keep_mask(seed, b, h, np.arange(N), np.arange(N), p)
            np.testing.assert_array_equal(m[b, h].astype(bool), want)


@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("N,p,seed", [(1024, 0.1, 2), (512, 0.7, 11)])
def test_forward_applies_oracle_mask(causal, N, p, seed):
    """Q = 0 makes P uniform; V[j] = e_(j - w0) on a 64-key window selects one
    column of P_drop per output column, so O[i, c] != 0 exactly when key w0 + c
    is kept for row i.  Head h uses window w0 = 64 h, so the heads together
    cover every key."""
    from exact_io_aware_49_b200 import fa_fwd
    d = 64
    H = N // 64
    q = torch.zeros(1, H, N, d, dtype=torch.bfloat16, device="cuda")
    k = torch.randn(1, H, N, d, dtype=torch.bfloat16, device="cuda")
    v = torch.zeros(1, H, N, d, dtype=torch.bfloat16)
    for h in range(H):
        v[0, h, 64 * h:64 * h + 64] = torch.eye(64, dtype=torch.bfloat16)
    o, _ = fa_fwd(q, k, v.cuda(), causal, 0.125, p, seed)
    o = o.cpu().to(torch.float32).numpy()
    rows = np.arange(N)
    for h in range(H):
        cols = np.arange(64 * h, 64 * h + 64)
        want = philox.keep_mask(seed, 0, h, rows, cols, p)
        got = o[0, h] != 0.0
        if causal:
            valid = cols[None, :] <= rows[:, None]
            np.testing.assert_array_equal(got[valid], want[valid])
            assert not got[~valid].any()
        else:
            np.testing.assert_array_equal(got, want)


def _backward_mask_windows(B, H, N, d, causal, p, seed, windows):
    """Bit-exact check of the mask the backward kernel regenerates.

    Q = 0 makes every visible score 0, so P is uniform over the visible keys;
    dO[i] = e_(i - w0) for the d query rows i = w0 .. w0 + d - 1 of a window
    (zero elsewhere) makes dV[j, c] = P_d[w0 + c, j] = Z[w0 + c, j] / (n (1 - p)):
    non-zero exactly where key j is kept for query w0 + c (and visible to it).
    The backward draws its mask through its own code path (per-key threads,
    shuffled bit blocks), independent of the forward's."""
    from exact_io_aware_49_b200 import fa_bwd, fa_fwd, fa_last_device_error
    g = torch.Generator(device="cuda").manual_seed(seed)
    q = torch.zeros(B, H, N, d, dtype=torch.bfloat16, device="cuda")
    k = torch.randn(B, H, N, d, generator=g, device="cuda").to(torch.bfloat16)
    v = torch.randn(B, H, N, d, generator=g, device="cuda").to(torch.bfloat16)
    o, lse = fa_fwd(q, k, v, causal, d ** -0.5, p, seed)
    cols = np.arange(N)
    for w0 in windows:
        n_c = min(d, N - w0)
        do = torch.zeros(B, H, N, d, dtype=torch.bfloat16, device="cuda")
        idx = torch.arange(n_c, device="cuda")
        do[:, :, w0 + idx, idx] = 1.0
        _, _, dv = fa_bwd(q, k, v, o, do, lse, causal, d ** -0.5, p, seed)
        got_all = (dv[:, :, :, :n_c] != 0).cpu().numpy()
        rows = np.arange(w0, w0 + n_c)

        def one(bh):
            b, h = bh
            want = philox.keep_mask(seed, b, h, rows, cols, p).T  # [key j, window column c]
            got = got_all[b, h]
            if causal:
                valid = cols[:, None] <= rows[None, :]
                np.testing.assert_array_equal(got[valid], want[valid], err_msg=f"window {w0} head {(b, h)}")
                assert not got[~valid].any(), f"window {w0} head {(b, h)}: masked key has a gradient"
            else:
                np.testing.assert_array_equal(got, want, err_msg=f"window {w0} head {(b, h)}")

        pu.map_heads(one, [(b, h) for b in range(B) for h in range(H)])
    torch.cuda.synchronize()
    assert fa_last_device_error() == 0


@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("N,d,p,seed", [(1024, 128, 0.1, 2), (1024, 128, 0.7, 11), (333, 64, 0.1, 0xFFFFFFFF00000005)])
def test_backward_applies_oracle_mask_every_query(causal, N, d, p, seed):
    """Windows of d queries slid over every query row (ragged last window for N = 333)."""
    _backward_mask_windows(2, 3, N, d, causal, p, seed, list(range(0, N, d)))


@pytest.mark.parametrize("causal,p", [(True, 0.1), (False, 0.7)])
@pytest.mark.parametrize("B,H,N,seed", [(4, 16, 4096, 2), (1, 32, 32768, 4)])
def test_backward_applies_oracle_mask_full_size(B, H, N, seed, causal, p):
    """The two dropout workloads' shapes (d = 128): sampled windows at the
    start, in the middle and at the end, on every head; the workloads' own
    causal p = 0.1 and a non-causal p = 0.7 case (every key visible, most of
    them dropped)."""
    _backward_mask_windows(B, H, N, 128, causal, p, seed, [0, N // 2 - 64, N - 128])
