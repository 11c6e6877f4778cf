"""Dropout mask parity: the device Philox (fa_dropout_mask) and the mask the
forward kernel actually applies must equal the oracle's mask bit for bit."""

import numpy as np
import pytest
import torch

from oracle import philox

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
