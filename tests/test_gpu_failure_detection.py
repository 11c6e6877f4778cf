"""Failure detection without a GPU fault.

A kernel wait that can only run out (an mbarrier nothing ever completes,
limit 1 ms) must end by itself, report FA_ERR_TIMEOUT through the device
error word, and leave the context usable for normal work afterwards."""

import pytest
import torch

pytestmark = pytest.mark.gpu


def test_bounded_wait_times_out_and_context_survives():
    from exact_io_aware_49_b200 import fa_fwd, fa_last_device_error, fa_selftest_wait_timeout
    assert fa_last_device_error() == 0
    fa_selftest_wait_timeout(1000)
    torch.cuda.synchronize()
    assert fa_last_device_error() == 4  # FA_ERR_TIMEOUT
    assert fa_last_device_error() == 0  # reading clears it
    q = torch.randn(1, 1, 128, 64, device="cuda", dtype=torch.bfloat16)
    o, lse = fa_fwd(q, q, q, True)
    torch.cuda.synchronize()
    assert torch.isfinite(o.float()).all() and torch.isfinite(lse).all()
    assert fa_last_device_error() == 0


def test_selftest_rejects_bad_limits():
    from exact_io_aware_49_b200 import FAError, fa_selftest_wait_timeout
    with pytest.raises(FAError):
        fa_selftest_wait_timeout(0)
    with pytest.raises(FAError):
        fa_selftest_wait_timeout(2_000_000)
