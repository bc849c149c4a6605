"""Failure detection without a GPU fault: every wait inside the kernels is
bounded; on expiry a kernel records FA_ERR_TIMEOUT in a device status word and
returns, and fa_check() reports it.  The self-test kernel waits on a barrier
that nothing completes, with a short limit."""

import pytest
import torch

import io_aware_exact_forward_b200 as fa

FA_ERR_TIMEOUT = 6


def test_selftest_rejects_bad_limits_on_host():
    lib = fa.load_library()
    assert lib.fa_selftest_bounded_wait(0, None) == 1
    assert lib.fa_selftest_bounded_wait(2_000_000, None) == 1


@pytest.mark.gpu
def test_bounded_wait_reports_timeout_and_context_stays_usable():
    assert fa.check() == 0
    assert fa.selftest_bounded_wait(20_000) == 0       # 20 ms limit
    assert fa.check() == FA_ERR_TIMEOUT               # reported ...
    assert fa.check() == 0                             # ... and cleared
    # the context still works: a small forward runs and succeeds
    q = torch.randn(1, 64, 1, 64, device="cuda").to(torch.bfloat16)
    o, lse = fa.forward(q, q, q)
    assert fa.check() == 0
    assert torch.isfinite(o.float()).all()
