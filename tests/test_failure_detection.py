"""Failure detection without a fault: the bounded device wait used by every tensor-core kernel
gives up after its limit, reports MLA_ERR_TIMEOUT through dev_status and leaves the context
usable (a wait on a barrier that nothing completes, by construction)."""
import time

import pytest

pytestmark = pytest.mark.gpu


def test_bounded_wait_reports_timeout_and_context_survives(lib):
    import torch
    mla = lib
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    torch.cuda.synchronize()
    t0 = time.time()
    mla.mla_wait_selftest(20_000_000, st)          # 20 ms limit
    torch.cuda.synchronize()
    elapsed = time.time() - t0
    assert mla.STATUS[int(st.item())] == "MLA_ERR_TIMEOUT"
    assert elapsed < 2.0, elapsed
    # The first error wins: a second expiry leaves the status as it is.
    mla.mla_wait_selftest(1_000_000, st)
    torch.cuda.synchronize()
    assert mla.STATUS[int(st.item())] == "MLA_ERR_TIMEOUT"
    # The context is still usable: a real computation afterwards runs and is correct.
    x = torch.arange(1 << 20, device="cuda", dtype=torch.float32)
    assert float(x.sum().item()) == float((1 << 20) * ((1 << 20) - 1) // 2)


def test_selftest_rejects_bad_arguments(lib):
    import torch
    mla = lib
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    for bad in (0, -5, 10**11):
        with pytest.raises(mla.MlaError):
            mla.mla_wait_selftest(bad, st)
