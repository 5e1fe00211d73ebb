"""Failure detection on the GPU without a fault: a bounded wait on an mbarrier
that nothing completes gives up after its limit, records CP_ERR_TIMEOUT in the
device status word, and the context stays usable."""
import pytest
import torch

import context_zigzag_cp_b200 as cz

pytestmark = pytest.mark.gpu


def test_bounded_wait_times_out_and_context_survives():
    assert cz.get_device_status() == 0
    cz.selftest_wait_timeout(2_000_000)          # 2 ms
    torch.cuda.synchronize()
    assert cz.get_device_status() == 4           # CP_ERR_TIMEOUT
    assert cz.get_device_status() == 0           # read-and-clear
    x = torch.arange(10, device="cuda").sum()    # the context still works
    assert int(x) == 45


def test_wait_limit_roundtrip():
    cz.set_wait_limit_ns(1_500_000_000)
    cz.set_wait_limit_ns(2_000_000_000)
