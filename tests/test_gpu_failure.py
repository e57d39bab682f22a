"""Failure handling on the device, without a fault: a bounded wait that runs out reports
MSA_ERR_TIMEOUT through the device error word, and the CTA's abort flag ends every other wait of
the CTA at once, so the kernel finishes after about one limit.  Nothing faults, traps or hangs:
the waits are on mbarriers that nothing arrives on, with a limit of a millisecond."""
import pytest

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def msa(cuda_device):
    import long_context_memory_b200 as m

    return m


@pytest.mark.parametrize("n_waits", [1, 8, 64])
def test_bounded_wait_gives_up_and_reports_timeout(msa, cuda_device, n_waits):
    import torch

    assert msa.check_device_errors() == 0          # a clean word before the test
    limit_us = 1000
    elapsed = msa.selftest_wait_timeout(limit_us, n_waits)
    torch.cuda.synchronize()                         # the kernel returned: the context is usable
    with pytest.raises(msa.MSAError) as e:
        msa.check_device_errors()
    assert e.value.code == 5 and "bounded device wait" in str(e.value)
    assert msa.check_device_errors() == 0          # reading the word cleared it
    ns = int(elapsed.item())
    # four warps, n_waits waits each: one limit in all, not n_waits of them
    assert limit_us * 1000 <= ns < 3 * limit_us * 1000, ns
    # and the device keeps working afterwards
    x = torch.arange(1024, device=cuda_device, dtype=torch.float32)
    assert float(x.sum().item()) == 1023 * 1024 / 2


def test_selftest_rejects_bad_arguments(msa, cuda_device):
    import ctypes

    out = msa.selftest_wait_timeout  # noqa: F841 (binding present)
    assert msa.lib.msa_selftest_wait_timeout(0, 1, 0x10000, None) == 1
    assert msa.lib.msa_selftest_wait_timeout(100, 0, 0x10000, None) == 1
    assert msa.lib.msa_selftest_wait_timeout(100, 1, None, None) == 1
    assert msa.lib.msa_selftest_wait_timeout(200000, 1, 0x10000, None) == 1
    del ctypes
