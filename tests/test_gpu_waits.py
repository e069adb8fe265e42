"""Failure detection without a GPU fault: a kernel waits on an mbarrier that
nothing will complete; its bounded wait must give up, record SPK_ERR_TIMEOUT
in the device error word and return, leaving the context usable."""
import pytest

pytestmark = pytest.mark.gpu


def test_bounded_wait_times_out_cleanly():
    import torch
    from prompt_compression_b200 import build
    build.build_library()
    import prompt_compression_b200 as P
    P.spk_device_error(clear=True)
    P.spk_selftest_wait_timeout(2_000_000)           # 2 ms limit
    st, site = P.spk_device_error(clear=True)
    assert st == P.binding.SPK_ERR_TIMEOUT and site == 999
    x = torch.arange(10, device="cuda", dtype=torch.float32)
    assert float(x.sum().item()) == 45.0              # the context still works
    assert P.spk_device_error() == (0, 0)
