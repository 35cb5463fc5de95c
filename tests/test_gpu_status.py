"""Failure detection without a GPU fault: a kernel waits on an mbarrier that
nothing arrives on, with a 50 ms limit; it must record JATTN_DEV_TIMEOUT in
the device status word and return, leaving the context usable."""
import pytest
import torch

from diffusion_transformer_joint_jattn_b200 import jattn

pytestmark = pytest.mark.gpu


def test_bounded_wait_times_out_and_reports(cuda_device):
    jattn.device_status(clear=True)
    jattn.selftest_wait_timeout(50)
    # the boundary's query reports it without clearing the word
    assert jattn.last_device_status() == jattn.ERR_TIMEOUT
    assert jattn.last_device_status() == jattn.ERR_TIMEOUT
    code, bits = jattn.device_status(clear=True)
    assert code == jattn.ERR_TIMEOUT and bits & jattn.DEV_TIMEOUT
    # the status is cleared and the context still runs work
    assert jattn.device_status(clear=False) == (jattn.OK, 0)
    assert jattn.last_device_status() == jattn.OK
    x = torch.ones(4, device=cuda_device)
    assert float((x * 2).sum()) == 8.0
