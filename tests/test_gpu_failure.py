"""The failure channel on the GPU, exercised without a fault.

tok_selftest_wait_timeout launches a kernel whose shared-memory barrier waits for a
copy that is never issued; its bounded wait runs out after a few thousand polls, it
counts a timeout the way the TMA kernels do and returns.  tok_check_device must then
report TOK_ERR_TIMEOUT once, clear the record, and the device must stay usable.
"""
import pytest
import torch

import haar_wavelet_patching_b200 as hwp

pytestmark = pytest.mark.gpu


def test_wait_that_runs_out_is_reported_once_and_cleared():
    hwp.tok_check_device()                    # nothing pending from earlier calls
    hwp.tok_selftest_wait_timeout(4096)
    with pytest.raises(hwp.TokError) as e:
        hwp.tok_check_device()
    assert e.value.status == hwp.TOK_ERR_TIMEOUT
    hwp.tok_check_device()                    # the record was cleared: TOK_OK


def test_device_is_usable_after_a_timeout():
    hwp.tok_selftest_wait_timeout(4096)
    hwp.tok_selftest_wait_timeout(4096)
    with pytest.raises(hwp.TokError) as e:
        hwp.tok_check_device()
    assert e.value.status == hwp.TOK_ERR_TIMEOUT
    x = torch.full((1, 2, 5, 8, 16), 0.5, device="cuda")
    y = hwp.haar_fwd(x)
    hwp.tok_check_device()
    assert torch.all(y[:, :2] == 4.0) and torch.all(y[:, 2:] == 0)
