"""Failure detection on the GPU without a fault: a bounded device-side wait that
nothing satisfies must give up, record LQ_ERR_DEVICE_TIMEOUT, and leave the
context usable (the next calls succeed)."""
import numpy as np
import pytest
import torch

from bit_ptq_looped_b200 import lq

pytestmark = pytest.mark.gpu


def test_bounded_wait_times_out_and_reports():
    lq.lq_check_device()  # clean state
    lq.lq_selftest_bounded_wait(2000)  # 2 ms limit
    with pytest.raises(lq.LQError) as e:
        lq.lq_check_device()
    assert e.value.status == lq.LQ_ERR_DEVICE_TIMEOUT
    lq.lq_check_device()  # the status word was cleared
    # the context still works: a quantize call runs and is checked
    x = torch.arange(64, dtype=torch.float32, device="cuda").reshape(2, 32) - 31.5
    q8, _, s = lq.lq_quantize_act(x, None, None, 1.0, 4)
    torch.cuda.synchronize()
    assert torch.all(q8.abs() <= 7)
    assert np.isclose(s[0, 0].item(), 31.5 / 7)


def test_selftest_rejects_bad_limits():
    for bad in (0, -5, 10**8):
        with pytest.raises(lq.LQError) as e:
            lq.lq_selftest_bounded_wait(bad)
        assert e.value.status == lq.LQ_ERR_ARG


def test_grid_barrier_times_out_and_reports():
    """The persistent decode kernel's grid barrier, waiting for a block that
    never arrives, gives up after its limit and records the timeout."""
    lq.lq_check_device()
    scratch = torch.zeros(2, dtype=torch.int32, device="cuda")
    lq.lq_selftest_grid_wait(scratch, 2000)  # 2 ms limit
    with pytest.raises(lq.LQError) as e:
        lq.lq_check_device()
    assert e.value.status == lq.LQ_ERR_DEVICE_TIMEOUT
    lq.lq_check_device()  # cleared
    with pytest.raises(lq.LQError) as e:
        lq.lq_selftest_grid_wait(scratch, 0)
    assert e.value.status == lq.LQ_ERR_ARG
