"""Bounded on-device waits: a wait that nothing will satisfy runs out, records
FP8Q_ERR_TIMEOUT, and the kernel returns; the context stays usable.  Nothing
faults, traps or hangs."""
import numpy as np
import pytest
import torch

import fp8_fine_grained_quant_b200 as fq

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dev():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch.device("cuda:0")


def test_wait_times_out_and_reports(dev):
    assert fq.get_device_error(device=dev) == fq.OK
    fq.selftest_wait_timeout(20_000_000, device=dev)  # 20 ms
    assert fq.get_device_error(device=dev) == fq.ERR_TIMEOUT
    assert fq.get_device_error(device=dev) == fq.OK  # reading clears it


def test_context_usable_after_timeout(dev):
    fq.selftest_wait_timeout(5_000_000, device=dev)
    assert fq.get_device_error(device=dev) == fq.ERR_TIMEOUT
    x = torch.ones((4, 256), dtype=torch.bfloat16, device=dev)
    q, s = fq.fp8_quant_act_1x128(x)
    torch.cuda.synchronize(dev)
    assert torch.all(q.view(torch.uint8) == 0x7E)
    assert fq.get_device_error(device=dev) == fq.OK


def test_launch_counter_counts(dev):
    n0 = fq.launch_count()
    x = torch.ones((4, 256), dtype=torch.bfloat16, device=dev)
    fq.fp8_quant_act_1x128(x)
    assert fq.launch_count() == n0 + 1


def test_set_timeout_roundtrip(dev):
    fq.set_wait_timeout_ns(2_000_000_000)
    fq.set_wait_timeout_ns(0)  # restores the default
