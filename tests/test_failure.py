"""Failure detection without a GPU fault: a bounded wait that nothing completes gives up,
the device status word reports FA_ERR_TIMEOUT once, and the context stays usable.

The wait is the same bounded mbarrier wait every kernel's pipeline uses (with a short
limit here); nothing traps, faults or spins without bound."""

import numpy as np
import pytest
import torch

import oracle
from exact_io_aware_63_b200 import binding, inputs
from gpu_helpers import check_all_heads

pytestmark = pytest.mark.gpu

FA_ERR_TIMEOUT = -7


def _wait(arrive, limit_us):
    result = torch.full((1,), -1, dtype=torch.int32, device="cuda:0")
    rc = binding.fa_selftest_wait_timeout(arrive, limit_us, result)
    assert rc == 0, binding.fa_status_string(rc)
    torch.cuda.synchronize()
    return int(result.item())


def test_wait_that_nothing_completes_times_out_and_reports(cuda_device):
    assert binding.fa_get_device_status() == 0
    assert _wait(arrive=0, limit_us=20_000) == 0
    assert binding.fa_get_device_status() == FA_ERR_TIMEOUT
    # reported once: reading the status clears it
    assert binding.fa_get_device_status() == 0


def test_completed_wait_reports_nothing(cuda_device):
    assert _wait(arrive=1, limit_us=20_000) == 1
    assert binding.fa_get_device_status() == 0


def test_context_usable_after_a_timeout(cuda_device):
    assert _wait(arrive=0, limit_us=5_000) == 0
    assert binding.fa_get_device_status() == FA_ERR_TIMEOUT
    # the attention kernels still run and agree with the oracle
    check_all_heads(inputs.make_inputs(1, 2, 256, 64, causal=True, seed=500))
