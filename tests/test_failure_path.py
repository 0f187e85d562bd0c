"""The failure path of the kernels' bounded device waits, exercised without a
GPU fault: a wait that nothing releases runs out, the kernel records
FA_ERR_TIMEOUT in the device error word and returns, the host reads the
status, and the context keeps working."""
import pytest
import torch

import exact_attention_109_b200 as fa
from exact_attention_109_b200.inputs import default_scale
from parity_util import check_forward_full, gpu_inputs, run_forward

pytestmark = pytest.mark.gpu


def test_wait_that_runs_out_reports_timeout_and_context_survives():
    assert fa.fa_get_device_error() == fa.FA_OK          # start clean
    assert fa.fa_selftest_wait_timeout(20_000) == fa.FA_OK  # 20 ms limit
    assert fa.fa_get_device_error() == fa.FA_ERR_TIMEOUT
    assert fa.fa_get_device_error() == fa.FA_OK          # the word was cleared
    host, dev = gpu_inputs(1, 2, 300, 128, seed=7)
    o, lse = run_forward(dev, True, default_scale(128))
    check_forward_full(host, o, lse, True, default_scale(128))


def test_selftest_rejects_out_of_range_limits():
    assert fa.fa_selftest_wait_timeout(0) == fa.FA_ERR_INVALID_ARG
    assert fa.fa_selftest_wait_timeout(3_000_000) == fa.FA_ERR_INVALID_ARG
