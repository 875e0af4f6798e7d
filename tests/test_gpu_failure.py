"""The failure path on the GPU, without faulting or hanging it: a kernel's
bounded wait on a barrier that nothing arrives on gives up after its limit,
records FP8BQ_ERR_TIMEOUT in the device status word, and returns; the host
reads (and clears) the status, and the context keeps working."""
import numpy as np
import pytest
import torch

import fp8_block_scaled_09_b200 as fp8bq
import oracle
import workloads
from gpu_util import bf16_to_f64, to_dev_codes, to_dev_f32, tolerance_report

pytestmark = pytest.mark.gpu

TIMEOUT = 6


def test_bounded_wait_reports_timeout_and_context_survives():
    assert torch.cuda.is_available()
    assert fp8bq.last_device_status() == 0
    fp8bq.selftest_timeout(20000)                     # 20 ms limit
    assert fp8bq.last_device_status() == TIMEOUT
    assert fp8bq.last_device_status() == 0            # read clears it
    # the context is still usable: a GEMM runs and is correct
    x = workloads.activation(8, 512, 1)
    qw, sw = oracle.quantize_weight(workloads.weight(256, 512, 2))
    y = fp8bq.linear(x.cuda(), to_dev_codes(qw), to_dev_f32(sw))
    torch.cuda.synchronize()
    ok, ratio, _ = tolerance_report(bf16_to_f64(y), oracle.linear_ref(x, qw, sw))
    assert ok, ratio
    assert fp8bq.last_device_status() == 0


def test_selftest_rejects_bad_limits():
    with pytest.raises(fp8bq.Fp8bqError):
        fp8bq.selftest_timeout(0)
    with pytest.raises(fp8bq.Fp8bqError):
        fp8bq.selftest_timeout(3_000_000)
