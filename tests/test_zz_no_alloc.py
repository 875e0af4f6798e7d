"""fp8bq_gemm_noalloc: the GEMM for callers that cannot allocate device memory.

Some callers have no allocator to call (an embedding runtime that hands the
library fixed buffers only, or code running where cudaMalloc is not allowed),
so they cannot supply the workspace fp8bq_gemm asks for.  fp8bq_gemm_noalloc
uses scratch built into the library instead.  These tests call it through the
C ABI and check, on two calls in a row, that its output matches the existing
entry point fp8bq_gemm within the accuracy tolerance the other GPU tests use,
and that a problem too big for the built-in scratch is refused before any
work is queued.  The file is named so that pytest collects it last.
"""
import ctypes

import numpy as np
import pytest
import torch

import fp8_block_scaled_09_b200 as fp8bq
import oracle
import workloads
from gpu_util import bf16_to_f64, to_dev_codes, to_dev_f32, tolerance_report

pytestmark = pytest.mark.gpu

WORKSPACE_TOO_SMALL = 4


@pytest.fixture(scope="module", autouse=True)
def _device():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    fp8bq.lib()
    yield
    assert fp8bq.last_device_status() == 0


def _operands(M, N, K, seed):
    x = workloads.activation(M, K, seed, outliers=3)
    w = workloads.weight(N, K, seed + 1)
    qa, sa = oracle.quantize_act(x)
    qw, sw = oracle.quantize_weight(w)
    return to_dev_codes(qa), to_dev_f32(sa), to_dev_codes(qw), to_dev_f32(sw)


def _noalloc_via_c_abi(qa, sa, qw, sw, y):
    M, K = qa.shape
    N = qw.shape[0]
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    P = lambda t: ctypes.c_void_p(t.data_ptr())
    return fp8bq.lib().fp8bq_gemm_noalloc(P(qa), P(sa), P(qw), P(sw), M, N, K, P(y), stream)


@pytest.mark.parametrize("first,second", [((8, 9216, 7168), (16, 1024, 7168)),
                                          ((1, 2048, 1024), (300, 384, 1024)),
                                          ((100, 1152, 7168), (4, 7168, 7168))])
def test_noalloc_matches_gemm_on_two_calls_in_a_row(first, second):
    for (M, N, K), seed in ((first, 11), (second, 12)):
        qa, sa, qw, sw = _operands(M, N, K, seed)
        y_ref = fp8bq.gemm(qa, sa, qw, sw)
        y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
        assert _noalloc_via_c_abi(qa, sa, qw, sw, y) == 0
        torch.cuda.synchronize()
        ok, ratio, _ = tolerance_report(bf16_to_f64(y), bf16_to_f64(y_ref))
        assert ok, f"fp8bq_gemm_noalloc differs from fp8bq_gemm: worst error/bound {ratio:.3f}"


def test_noalloc_repeated_calls_keep_agreeing():
    # the built-in scratch keeps the previous call's contents; back-to-back calls
    # on the same inputs must still agree with the workspace entry point
    qa, sa, qw, sw = _operands(4, 7168, 7168, 21)
    y_ref = bf16_to_f64(fp8bq.gemm(qa, sa, qw, sw))
    for _ in range(2):
        y = torch.empty((4, 7168), dtype=torch.bfloat16, device="cuda")
        fp8bq.gemm_noalloc(qa, sa, qw, sw, out=y)
        torch.cuda.synchronize()
        ok, ratio, _ = tolerance_report(bf16_to_f64(y), y_ref)
        assert ok, f"worst error/bound {ratio:.3f}"


def test_noalloc_refuses_problems_beyond_its_scratch():
    # M <= 16 with N > 32512 needs more split-K scratch than the built-in 4 MiB;
    # the call must refuse on the host, before anything is queued
    M, N, K = 8, 32768, 128
    qa = torch.zeros((M, K), dtype=torch.uint8, device="cuda")
    sa = torch.ones((M, 1), dtype=torch.float32, device="cuda")
    qw = torch.zeros((N, K), dtype=torch.uint8, device="cuda")
    sw = torch.ones((N // 128, 1), dtype=torch.float32, device="cuda")
    y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    assert _noalloc_via_c_abi(qa, sa, qw, sw, y) == WORKSPACE_TOO_SMALL
