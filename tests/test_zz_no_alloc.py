"""fp8bq_gemm_noalloc: the GEMM for callers that cannot allocate device memory.

Some callers have no allocator to call (an embedding runtime that hands the
library fixed buffers only, or code running where cudaMalloc is not allowed),
so they cannot supply the workspace fp8bq_gemm asks for.  fp8bq_gemm_noalloc
uses scratch built into the library instead.  These tests call it through the
C ABI and check, on two calls in a row, that its output matches the existing
entry point fp8bq_gemm and the oracle's FP64 reference within the accuracy
tolerance the other GPU tests use, that 16 < M <= 128 problems too big for the
built-in scratch run correctly on the kernel that needs none, and that an
M <= 16 problem too big for it is refused before any work is queued.  The file
is named so that pytest collects it last.
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


def _host_operands(M, N, K, seed):
    x = workloads.activation(M, K, seed, outliers=3)
    w = workloads.weight(N, K, seed + 1)
    qa, sa = oracle.quantize_act(x)
    qw, sw = oracle.quantize_weight(w)
    return qa, sa, qw, sw


def _operands(M, N, K, seed):
    qa, sa, qw, sw = _host_operands(M, N, K, seed)
    return to_dev_codes(qa), to_dev_f32(sa), to_dev_codes(qw), to_dev_f32(sw)


def _check(y, ref, what):
    ok, ratio, _ = tolerance_report(bf16_to_f64(y), ref)
    assert ok, f"fp8bq_gemm_noalloc differs from {what}: worst error/bound {ratio:.3f}"


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
        hqa, hsa, hqw, hsw = _host_operands(M, N, K, seed)
        qa, sa, qw, sw = to_dev_codes(hqa), to_dev_f32(hsa), to_dev_codes(hqw), to_dev_f32(hsw)
        y_ref = fp8bq.gemm(qa, sa, qw, sw)
        y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
        assert _noalloc_via_c_abi(qa, sa, qw, sw, y) == 0
        torch.cuda.synchronize()
        _check(y, bf16_to_f64(y_ref), "fp8bq_gemm")
        _check(y, oracle.gemm_ref(hqa, hsa, hqw, hsw), "the oracle")


@pytest.mark.parametrize("M,N,K", [(64, 20480, 1024), (17, 24576, 7168)])
def test_noalloc_beyond_its_scratch_with_mid_size_m(M, N, K):
    # 16 < M <= 128 with more n-blocks than SMs: the decode kernel would take
    # stream-K, whose split-K scratch is larger than the built-in array, so the
    # call runs on the kernel that needs none (a single partial row tile here).
    # Two calls in a row, against the oracle and against fp8bq_gemm.
    assert M > 16 and N // 128 > torch.cuda.get_device_properties(0).multi_processor_count
    hqa, hsa, hqw, hsw = _host_operands(M, N, K, 31)
    qa, sa, qw, sw = to_dev_codes(hqa), to_dev_f32(hsa), to_dev_codes(hqw), to_dev_f32(hsw)
    rows = np.unique(np.array([0, 1, M // 2, M - 1], dtype=np.int64))
    ref = oracle.gemm_ref(hqa, hsa, hqw, hsw, rows=rows)
    y_gemm = bf16_to_f64(fp8bq.gemm(qa, sa, qw, sw))
    for _ in range(2):
        y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
        assert _noalloc_via_c_abi(qa, sa, qw, sw, y) == 0
        torch.cuda.synchronize()
        assert fp8bq.last_device_status() == 0
        _check(y, y_gemm, "fp8bq_gemm")
        _check(y[torch.from_numpy(rows).cuda()], ref, "the oracle")


def test_noalloc_repeated_calls_keep_agreeing():
    # the built-in scratch keeps the previous call's contents; back-to-back calls
    # on the same inputs must still agree with the workspace entry point
    hqa, hsa, hqw, hsw = _host_operands(4, 7168, 7168, 21)
    qa, sa, qw, sw = to_dev_codes(hqa), to_dev_f32(hsa), to_dev_codes(hqw), to_dev_f32(hsw)
    y_ref = bf16_to_f64(fp8bq.gemm(qa, sa, qw, sw))
    ref = oracle.gemm_ref(hqa, hsa, hqw, hsw)
    for _ in range(2):
        y = torch.empty((4, 7168), dtype=torch.bfloat16, device="cuda")
        fp8bq.gemm_noalloc(qa, sa, qw, sw, out=y)
        torch.cuda.synchronize()
        _check(y, y_ref, "fp8bq_gemm")
        _check(y, ref, "the oracle")


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
