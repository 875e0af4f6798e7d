"""GPU parity of the NVFP4 weight-only (A16) path.

Page "ProCreations/Nanbeige4.3-33B-NVFP4-A16", recipe paragraph: FP4 E2M1
weights in groups of 16 with E4M3 block scales and a global scale, BF16
activations.  The quantizer's packed codes, block scales and global scale are
bit-exact with the oracle's min-max quantizer; the GEMM is within the library
tolerance of the oracle's FP64 X . dequant(W)^T, on decode shapes (one and
several clusters, ragged M), a multi-tile M and the full QKV / o_proj weights.
"""
import numpy as np
import pytest
import torch

import fp8_block_scaled_09_b200 as fp8bq
import oracle
import workloads
from gpu_util import Guarded, bf16_to_f64, tolerance_report

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _device():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    fp8bq.lib()
    yield
    assert fp8bq.last_device_status() == 0


def _check(y, ref):
    ok, ratio, rms = tolerance_report(y, ref)
    assert ok, f"worst error / bound = {ratio:.3f} (rms(ref) = {rms:.4g})"


@pytest.mark.parametrize("N,K,seed", [(128, 256, 1), (384, 1024, 2), (1024, 7168, 3)])
def test_nvfp4_quantize_weight_bit_exact(N, K, seed):
    w = workloads.weight(N, K, seed)
    w[0, 7] = 0.5                            # sets the global scale
    w[5, 64:80] = 0.0                        # an all-zero group
    packed, sb, g = fp8bq.nvfp4_quantize_weight(w.cuda())
    torch.cuda.synchronize()
    rp, rsb, rg = oracle.nvfp4_quantize(w)
    assert g.item() == rg
    assert np.array_equal(sb.cpu().numpy(), rsb)
    assert np.array_equal(packed.cpu().numpy(), rp)


def test_nvfp4_quantize_weight_full_qkv():
    g = workloads.by_name("qkv_m1")
    w = g.make_w()
    packed, sb, gs = fp8bq.nvfp4_quantize_weight(w.cuda())
    torch.cuda.synchronize()
    rp, rsb, rg = oracle.nvfp4_quantize(w)
    assert gs.item() == rg
    assert np.array_equal(sb.cpu().numpy(), rsb) and np.array_equal(packed.cpu().numpy(), rp)


def _run(M, N, K, seed):
    x = workloads.activation(M, K, seed, outliers=max(1, K // 1024))
    w = workloads.weight(N, K, seed + 1)
    packed, sb, g = oracle.nvfp4_quantize(w)
    pd = torch.from_numpy(packed).cuda()
    sd = torch.from_numpy(sb).cuda()
    gd = torch.tensor([g], dtype=torch.float32, device="cuda")
    y = Guarded((M, N), torch.bfloat16)
    fp8bq.nvfp4_gemm_a16(x.cuda(), pd, sd, gd, out=y.t)
    torch.cuda.synchronize()
    assert y.guards_intact()
    return x, packed, sb, g, y.t


# M <= 2 runs the CUDA-core kernel (token buckets 1, 2), larger M the tensor-core one
@pytest.mark.parametrize("M,N,K", [(1, 128, 256), (4, 384, 1024), (16, 1024, 7168),
                                   (7, 640, 2048), (1, 9216, 7168), (8, 7168, 7168),
                                   (33, 256, 512), (3, 20480, 256), (2, 9216, 7168),
                                   (2, 128, 21504), (3, 1024, 7168)])
def test_nvfp4_gemm_a16_matches_oracle(M, N, K):
    x, packed, sb, g, y = _run(M, N, K, 50 + M)
    _check(bf16_to_f64(y), oracle.nvfp4_gemm_ref(x, packed, sb, g))


@pytest.mark.parametrize("M", [1, 2, 3, 5])
def test_nvfp4_gemm_a16_exact_regime_bit_exact(M):
    # small-integer activations and power-of-two block scales: every partial sum
    # is exact in FP32, so the output is the BF16 rounding of the exact value
    rng = np.random.default_rng(9 + M)
    N, K = 256, 512
    x = torch.from_numpy(rng.integers(-3, 4, (M, K)).astype(np.float32)).to(torch.bfloat16)
    packed = rng.integers(0, 256, (N, K // 2)).astype(np.uint8)
    sb = rng.choice(np.array([0x30, 0x38, 0x40], np.uint8), size=(N, K // 16))  # 0.5, 1, 2
    g = 0.25
    y = fp8bq.nvfp4_gemm_a16(x.cuda(), torch.from_numpy(packed).cuda(), torch.from_numpy(sb).cuda(),
                             torch.tensor([g], dtype=torch.float32, device="cuda"))
    torch.cuda.synchronize()
    ref = oracle.nvfp4_gemm_ref(x, packed, sb, g)
    got = y.cpu().view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(got, oracle.bf16_round(ref))


@pytest.mark.parametrize("M", [2, 6])
def test_nvfp4_gemm_a16_every_code_and_sign(M):
    # each row of W cycles through all 16 E2M1 codes: the code decoding of both
    # kernels (magnitudes, signs, nibble order) is checked against the oracle
    N, K = 128, 256
    codes = (np.arange(N * K) % 16).astype(np.uint8).reshape(N, K)
    packed = (codes[:, 0::2] | (codes[:, 1::2] << 4)).astype(np.uint8)
    sb = np.full((N, K // 16), 0x38, np.uint8)
    x = torch.eye(K, dtype=torch.bfloat16)[:M]           # rows pick single columns of W
    y = fp8bq.nvfp4_gemm_a16(x.cuda(), torch.from_numpy(packed).cuda(), torch.from_numpy(sb).cuda(),
                             torch.tensor([1.0], dtype=torch.float32, device="cuda"))
    torch.cuda.synchronize()
    ref = oracle.nvfp4_gemm_ref(x, packed, sb, 1.0)
    assert np.array_equal(bf16_to_f64(y), ref)


def test_nvfp4_quantize_then_gemm_on_the_gpu():
    M, N, K = 4, 1152, 2048
    x = workloads.activation(M, K, 31, outliers=2)
    w = workloads.weight(N, K, 32)
    packed, sb, g = fp8bq.nvfp4_quantize_weight(w.cuda())
    y = fp8bq.nvfp4_gemm_a16(x.cuda(), packed, sb, g)
    torch.cuda.synchronize()
    rp, rsb, rg = oracle.nvfp4_quantize(w)
    _check(bf16_to_f64(y), oracle.nvfp4_gemm_ref(x, rp, rsb, rg))
