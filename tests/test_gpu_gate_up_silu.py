"""GPU parity of the gate/up GEMM with the SiLU-gated product quantized in its
epilogue (fp8bq_gemm_silu_mul_quantize).

Pages: "ProCreations/Nanbeige4.3-33B-DFlash2", "Architecture and checkpoint
format" (separate gate and up projections of the MLP) and
"ProCreations/Nanbeige4.3-33B-FP8", introduction (the down projection takes
group-128 dynamically quantized activations).

* The fused call equals, bit for bit, the two-step chain it replaces:
  fp8bq_gemm into the BF16 gate/up output, then fp8bq_silu_mul_quantize (codes,
  scales and h), on the prefill kernel (M > 128: ragged M, several tiles, the
  full drafter shape) and on the decode-sized fallback.
* Against the oracle: codes and scales bit-exact with the oracle's group-128
  quantization of the kernel's h, and h within the bound that the GEMM
  tolerance implies through silu(g) * u (derived in _h_bound).
"""
import numpy as np
import pytest
import torch

import fp8_block_scaled_09_b200 as fp8bq
import oracle
import workloads
from gpu_util import Guarded, to_dev_codes, to_dev_f32

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _device():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    fp8bq.lib()
    yield
    assert fp8bq.last_device_status() == 0


def _operands(M, I, K, seed):
    x = workloads.activation(M, K, seed, outliers=min(7, K // 128))
    w = workloads.weight(2 * I, K, seed + 1)
    qa, sa = oracle.quantize_act(x)
    qw, sw = oracle.quantize_weight(w)
    return qa, sa, qw, sw


def _fused(qa, sa, qw, sw, M, I):
    q = Guarded((M, I), torch.uint8)
    s = Guarded((M, I // 128), torch.float32)
    h = Guarded((M, I), torch.bfloat16)
    fp8bq.gemm_silu_mul_quantize(qa, sa, qw, sw, q=q.t, s=s.t, h=h.t)
    torch.cuda.synchronize()
    assert q.guards_intact() and s.guards_intact() and h.guards_intact()
    return q.t, s.t, h.t


def _chain(qa, sa, qw, sw, M, I):
    gu = fp8bq.gemm(qa, sa, qw, sw)
    h = torch.empty((M, I), dtype=torch.bfloat16, device="cuda")
    q, s = fp8bq.silu_mul_quantize(gu, h=h)
    torch.cuda.synchronize()
    return q, s, h


@pytest.mark.parametrize("M,I,K", [
    (129, 128, 128), (300, 256, 384), (1000, 384, 1024), (257, 640, 7168), (4096, 8192, 7168),
    (1, 256, 1024), (16, 384, 7168), (100, 256, 512), (128, 128, 256),
])
def test_fused_equals_gemm_then_silu_mul_quantize(M, I, K):
    hqa, hsa, hqw, hsw = _operands(M, I, K, 50 + M)
    qa, sa, qw, sw = to_dev_codes(hqa), to_dev_f32(hsa), to_dev_codes(hqw), to_dev_f32(hsw)
    fq, fs, fh = _fused(qa, sa, qw, sw, M, I)
    cq, cs, ch = _chain(qa, sa, qw, sw, M, I)
    assert torch.equal(fh.view(torch.int16), ch.view(torch.int16)), \
        f"h differs at {int((fh.view(torch.int16) != ch.view(torch.int16)).sum())} elements"
    assert torch.equal(fs.view(torch.int32), cs.view(torch.int32))
    assert torch.equal(fq, cq)


def _h_bound(gu_ref, I):
    """Bound on |h - h_ref| where h_ref = silu(g') u' with g', u' the BF16-rounded
    FP64 gate/up references.  The kernel's g (and u) differ from g' by at most
    the GEMM tolerance 1e-2 |g| + 2e-3 rms plus one BF16 step 2^-7 |g| (both
    values are rounded to BF16); |d silu / dg| <= 1.1; the final rounding of h
    and the fast exponential add at most 2^-7 |h|."""
    g, u = gu_ref[:, :I], gu_ref[:, I:]
    tol_g = 1e-2 * np.abs(g) + 2e-3 * np.sqrt(np.mean(g * g)) + 2.0 ** -7 * np.abs(g)
    tol_u = 1e-2 * np.abs(u) + 2e-3 * np.sqrt(np.mean(u * u)) + 2.0 ** -7 * np.abs(u)
    silu = g / (1.0 + np.exp(-g))
    h = silu * u
    return 1.1 * np.abs(u) * tol_g + (np.abs(silu) + 1.1 * tol_g) * tol_u + 2.0 ** -7 * np.abs(h) + 1e-30


@pytest.mark.parametrize("M,I,K", [(300, 256, 384), (200, 512, 7168), (64, 256, 1024)])
def test_fused_matches_oracle(M, I, K):
    hqa, hsa, hqw, hsw = _operands(M, I, K, 70 + M)
    qa, sa, qw, sw = to_dev_codes(hqa), to_dev_f32(hsa), to_dev_codes(hqw), to_dev_f32(hsw)
    q, s, h = _fused(qa, sa, qw, sw, M, I)
    # codes and scales: exactly the oracle's quantization of the kernel's h
    oq, os_ = oracle.quantize_act(h.cpu())
    assert np.array_equal(os_.view(np.uint32), s.cpu().numpy().view(np.uint32))
    assert np.array_equal(oq, q.cpu().numpy())
    # h: against silu(g') u' from the oracle's FP64 GEMM, rounded to BF16
    gu_ref = oracle.gemm_ref(hqa, hsa, hqw, hsw)
    gu_bits = oracle.bf16_round(gu_ref)
    h_ref = oracle.silu_mul(gu_bits)
    gu_b = gu_bits.astype(np.uint32) << 16
    gu_b = gu_b.view(np.float32).astype(np.float64)
    bound = _h_bound(gu_b, I)
    err = np.abs(h.float().cpu().numpy().astype(np.float64) - h_ref)
    worst = float((err / bound).max())
    assert worst <= 1.0, f"h outside the derived bound: worst error/bound {worst:.3f}"


def test_fused_workspace_and_repeated_calls():
    # decode-sized M needs the workspace (GEMM part + BF16 gate/up); two calls in
    # a row on one workspace give identical results (its counters return to zero)
    M, I, K = 8, 384, 7168
    hqa, hsa, hqw, hsw = _operands(M, I, K, 90)
    qa, sa, qw, sw = to_dev_codes(hqa), to_dev_f32(hsa), to_dev_codes(hqw), to_dev_f32(hsw)
    assert fp8bq.workspace_size(fp8bq.OP_GEMM_SILU, M, 2 * I, K) > 0
    assert fp8bq.workspace_size(fp8bq.OP_GEMM_SILU, 300, 2 * I, K) == 0
    ws = fp8bq.new_workspace(fp8bq.OP_GEMM_SILU, M, 2 * I, K, "cuda")
    out = []
    for _ in range(2):
        q, s = fp8bq.gemm_silu_mul_quantize(qa, sa, qw, sw, workspace=ws)
        out.append((q.clone(), s.clone()))
    torch.cuda.synchronize()
    assert torch.equal(out[0][0], out[1][0]) and torch.equal(out[0][1], out[1][1])
    assert int(ws[:16384].count_nonzero()) == 0
