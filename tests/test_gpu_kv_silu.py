"""GPU parity of the FP8 KV-cache write and the fused SiLU-mul quantizer.

KV write (page "ProCreations/Nanbeige4.3-33B-FP8", "Serving" / "Speed on
Vega": fp8_e4m3 KV cache with unit scales): whole caches bit-exact with the
oracle, rows taken straight from a fused QKV output (row stride 9216), slots
scattered by a permutation, saturating and non-finite values included (NaN
codes compared as NaN), out-of-range slots skipped and reported.

SiLU-gated product (introduction: dynamically quantized input of the down
projection): the kernel's BF16 h within one BF16 step of the exactly rounded
FP64 silu(gate) * up, and its codes and scales bit-exact with the oracle's
group-128 quantization of that same h.
"""
import numpy as np
import pytest
import torch

import fp8_block_scaled_09_b200 as fp8bq
import oracle
import workloads
from gpu_util import Guarded

pytestmark = pytest.mark.gpu

HIDDEN, KV = 7168, 1024


@pytest.fixture(scope="module", autouse=True)
def _device():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    fp8bq.lib()
    yield
    assert fp8bq.last_device_status() == 0


def _qkv(T, seed, big=False, specials=False):
    rng = np.random.default_rng(seed)
    y = rng.standard_normal((T, HIDDEN + 2 * KV)).astype(np.float32) * 3
    if big:
        y[:, ::17] *= 300            # beyond 448: saturation
    if specials and T > 0:
        flat = y.reshape(-1)
        idx = rng.choice(flat.size, size=min(64, flat.size), replace=False)
        flat[idx[:16]] = np.nan
        flat[idx[16:32]] = np.inf
        flat[idx[32:48]] = -np.inf
        flat[idx[48:]] = 2.0 ** -133   # BF16 subnormal
    return torch.from_numpy(y).to(torch.bfloat16)


def _same_codes(got, ref):
    nan_g = (got & 0x7F) == 0x7F
    nan_r = (ref & 0x7F) == 0x7F
    assert np.array_equal(nan_g, nan_r)
    bad = np.nonzero((got != ref) & ~nan_r)
    assert bad[0].size == 0, (bad[0][:5], got[bad][:5], ref[bad][:5])


@pytest.mark.parametrize("T,slots,big,specials", [(1, 4, False, False), (7, 64, True, True),
                                                   (128, 300, True, False), (2048, 2048, True, True)])
def test_kv_write_matches_oracle(T, slots, big, specials):
    qkv = _qkv(T, 40 + T, big, specials)
    rng = np.random.default_rng(T)
    loc = rng.permutation(slots)[:T].astype(np.int64)
    slot_bytes = KV + 16 * (T % 3)           # padded slots on some cases
    kc_ref = np.full((slots, slot_bytes), 0xA5, np.uint8)
    vc_ref = np.full((slots, slot_bytes), 0x5A, np.uint8)
    assert oracle.kv_write(qkv[:, HIDDEN:HIDDEN + KV], qkv[:, HIDDEN + KV:], loc, kc_ref, vc_ref) == 0
    d = qkv.cuda()
    kc = Guarded((slots, slot_bytes), torch.uint8, fill=0xA5)
    vc = Guarded((slots, slot_bytes), torch.uint8, fill=0x5A)
    fp8bq.kv_write_e4m3(d[:, HIDDEN:HIDDEN + KV], d[:, HIDDEN + KV:], torch.from_numpy(loc).cuda(),
                        kc.t, vc.t)
    torch.cuda.synchronize()
    assert kc.guards_intact() and vc.guards_intact()
    _same_codes(kc.t.cpu().numpy(), kc_ref)
    _same_codes(vc.t.cpu().numpy(), vc_ref)


def test_kv_write_long_prefill_rows():
    # the long-prefill token count: 32768 rows of K and V (134 MB of BF16 read)
    T = 32768
    qkv = _qkv(T, 7, big=True)
    loc = np.arange(T, dtype=np.int64)[::-1].copy()
    kc_ref = np.zeros((T, KV), np.uint8)
    vc_ref = np.zeros((T, KV), np.uint8)
    oracle.kv_write(qkv[:, HIDDEN:HIDDEN + KV], qkv[:, HIDDEN + KV:], loc, kc_ref, vc_ref)
    d = qkv.cuda()
    kc = torch.zeros((T, KV), dtype=torch.uint8, device="cuda")
    vc = torch.zeros((T, KV), dtype=torch.uint8, device="cuda")
    fp8bq.kv_write_e4m3(d[:, HIDDEN:HIDDEN + KV], d[:, HIDDEN + KV:], torch.from_numpy(loc).cuda(),
                        kc, vc)
    torch.cuda.synchronize()
    assert np.array_equal(kc.cpu().numpy(), kc_ref) and np.array_equal(vc.cpu().numpy(), vc_ref)


def test_kv_write_out_of_range_slots_are_skipped_and_reported():
    T, slots = 6, 10
    qkv = _qkv(T, 3)
    loc = np.array([2, -1, 9, 10, 0, 1 << 40], dtype=np.int64)
    kc_ref = np.full((slots, KV), 0x11, np.uint8)
    vc_ref = np.full((slots, KV), 0x22, np.uint8)
    assert oracle.kv_write(qkv[:, HIDDEN:HIDDEN + KV], qkv[:, HIDDEN + KV:], loc, kc_ref, vc_ref) == 3
    d = qkv.cuda()
    kc = torch.full((slots, KV), 0x11, dtype=torch.uint8, device="cuda")
    vc = torch.full((slots, KV), 0x22, dtype=torch.uint8, device="cuda")
    assert fp8bq.last_device_status() == 0
    fp8bq.kv_write_e4m3(d[:, HIDDEN:HIDDEN + KV], d[:, HIDDEN + KV:], torch.from_numpy(loc).cuda(),
                        kc, vc)
    torch.cuda.synchronize()
    assert fp8bq.last_device_status() == 8          # FP8BQ_ERR_INDEX, and the read clears it
    assert fp8bq.last_device_status() == 0
    assert np.array_equal(kc.cpu().numpy(), kc_ref) and np.array_equal(vc.cpu().numpy(), vc_ref)


def test_kv_write_empty_is_noop():
    k = torch.zeros((0, KV), dtype=torch.bfloat16, device="cuda")
    kc = torch.zeros((4, KV), dtype=torch.uint8, device="cuda")
    fp8bq.kv_write_e4m3(k, k, torch.zeros(0, dtype=torch.int64, device="cuda"), kc, kc.clone())


# ---------------------------------------------------------------- SiLU-mul + quantize

def _bf16_bits(t):
    return t.contiguous().cpu().view(torch.int16).numpy().view(np.uint16)


def _within_one_bf16_step(got_bits, exact):
    """got (BF16 bits) is the BF16 rounding of exact or one of its neighbours."""
    ref_bits = oracle.bf16_round(exact)
    g = got_bits.astype(np.int32)
    r = ref_bits.astype(np.int32)
    gs, rs = g >> 15, r >> 15
    gm, rm = g & 0x7FFF, r & 0x7FFF
    same = g == r
    neighbour = (gs == rs) & (np.abs(gm - rm) <= 1)
    zeros = (gm == 0) & (rm <= 1) | (rm == 0) & (gm <= 1)
    return same, same | neighbour | zeros


# (700, 5248): 41 groups per row (not a multiple of 4).  (2000, 5120): large
# enough for the 8-lane-team kernel, 40 groups per row so the second 32-group
# chunk of a row is ragged (some warps of its CTA have no group), and more rows
# than the grid's row count
@pytest.mark.parametrize("M,I,scale", [(1, 128, 1.0), (3, 384, 4.0), (130, 8192, 2.0),
                                        (17, 1024, 30.0), (700, 5248, 1.0), (2000, 5120, 1.0)])
def test_silu_mul_quantize_matches_oracle(M, I, scale):
    rng = np.random.default_rng(M * 7 + I)
    gu = torch.from_numpy(rng.standard_normal((M, 2 * I)).astype(np.float32) * scale).to(torch.bfloat16)
    gu[:, :128] = 0.0                                 # an all-zero gate group: h = 0, scale 1
    d = gu.cuda()
    h = Guarded((M, I), torch.bfloat16)
    q = Guarded((M, I), torch.uint8)
    s = Guarded((M, I // 128), torch.float32)
    fp8bq.silu_mul_quantize(d, q.t, s.t, h.t)
    torch.cuda.synchronize()
    assert h.guards_intact() and q.guards_intact() and s.guards_intact()
    h_bits = _bf16_bits(h.t)
    exact = oracle.silu_mul(gu)
    same, ok = _within_one_bf16_step(h_bits, exact)
    assert ok.all(), np.nonzero(~ok)[0][:5]
    assert same.mean() > 0.995
    # codes and scales: exactly the quantization of the kernel's own BF16 h
    rq, rs = oracle.quantize_act(h.t.cpu())
    assert np.array_equal(s.t.cpu().numpy().view(np.uint32), rs.view(np.uint32))
    assert np.array_equal(q.t.cpu().numpy(), rq)
    assert np.all(s.t.cpu().numpy()[:, 0] == 1.0)
    # without h requested the codes are the same
    q2, s2 = fp8bq.silu_mul_quantize(d)
    assert torch.equal(q2, q.t) and torch.equal(s2, s.t)


def test_silu_mul_quantize_drafter_mlp_shape():
    # the drafter MLP: gate/up output [4096, 16384] -> down-projection input [4096, 8192]
    g = workloads.DRAFTER_GATE_UP
    M, I = g.M, g.N // 2
    rng = np.random.default_rng(11)
    gu = torch.from_numpy(rng.standard_normal((M, 2 * I)).astype(np.float32) * 2).to(torch.bfloat16)
    d = gu.cuda()
    h = torch.empty((M, I), dtype=torch.bfloat16, device="cuda")
    q, s = fp8bq.silu_mul_quantize(d, h=h)
    torch.cuda.synchronize()
    same, ok = _within_one_bf16_step(_bf16_bits(h), oracle.silu_mul(gu))
    assert ok.all() and same.mean() > 0.995
    rq, rs = oracle.quantize_act(h.cpu())
    assert np.array_equal(q.cpu().numpy(), rq)
    assert np.array_equal(s.cpu().numpy().view(np.uint32), rs.view(np.uint32))


def test_silu_mul_quantize_feeds_the_down_gemm():
    # silu_mul_quantize -> gemm equals quantize_act(h) -> gemm bit for bit
    M, I, N = 9, 1024, 256
    rng = np.random.default_rng(2)
    gu = torch.from_numpy(rng.standard_normal((M, 2 * I)).astype(np.float32)).to(torch.bfloat16).cuda()
    w = workloads.weight(N, I, 5).cuda()
    qw, sw = fp8bq.quantize_weight(w)
    h = torch.empty((M, I), dtype=torch.bfloat16, device="cuda")
    q, s = fp8bq.silu_mul_quantize(gu, h=h)
    y1 = fp8bq.gemm(q, s, qw, sw)
    y2 = fp8bq.linear(h, qw, sw)
    torch.cuda.synchronize()
    assert torch.equal(y1.view(torch.int16), y2.view(torch.int16))
