"""GPU parity of the quantizers: E4M3 codes and FP32 scales bit-exact with the
oracle (page "ProCreations/Nanbeige4.3-33B-FP8", introduction and "Recipe and
calibration"), on seeded workloads, edge cases and the full long-prefill
activation [32768, 7168]; guard bands around every output stay intact."""
import numpy as np
import pytest
import torch

import fp8_block_scaled_09_b200 as fp8bq
import oracle
import workloads
from gpu_util import Guarded

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _device():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    fp8bq.lib()
    yield
    assert fp8bq.last_device_status() == 0


def gpu_quantize_act(x: torch.Tensor):
    M, K = x.shape
    q = Guarded((M, K), torch.uint8)
    s = Guarded((M, K // 128), torch.float32)
    fp8bq.quantize_act(x.cuda(), q.t, s.t)
    torch.cuda.synchronize()
    assert q.guards_intact() and s.guards_intact()
    return q.t.cpu().numpy(), s.t.cpu().numpy()


def gpu_quantize_weight(w: torch.Tensor):
    N, K = w.shape
    q = Guarded((N, K), torch.uint8)
    s = Guarded((N // 128, K // 128), torch.float32)
    fp8bq.quantize_weight(w.cuda(), q.t, s.t)
    torch.cuda.synchronize()
    assert q.guards_intact() and s.guards_intact()
    return q.t.cpu().numpy(), s.t.cpu().numpy()


def assert_same(got, ref):
    gq, gs = got
    rq, rs = ref
    assert gs.shape == rs.shape and gq.shape == rq.shape
    bad_s = np.nonzero(gs.view(np.uint32) != rs.view(np.uint32))
    assert bad_s[0].size == 0, (bad_s[0][:5], gs[bad_s][:5], rs[bad_s][:5])
    bad_q = np.nonzero(gq != rq)
    assert bad_q[0].size == 0, (len(bad_q[0]), [b[:5] for b in bad_q], gq[bad_q][:5], rq[bad_q][:5])


def _bf16(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16)


ACT_CASES = {
    "m1_k128": lambda: workloads.activation(1, 128, 1),
    "m3_k384_outliers": lambda: workloads.activation(3, 384, 2, outliers=5),
    "kproj_m16_zero_row": lambda: workloads.KPROJ_M16.make_x(),
    "ragged_m1001": lambda: workloads.activation(1001, 1024, 3, outliers=4),
    "t3_heavy_tail": lambda: workloads.activation(257, 7168, 4, t3_channels=72),
    "gated_product": lambda: workloads.gated_activation(130, 8192, 5),
    "subnormal": lambda: _bf16(np.random.default_rng(6).standard_normal((9, 640)) * 1e-39),
    "huge": lambda: _bf16(np.random.default_rng(7).standard_normal((5, 256)) * 1e37),
    "signed_zeros": lambda: _bf16(np.where(np.arange(512) % 3 == 0, -0.0, 0.0)[None, :].repeat(2, 0)),
    "every_bf16_binade": lambda: _bf16(np.stack([np.ldexp(1 + np.arange(128) / 128, e)
                                                 for e in range(-133, 127, 3)])),
    "ties_power_of_two_amax": lambda: _bf16(np.concatenate(
        [np.full((4, 1), 448.0), np.tile(np.arange(127) * 3.5 + 0.25, (4, 1))], axis=1)),
}


@pytest.mark.parametrize("case", sorted(ACT_CASES))
def test_quantize_act_bit_exact(case):
    x = ACT_CASES[case]()
    assert_same(gpu_quantize_act(x), oracle.quantize_act(x))


def test_quantize_act_full_long_prefill():
    # the whole [32768, 7168] activation of the long-prefill workload
    x = workloads.LONG_O_PROJ.make_x()
    assert_same(gpu_quantize_act(x), oracle.quantize_act(x))


def test_quantize_act_decode_set_and_prefill_qkv():
    for g in workloads.DECODE_SET + (workloads.PREFILL_QKV,):
        x = g.make_x()
        assert_same(gpu_quantize_act(x), oracle.quantize_act(x))


def test_quantize_act_empty_is_noop():
    x = torch.zeros((0, 256), dtype=torch.bfloat16, device="cuda")
    q, s = fp8bq.quantize_act(x)
    assert q.shape == (0, 256) and s.shape == (0, 2)


WEIGHT_CASES = {
    "one_block": lambda: workloads.weight(128, 128, 10),
    "ragged_3x5": lambda: workloads.weight(384, 640, 11),
    "identity": lambda: _bf16(np.eye(256)),
    "kproj_full": lambda: workloads.KPROJ_M16.make_w(),
    "zero_block": lambda: _bf16(np.where(np.arange(256)[:, None] < 128, 0.0,
                                         np.random.default_rng(1).standard_normal((256, 384)))),
}


@pytest.mark.parametrize("case", sorted(WEIGHT_CASES))
def test_quantize_weight_bit_exact(case):
    w = WEIGHT_CASES[case]()
    assert_same(gpu_quantize_weight(w), oracle.quantize_weight(w))


@pytest.mark.parametrize("name", ["qkv_m1", "o_proj_m1", "gate_up", "fc"])
def test_quantize_weight_full_shapes(name):
    w = workloads.by_name(name).make_w()
    assert_same(gpu_quantize_weight(w), oracle.quantize_weight(w))


def _near_tie_groups(n_scales=64, seed=3):
    """Groups whose quotients x / s land within a few binary32 ulps of an E4M3
    rounding midpoint (the quantizer's slowest and most fragile case)."""
    rng = np.random.default_rng(seed)
    all_bf16 = np.arange(0, 0x7F80, dtype=np.uint32)               # every finite positive BF16
    xs = (all_bf16 << 16).view(np.float32)
    rows = []
    for _ in range(n_scales):
        amax = np.float32(xs[rng.integers(0x3C00, 0x4700)])         # amax between ~2^-7 and ~2^15
        s = np.float32(amax / np.float32(448.0))
        cand = xs[xs <= amax]
        t = (cand / s).astype(np.float32)
        low = t.view(np.uint32) & 0xFFFFF
        near = cand[(np.abs(low.astype(np.int64) - 0x80000) <= 12) & (t >= 2.0 ** -6)]
        if near.size == 0:
            continue
        sign = np.where(rng.integers(0, 2, near.size) == 1, -1.0, 1.0).astype(np.float32)
        vals = np.resize(near * sign, 127)
        rows.append(np.concatenate([[amax], vals]).astype(np.float32))
    assert len(rows) >= 16, "too few near-tie groups generated"
    return _bf16(np.stack(rows))


def test_quantize_act_near_e4m3_ties_bit_exact():
    x = _near_tie_groups()
    assert_same(gpu_quantize_act(x), oracle.quantize_act(x))
