"""Exhaustive check of the quantizers' quotient on the GPU.

Every E4M3 code is the saturating round-to-nearest conversion of the binary32
quotient fl32(x / scale), scale = fl32(amax / 448) (page
"ProCreations/Nanbeige4.3-33B-FP8", introduction: dynamic per-token/group-128
activation scales).  The kernels form that quotient from one reciprocal and an
FMA correction instead of a division (except for tiny scales), so this test
runs fp8bq.quantize_act over every pair of a positive finite BF16 amax and a
BF16 x with |x| <= amax, both signs: about 1.07e9 elements, each group holding
its amax in channel 0.  Codes and scales must equal, bit for bit, torch's IEEE
binary32 division followed by its clamp-and-round cast to float8_e4m3fn (the
cast the oracle's encoder is pinned against).  The oracle's own comparison on
sampled groups of the same tensor closes the loop.
"""
import numpy as np
import pytest
import torch

import fp8_block_scaled_09_b200 as fp8bq
import oracle

pytestmark = pytest.mark.gpu

K = 7168                 # 56 groups per row
GROUPS_PER_ROW = K // 128
PER_GROUP = 127          # x values per group (channel 0 holds the amax)


@pytest.fixture(scope="module", autouse=True)
def _device():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    fp8bq.lib()
    yield
    assert fp8bq.last_device_status() == 0


def _groups(a_lo: int, a_hi: int, dev) -> torch.Tensor:
    """BF16 bit patterns [G, 128] (int32) of the groups for amax magnitudes
    a_lo <= a < a_hi: channel 0 = +a, channels 1..127 walk through every
    magnitude 0..a with both signs (zero-padded at the end of each amax)."""
    a = torch.arange(a_lo, a_hi, device=dev, dtype=torch.int64)
    n_x = 2 * (a + 1)                                    # magnitudes 0..a, two signs
    n_g = (n_x + PER_GROUP - 1) // PER_GROUP
    ga = torch.repeat_interleave(a, n_g)
    first = torch.cumsum(n_g, 0) - n_g
    k = torch.arange(ga.numel(), device=dev) - torch.repeat_interleave(first, n_g)
    t = k[:, None] * PER_GROUP + torch.arange(PER_GROUP, device=dev)[None, :]
    valid = t < 2 * (ga[:, None] + 1)
    bits = torch.where(valid, ((t & 1) << 15) | (t >> 1), torch.zeros_like(t))
    return torch.cat([ga[:, None], bits], dim=1).to(torch.int32)


def _as_bf16_rows(bits: torch.Tensor) -> torch.Tensor:
    G = bits.shape[0]
    pad = (-G) % GROUPS_PER_ROW                          # all-zero groups (scale 1)
    if pad:
        bits = torch.cat([bits, torch.zeros((pad, 128), dtype=bits.dtype, device=bits.device)])
    return bits.to(torch.int16).view(torch.bfloat16).reshape(-1, K)


def _reference(x: torch.Tensor):
    xf = x.float().reshape(-1, 128)
    amax = xf.abs().amax(dim=1)
    # a tensor divisor: torch turns division by a Python scalar into a
    # multiplication by its reciprocal, which is not the IEEE quotient
    s = torch.where(amax == 0, torch.ones_like(amax), amax / torch.full_like(amax, 448.0))
    q = (xf / s[:, None]).clamp(-448.0, 448.0).to(torch.float8_e4m3fn)
    return q.view(torch.uint8).reshape(x.shape), s.reshape(x.shape[0], -1)


def test_quotient_codes_over_every_bf16_amax_and_x():
    dev = torch.device("cuda")
    a_max = 0x7F7F                                       # largest finite BF16 magnitude
    # chunk boundaries so each chunk holds about 1e6 groups (sum of 2(a+1)/127)
    bounds = [1]
    while bounds[-1] <= a_max:
        a0 = bounds[-1]
        a1 = int(np.sqrt(a0 * a0 + 127e6)) + 1
        bounds.append(min(a1, a_max + 1))
    checked = 0
    sampled_oracle = 0
    for a0, a1 in zip(bounds[:-1], bounds[1:]):
        x = _as_bf16_rows(_groups(a0, a1, dev))
        q, s = fp8bq.quantize_act(x)
        qr, sr = _reference(x)
        torch.cuda.synchronize()
        bad_s = (s.view(torch.int32) != sr.view(torch.int32)).nonzero()
        assert bad_s.numel() == 0, f"amax [{a0}, {a1}): scales differ at {bad_s[:4].tolist()}"
        bad_q = (q != qr).nonzero()
        if bad_q.numel():
            r, c = bad_q[0].tolist()
            raise AssertionError(
                f"amax [{a0}, {a1}): {bad_q.shape[0]} codes differ; first at row {r} col {c}: "
                f"x bits {int(x[r, c].view(torch.int16)) & 0xFFFF:#06x}, scale {float(s[r, c // 128])!r}, "
                f"code {int(q[r, c]):#04x} vs {int(qr[r, c]):#04x}")
        checked += x.numel()
        # the oracle on a few rows of each chunk (first, middle, last)
        rows = np.unique(np.array([0, x.shape[0] // 2, x.shape[0] - 1], dtype=np.int64))
        xh = x[torch.from_numpy(rows).to(dev)].cpu()
        oq, os_ = oracle.quantize_act(xh)
        assert np.array_equal(oq, q[torch.from_numpy(rows).to(dev)].cpu().numpy())
        assert np.array_equal(os_.view(np.uint32),
                              s[torch.from_numpy(rows).to(dev)].cpu().numpy().view(np.uint32))
        sampled_oracle += xh.numel()
        del x, q, s, qr, sr
    # every (amax, x) pair: sum over a of 2 (a + 1) x values, plus the amax channels
    assert checked >= sum(2 * (a + 1) for a in range(1, a_max + 1))
    assert sampled_oracle > 0
