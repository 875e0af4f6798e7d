"""Pins for the oracle's NVFP4 weight-only (A16) functions (CPU only).

Page "ProCreations/Nanbeige4.3-33B-NVFP4-A16", recipe paragraph: FP4 E2M1
weights in groups of 16 with E4M3 block scales and a global weight scale,
activations in BF16.

* E2M1 decode against the format's structure (sign-magnitude, 2-bit exponent
  with bias 1, 1-bit mantissa, subnormals at exponent 0): monotone, smallest
  step 0.5, largest value 6, each binade twice the step of the one below.
* E2M1 encode against a vectorised nearest-value search (ties to the even
  mantissa) over a dense grid of binary32 values of both signs.
* The min-max quantizer against an independent numpy/torch implementation
  (E4M3 through torch's cast after clamping) and its invariants.
* The GEMM reference against exact rational sums.
"""
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle


def test_e2m1_decode_structure():
    vals = [oracle.e2m1_decode(c) for c in range(16)]
    pos = vals[:8]
    assert pos[0] == 0.0 and pos[1] == 0.5 and pos[7] == 6.0
    assert all(b > a for a, b in zip(pos, pos[1:]))
    steps = np.diff(pos)
    assert list(steps) == [0.5, 0.5, 0.5, 0.5, 1.0, 1.0, 2.0]   # subnormal + 3 binades
    for c in range(8):
        assert vals[8 + c] == -pos[c] and np.signbit(vals[8 + c])


def _nearest_e2m1(y):
    mags = np.array([oracle.e2m1_decode(c) for c in range(8)])
    a = np.minimum(np.abs(y), 6.0)
    d = np.abs(a[:, None] - mags[None, :])
    best = d.min(axis=1, keepdims=True)
    cand = np.where(d == best, np.arange(8)[None, :], 99)
    # among equally near codes prefer the even mantissa (code bit 0 clear)
    even = np.where((cand % 2 == 0) & (cand != 99), cand, 99).min(axis=1)
    any_ = cand.min(axis=1)
    code = np.where(even != 99, even, any_)
    return (code | np.where(np.signbit(y), 8, 0)).astype(np.uint8)


def test_e2m1_encode_matches_nearest_search():
    rng = np.random.default_rng(0)
    ys = np.concatenate([
        np.arange(-8.0, 8.0, 1 / 64),                      # dense grid incl. every midpoint
        rng.standard_normal(20000) * 3,
        np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, -0.25, 6.0, 6.5, 1e30, -1e30, 1e-30]),
    ]).astype(np.float32)
    got = np.array([oracle.e2m1_encode(float(y)) for y in ys], dtype=np.uint8)
    assert np.array_equal(got, _nearest_e2m1(ys.astype(np.float64)))


def _numpy_minmax_nvfp4(w):
    """Independent restatement of the min-max recipe with numpy float32 ops and
    torch's E4M3 cast; returns packed, block scales and g."""
    x = w.float().numpy().astype(np.float32)
    N, K = x.shape
    amax = np.float32(np.abs(x).max())
    g = np.float32(1.0) if amax == 0 else np.float32(amax / np.float32(2688.0))
    six_g = np.float32(np.float32(6.0) * g)
    blocks = np.abs(x).reshape(N, K // 16, 16).max(axis=2).astype(np.float32)
    t = (blocks / six_g).astype(np.float32)
    sb = torch.clamp(torch.from_numpy(t), -448, 448).to(torch.float8_e4m3fn)
    sb_val = sb.float().numpy().astype(np.float32)
    sig = (sb_val * g).astype(np.float32)
    q = np.zeros((N, K), np.uint8)
    sig_full = np.repeat(sig, 16, axis=1)
    nz = sig_full != 0
    quot = np.zeros((N, K), np.float32)
    quot[nz] = (x[nz] / sig_full[nz]).astype(np.float32)
    q[nz] = _nearest_e2m1(quot[nz].astype(np.float64))
    packed = (q[:, 0::2] | (q[:, 1::2] << 4)).astype(np.uint8)
    return packed, sb.view(torch.uint8).numpy(), float(g)


@pytest.mark.parametrize("N,K,seed", [(128, 256, 1), (256, 1024, 2)])
def test_nvfp4_quantize_matches_independent_restatement(N, K, seed):
    rng = np.random.default_rng(seed)
    w = torch.from_numpy(rng.standard_normal((N, K)).astype(np.float32) * 0.02)
    w[0, 5] = 0.9                          # one large weight sets g
    w[3, 32:48] = 0.0                      # an all-zero group
    w = w.to(torch.bfloat16)
    packed, sb, g = oracle.nvfp4_quantize(w)
    rp, rsb, rg = _numpy_minmax_nvfp4(w)
    assert g == rg
    assert np.array_equal(sb, rsb)
    assert np.array_equal(packed, rp)


def test_nvfp4_quantize_invariants():
    rng = np.random.default_rng(3)
    w = torch.from_numpy(rng.standard_normal((128, 512)).astype(np.float32)).to(torch.bfloat16)
    packed, sb, g = oracle.nvfp4_quantize(w)
    x = w.float().numpy()
    amax = np.abs(x).max()
    assert g == pytest.approx(amax / 2688, rel=1e-7)
    n, k = np.unravel_index(np.argmax(np.abs(x)), x.shape)
    # the tensor's largest weight: block scale 448 and code +-6
    assert sb[n, k // 16] == 0x7E
    q = (packed[n, k // 2] >> (4 * (k % 2))) & 0xF
    assert q & 0x7 == 0x7 and bool(q & 0x8) == bool(x[n, k] < 0)
    # element order in a byte: element 2j low nibble, 2j+1 high nibble
    w2 = torch.zeros((128, 32), dtype=torch.bfloat16)
    w2[0, 0] = 6.0
    w2[1, 1] = 6.0
    p2, s2, g2 = oracle.nvfp4_quantize(w2)
    assert p2[0, 0] == 0x07 and p2[1, 0] == 0x70
    assert np.all(p2[2:] == 0) and np.all(s2[2:] == 0)      # all-zero groups: scale 0, codes 0
    # dequantized values stay within half an E2M1 step of the scaled weight
    vals = np.array([oracle.e2m1_decode(c) for c in range(16)])
    codes = np.stack([packed & 0xF, packed >> 4], axis=2).reshape(128, 512)
    sbv = torch.from_numpy(sb).view(torch.float8_e4m3fn).float().numpy().astype(np.float64)
    deq = vals[codes] * np.repeat(sbv, 16, axis=1) * g
    sig = np.repeat(sbv, 16, axis=1) * g
    step = np.where(np.abs(x) / sig >= 4, 2.0, np.where(np.abs(x) / sig >= 2, 1.0, 0.5))
    assert np.all(np.abs(deq - x) <= 0.5 * step * sig * (1 + 1e-6))


def test_nvfp4_gemm_ref_exact_sums():
    rng = np.random.default_rng(4)
    M, N, K = 3, 128, 64
    x = torch.from_numpy(rng.integers(-8, 9, (M, K)).astype(np.float32) / 4).to(torch.bfloat16)
    packed = rng.integers(0, 256, (N, K // 2)).astype(np.uint8)
    sb = rng.choice(np.array([0x30, 0x38, 0x40, 0x44, 0x2C], np.uint8), size=(N, K // 16))
    g = 0.375
    y = oracle.nvfp4_gemm_ref(x, packed, sb, g)
    vals = [Fraction(oracle.e2m1_decode(c)) for c in range(16)]
    sbv = {c: Fraction(float(torch.tensor([c], dtype=torch.uint8).view(torch.float8_e4m3fn).float()))
           for c in np.unique(sb)}
    xf = [[Fraction(float(v)) for v in row] for row in x.float().numpy()]
    for m in range(M):
        for n in (0, 1, 77, 127):
            acc = Fraction(0)
            for k in range(K):
                q = (int(packed[n, k // 2]) >> (4 * (k % 2))) & 0xF
                acc += xf[m][k] * vals[q] * sbv[sb[n, k // 16]] * Fraction(g)
            assert y[m, n] == float(acc)
    rows = np.array([2, 0])
    assert np.array_equal(oracle.nvfp4_gemm_ref(x, packed, sb, g, rows=rows), y[rows])
