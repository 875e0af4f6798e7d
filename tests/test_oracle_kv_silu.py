"""Pins for the oracle's FP8 KV-cache write and SiLU-gated product (CPU only).

KV write (page "ProCreations/Nanbeige4.3-33B-FP8", "Serving" and "Speed on
Vega": fp8_e4m3 KV cache with unit scales): every BF16 bit pattern is checked
against a library routine (PyTorch's float8_e4m3fn cast after clamping to
+-448, since that cast does not saturate), the slot scatter against a plain
permutation, and exactly representable values against the identity.

SiLU product (the MLP input of the down projection): closed forms at 0, 1 and
large |gate|, and agreement with scipy's logistic function on random inputs.
"""
import numpy as np
import pytest
import scipy.special
import torch

import oracle


def _all_bf16_rows(width=256):
    bits = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    return bits.reshape(-1, width)


def test_kv_code_of_every_bf16_pattern():
    k = _all_bf16_rows()
    v = k[::-1].copy()
    T, W = k.shape
    kc = np.zeros((T, W), np.uint8)
    vc = np.zeros((T, W), np.uint8)
    assert oracle.kv_write(k, v, np.arange(T), kc, vc) == 0
    for src, got in ((k, kc), (v, vc)):
        x = torch.from_numpy(src.view(np.int16).copy()).view(torch.bfloat16).float()
        finite = torch.isfinite(x).numpy()
        ref = torch.clamp(x, -448.0, 448.0).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
        assert np.array_equal(got[finite], ref[finite])
        nan = torch.isnan(x).numpy()
        assert np.all((got[nan] & 0x7F) == 0x7F)
        xf = x.numpy()
        assert np.all(got[np.isposinf(xf)] == 0x7E) and np.all(got[np.isneginf(xf)] == 0xFE)


def test_kv_exactly_representable_values_round_trip():
    codes = np.array([c for c in range(256) if (c & 0x7F) != 0x7F], dtype=np.uint8)
    vals = oracle.e4m3_decode(codes)                   # exact E4M3 values, all BF16-exact
    x = torch.tensor(vals, dtype=torch.float32).to(torch.bfloat16)
    assert np.array_equal(x.float().numpy(), vals.astype(np.float32))
    W = 64
    rows = -(-len(codes) // W)
    k = torch.zeros(rows * W, dtype=torch.bfloat16)
    k[:len(codes)] = x
    k = k.view(rows, W)
    kc = np.zeros((rows, W), np.uint8)
    vc = np.zeros((rows, W), np.uint8)
    oracle.kv_write(k, k, np.arange(rows), kc, vc)
    got = kc.reshape(-1)[:len(codes)]
    # +-0 keep their sign; every other value maps back to its own code
    assert np.array_equal(got, codes)


def test_kv_scatter_strided_rows_into_slots():
    rng = np.random.default_rng(5)
    T, W, slots = 37, 128, 100
    # a fused [T, q | k | v] activation: K and V are column slices with row stride 3W
    qkv = torch.randn(T, 3 * W).mul(100).to(torch.bfloat16)
    base = qkv.view(torch.int16).numpy().view(np.uint16)
    k, v = base[:, W:2 * W], base[:, 2 * W:]
    assert k.strides[0] == 3 * W * 2
    loc = rng.permutation(slots)[:T].astype(np.int64)
    loc[5], loc[11] = -1, slots                      # two rows point outside the cache
    sentinel = 0x5A
    kc = np.full((slots, W), sentinel, np.uint8)
    vc = np.full((slots, W), sentinel, np.uint8)
    assert oracle.kv_write(k, v, loc, kc, vc) == 2
    ref_k = torch.clamp(qkv[:, W:2 * W].float(), -448, 448).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    ref_v = torch.clamp(qkv[:, 2 * W:].float(), -448, 448).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    written = set()
    for t in range(T):
        if 0 <= loc[t] < slots:
            assert np.array_equal(kc[loc[t]], ref_k[t]) and np.array_equal(vc[loc[t]], ref_v[t])
            written.add(int(loc[t]))
    untouched = [s for s in range(slots) if s not in written]
    assert np.all(kc[untouched] == sentinel) and np.all(vc[untouched] == sentinel)


def test_kv_slot_wider_than_row_leaves_padding():
    k = torch.ones(2, 64, dtype=torch.bfloat16)
    kc = np.full((2, 80), 7, np.uint8)
    vc = np.full((2, 80), 7, np.uint8)
    oracle.kv_write(k, k, np.array([1, 0]), kc, vc)
    assert np.all(kc[:, :64] == 0x38) and np.all(kc[:, 64:] == 7)


def _gu(gate, up):
    return torch.cat([torch.as_tensor(gate, dtype=torch.float32),
                      torch.as_tensor(up, dtype=torch.float32)], dim=1).to(torch.bfloat16)


def test_silu_mul_closed_forms():
    gate = np.array([[0.0, 1.0, -1.0, 40.0, -40.0, 2.0]])
    up = np.array([[3.0, 2.0, 2.0, 0.5, 1.0, -1.0]])
    h = oracle.silu_mul(_gu(gate, up))[0]
    e = np.e
    assert h[0] == 0.0
    assert h[1] == pytest.approx(2.0 * e / (1.0 + e), rel=1e-15)
    assert h[2] == pytest.approx(-2.0 / (1.0 + e), rel=1e-15)
    assert h[3] == pytest.approx(20.0, rel=1e-15)           # silu(40) = 40 (1 - 4e-18)
    assert abs(h[4]) < 1e-15                                   # silu(-40) ~ -1.7e-16
    assert h[5] == pytest.approx(-2.0 / (1.0 + np.exp(-2.0)), rel=1e-15)


def test_silu_mul_gate_is_the_first_half():
    gu = _gu([[1.0, -3.0]], [[5.0, 0.25]])
    h = oracle.silu_mul(gu)[0]
    swapped = oracle.silu_mul(_gu([[5.0, 0.25]], [[1.0, -3.0]]))[0]
    assert h[0] == pytest.approx(1.0 / (1 + np.exp(-1.0)) * 5.0, rel=1e-15)
    assert not np.allclose(h, swapped)


def test_silu_mul_matches_scipy_logistic():
    rng = np.random.default_rng(8)
    M, I = 7, 384
    gu = torch.from_numpy(rng.standard_normal((M, 2 * I)).astype(np.float32) * 4).to(torch.bfloat16)
    g = gu[:, :I].double().numpy()
    u = gu[:, I:].double().numpy()
    ref = g * scipy.special.expit(g) * u
    h = oracle.silu_mul(gu)
    np.testing.assert_allclose(h, ref, rtol=1e-13, atol=1e-300)
