"""Exact (rational) arithmetic and library-routine helpers used to pin the oracle.

Nothing here calls the oracle or the CUDA library.  E4M3 values are decoded
through torch's float8_e4m3fn dtype (a library routine), and sums are formed
exactly with Python integers, so these helpers are independent of both sides.
"""
from __future__ import annotations

from fractions import Fraction

import numpy as np
import torch

GROUP = 128


def torch_e4m3_values() -> np.ndarray:
    """FP64 value of each of the 256 E4M3 codes, decoded by torch."""
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    return codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()


E4M3 = torch_e4m3_values()


def dq(codes: np.ndarray) -> np.ndarray:
    return E4M3[np.asarray(codes, dtype=np.uint8)]


def torch_encode(y: np.ndarray) -> np.ndarray:
    """Saturating E4M3 encoding through torch: clamp to +-448, then the RNE cast."""
    t = torch.from_numpy(np.ascontiguousarray(y, dtype=np.float32))
    return t.clamp(-448.0, 448.0).to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def tolerance_ok(y, ref) -> np.ndarray:
    """|y - ref| <= 1e-2 |ref| + 2e-3 rms(ref), elementwise; rms over the given output."""
    ref = np.asarray(ref, dtype=np.float64)
    rms = float(np.sqrt(np.mean(ref * ref))) if ref.size else 0.0
    return np.abs(np.asarray(y, dtype=np.float64) - ref) <= 1e-2 * np.abs(ref) + 2e-3 * rms


def _to_scaled_ints(v: np.ndarray):
    """Exact integers I and shift P with v == I / 2^P (v: finite dyadic doubles)."""
    flat = np.asarray(v, dtype=np.float64).reshape(-1)
    ratios = [float(t).as_integer_ratio() for t in flat]
    P = max(den.bit_length() - 1 for _, den in ratios) if ratios else 0
    ints = np.array([num << (P - (den.bit_length() - 1)) for num, den in ratios], dtype=object)
    return ints.reshape(np.shape(v)), P


def exact_gemm(qa, sa, qw, sw) -> tuple[np.ndarray, np.ndarray]:
    """Exact value of sum_k (dq(qa) sa[m, k/128]) (dq(qw) sw[n/128, k/128]).

    Returns (exact values as Fraction object array [M, N], sum of |terms| as
    float64 [M, N]) -- the latter bounds the rounding error of any FP64
    recursive summation of the same terms.
    """
    qa = np.asarray(qa)
    qw = np.asarray(qw)
    M, K = qa.shape
    N = qw.shape[0]
    a = dq(qa) * np.repeat(np.asarray(sa, np.float64), GROUP, axis=1)            # exact in FP64
    w = dq(qw) * np.repeat(np.repeat(np.asarray(sw, np.float64), GROUP, axis=0), GROUP, axis=1)[:N, :K]
    ai, pa = _to_scaled_ints(a)
    wi, pw = _to_scaled_ints(w)
    num = ai.dot(wi.T)                       # Python-int dot products: exact
    den = 1 << (pa + pw)
    exact = np.empty((M, N), dtype=object)
    for i in range(M):
        for j in range(N):
            exact[i, j] = Fraction(int(num[i, j]), den)
    abs_sum = np.abs(a).dot(np.abs(w).T)
    return exact, abs_sum
