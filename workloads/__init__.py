"""Seeded synthetic inputs for the W8A8 FP8 block-scaled linear layer.

This module is shared by the oracle-side tests and the CUDA-side tests and
benchmark.  It holds none of the method's arithmetic: it draws BF16 tensors
with the shapes and value structure of the five workloads and nothing else.

Shapes follow the Nanbeige4.3-33B geometry stated on the page
"shisa-ai/Nanbeige4.3-33B-DMS-2x" (section "Format": hidden 7168, 56 query
heads and 8 KV heads of dimension 128, so fused QKV is 9216 x 7168 and o_proj
7168 x 7168) and the drafter geometry on "ProCreations/Nanbeige4.3-33B-DFlash2"
(section "Architecture": MLP 8192, fusion fc 21504 -> 7168).

Recipe (all draws float32 from numpy PCG64 ``default_rng(seed)``, then one
round-to-nearest-even cast to BF16 by torch):

* activations ~ N(0, 1); weights ~ N(0, 0.02^2);
* "outlier channels": a seeded set of distinct channel indices, multiplied by
  20 before the cast (8 channels for the k_proj workload, round(0.001 K) = 7
  elsewhere);
* "one row all zeros" (k_proj workload): the last activation row is +0.0;
* heavy-tailed channels (long-prefill workload): 1% of channels (72 of 7168)
  redrawn from Student-t with 3 degrees of freedom;
* SiLU-gated input to the down projection: the product u * v of two
  independent N(0, 1) draws, taken literally.

Seeds: workload c (1-based) tensor t uses seed 1000 (c - 1) + t, so the
k_proj workload starts at seed 0.
"""
from __future__ import annotations

import dataclasses

import numpy as np

HIDDEN = 7168
QKV = 9216
KPROJ = 1024
MLP = 8192
FUSION_IN = 21504
GATE_UP = 16384


def seed_of(workload: int, tensor: int) -> int:
    return 1000 * (workload - 1) + tensor


def _to_bf16(a: np.ndarray):
    import torch
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16)


def normal(shape, seed: int, std: float = 1.0) -> np.ndarray:
    rng = np.random.default_rng(seed)
    a = rng.standard_normal(shape, dtype=np.float32)
    if std != 1.0:
        a *= np.float32(std)
    return a


def outlier_channels(K: int, count: int, seed: int) -> np.ndarray:
    rng = np.random.default_rng(seed)
    return np.sort(rng.choice(K, size=count, replace=False))


def activation(M: int, K: int, seed: int, outliers: int = 0, outlier_scale: float = 20.0,
               zero_last_row: bool = False, t3_channels: int = 0):
    """BF16 [M, K] activation with the requested structure (torch CPU tensor)."""
    a = normal((M, K), seed)
    if outliers:
        ch = outlier_channels(K, outliers, seed + 500)
        a[:, ch] *= np.float32(outlier_scale)
    if t3_channels:
        rng = np.random.default_rng(seed + 700)
        ch = np.sort(rng.choice(K, size=t3_channels, replace=False))
        a[:, ch] = rng.standard_t(3, size=(M, t3_channels)).astype(np.float32)
    if zero_last_row and M > 0:
        a[M - 1, :] = 0.0
    return _to_bf16(a)


def gated_activation(M: int, K: int, seed: int):
    """BF16 [M, K] drawn as u * v with u, v iid N(0, 1) (the down-projection input)."""
    u = normal((M, K), seed)
    v = normal((M, K), seed + 1)
    return _to_bf16(u * v)


def weight(N: int, K: int, seed: int, std: float = 0.02):
    """BF16 [N, K] ~ N(0, std^2) (out x in, nn.Linear layout)."""
    return _to_bf16(normal((N, K), seed, std))


@dataclasses.dataclass(frozen=True)
class Gemm:
    """One linear layer instance: Y[M, N] = X[M, K] W[N, K]^T."""
    name: str
    M: int
    N: int
    K: int
    workload: int
    x_kind: str = "normal"          # normal | gated | t3
    outliers: int = 0
    zero_last_row: bool = False
    t3_channels: int = 0
    x_seed_t: int = 0               # tensor index of X within the workload
    w_seed_t: int = 1               # tensor index of W within the workload

    @property
    def flops(self) -> int:
        return 2 * self.M * self.N * self.K

    def make_x(self, M: int | None = None):
        M = self.M if M is None else M
        seed = seed_of(self.workload, self.x_seed_t)
        if self.x_kind == "gated":
            return gated_activation(M, self.K, seed)
        return activation(M, self.K, seed, outliers=self.outliers,
                          zero_last_row=self.zero_last_row, t3_channels=self.t3_channels)

    def make_w(self):
        return weight(self.N, self.K, seed_of(self.workload, self.w_seed_t))


OUTLIERS_0P1 = round(0.001 * HIDDEN)  # 7 channels

# workload 1: k_proj-shaped linear, decode-sized
KPROJ_M16 = Gemm("k_proj", 16, KPROJ, HIDDEN, 1, outliers=8, zero_last_row=True)

# workload 2: decode GEMV set, M in {1, 4, 8}, fused QKV and o_proj
DECODE_SET = tuple(
    Gemm(f"{nm}_m{m}", m, n, HIDDEN, 2, outliers=OUTLIERS_0P1, x_seed_t=10 * i + 2 * j,
         w_seed_t=1 + 2 * j)
    for i, m in enumerate((1, 4, 8))
    for j, (nm, n) in enumerate((("qkv", QKV), ("o_proj", HIDDEN)))
)

# workload 3: prefill fused QKV
PREFILL_QKV = Gemm("qkv_prefill", 8192, QKV, HIDDEN, 3, outliers=OUTLIERS_0P1)

# workload 4: drafter-shaped MLP and fusion at M = 4096
DRAFTER_FC = Gemm("fc", 4096, HIDDEN, FUSION_IN, 4, outliers=0, x_seed_t=0, w_seed_t=1)
DRAFTER_GATE_UP = Gemm("gate_up", 4096, GATE_UP, HIDDEN, 4, x_seed_t=2, w_seed_t=3)
DRAFTER_DOWN = Gemm("down", 4096, HIDDEN, MLP, 4, x_kind="gated", x_seed_t=4, w_seed_t=6)
DRAFTER_MLP = (DRAFTER_FC, DRAFTER_GATE_UP, DRAFTER_DOWN)

# workload 5: long-prefill o_proj and the standalone activation quantizer
LONG_O_PROJ = Gemm("o_proj_long", 32768, HIDDEN, HIDDEN, 5, x_kind="t3",
                   t3_channels=round(0.01 * HIDDEN))  # 72 channels

# workload 6: mid-size batches between the decode and prefill regimes (the
# 128-stream aggregate decode step and a 32-row batch), fused QKV and o_proj
MIDM_SET = tuple(
    Gemm(f"{nm}_m{m}", m, n, HIDDEN, 6, outliers=OUTLIERS_0P1, x_seed_t=10 * i + 2 * j,
         w_seed_t=1 + 2 * j)
    for i, m in enumerate((32, 128))
    for j, (nm, n) in enumerate((("qkv", QKV), ("o_proj", HIDDEN)))
)

ALL = (KPROJ_M16,) + DECODE_SET + (PREFILL_QKV,) + DRAFTER_MLP + (LONG_O_PROJ,) + MIDM_SET


def by_name(name: str) -> Gemm:
    for g in ALL:
        if g.name == name:
            return g
    raise KeyError(name)


def scaled(g: Gemm, M: int | None = None, N: int | None = None, K: int | None = None) -> Gemm:
    """Same structure at a smaller size (tests that the oracle finishes in seconds)."""
    return dataclasses.replace(g, M=g.M if M is None else M, N=g.N if N is None else N,
                               K=g.K if K is None else K,
                               outliers=min(g.outliers, (K or g.K) // 16),
                               t3_channels=min(g.t3_channels, (K or g.K) // 16))
