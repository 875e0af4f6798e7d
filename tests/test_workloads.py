"""The synthetic inputs follow the stated recipe (CPU only).

Shapes are the layer geometry of the pages: hidden 7168, fused QKV 9216
(56 + 2 x 8 heads of 128, page "shisa-ai/Nanbeige4.3-33B-DMS-2x", "Format"),
k_proj 1024, drafter MLP 8192 and fusion input 21504 (page
"ProCreations/Nanbeige4.3-33B-DFlash2", "Architecture").  The values follow the
recipe in workloads/__init__.py: N(0, 1) activations, N(0, 0.02^2) weights,
seeded outlier channels x 20, an all-zero k_proj row, Student-t(3) channels in
the long prefill, u * v for the down projection, one RNE cast to BF16.
"""
import numpy as np
import torch

import workloads as W


def bf16_bits(x: torch.Tensor) -> np.ndarray:
    return x.contiguous().view(torch.int16).numpy().view(np.uint16)


def test_shapes_of_every_workload():
    assert (W.KPROJ_M16.M, W.KPROJ_M16.N, W.KPROJ_M16.K) == (16, 1024, 7168)
    assert {(g.M, g.N, g.K) for g in W.DECODE_SET} == {
        (m, n, 7168) for m in (1, 4, 8) for n in (9216, 7168)}
    assert (W.PREFILL_QKV.M, W.PREFILL_QKV.N, W.PREFILL_QKV.K) == (8192, 9216, 7168)
    assert [(g.M, g.N, g.K) for g in W.DRAFTER_MLP] == [
        (4096, 7168, 21504), (4096, 16384, 7168), (4096, 7168, 8192)]
    assert (W.LONG_O_PROJ.M, W.LONG_O_PROJ.N, W.LONG_O_PROJ.K) == (32768, 7168, 7168)
    assert {(g.M, g.N) for g in W.MIDM_SET} == {(m, n) for m in (32, 128) for n in (9216, 7168)}
    names = [g.name for g in W.ALL]
    assert len(names) == len(set(names))
    assert all(W.by_name(n).name == n for n in names)
    # every dimension the kernels tile is a multiple of 128
    assert all(g.N % 128 == 0 and g.K % 128 == 0 for g in W.ALL)


def test_seeds_follow_workload_and_tensor_index():
    assert W.seed_of(1, 0) == 0          # the k_proj workload starts at seed 0
    assert W.seed_of(3, 2) == 2002
    x_seeds = {W.seed_of(g.workload, g.x_seed_t) for g in W.DECODE_SET}
    assert len(x_seeds) == len(W.DECODE_SET)   # every decode layer gets its own X
    w_seeds = {(g.N, W.seed_of(g.workload, g.w_seed_t)) for g in W.DECODE_SET}
    assert len(w_seeds) == 2                   # one QKV and one o_proj weight


def test_bf16_is_one_round_to_nearest_even_cast_of_the_float32_draw():
    a = W.normal((16, 512), 11)
    x = W.activation(16, 512, 11)
    bits = a.view(np.uint32).astype(np.uint64)
    rne = ((bits + 0x7FFF + ((bits >> 16) & 1)) >> 16).astype(np.uint16)  # no NaN in a draw
    assert np.array_equal(bf16_bits(x), rne)


def test_outlier_channels_are_a_seeded_set_scaled_by_20():
    M, K, seed = 64, 7168, 5
    plain = W.normal((M, K), seed)
    x = W.activation(M, K, seed, outliers=7)
    ch = W.outlier_channels(K, 7, seed + 500)
    assert len(set(ch.tolist())) == 7
    changed = np.nonzero(np.any(bf16_bits(x) != bf16_bits(W.activation(M, K, seed)), axis=0))[0]
    assert np.array_equal(changed, ch)
    expect = torch.from_numpy(np.ascontiguousarray(plain[:, ch] * np.float32(20))).to(torch.bfloat16)
    assert torch.equal(x[:, ch], expect)
    assert W.OUTLIERS_0P1 == 7 and W.KPROJ_M16.outliers == 8
    assert all(g.outliers == 7 for g in W.DECODE_SET + W.MIDM_SET + (W.PREFILL_QKV,))


def test_kproj_last_row_is_positive_zero():
    x = W.KPROJ_M16.make_x()
    assert np.all(bf16_bits(x[-1]) == 0)       # +0.0, not -0.0
    assert np.all(np.any(bf16_bits(x[:-1]) != 0, axis=1))


def test_long_prefill_has_72_student_t_channels():
    g = W.LONG_O_PROJ
    assert g.t3_channels == 72 and g.x_kind == "t3"
    M, K, seed = 512, g.K, W.seed_of(g.workload, g.x_seed_t)
    x = W.activation(M, K, seed, t3_channels=72)
    changed = np.nonzero(np.any(bf16_bits(x) != bf16_bits(W.activation(M, K, seed)), axis=0))[0]
    assert len(changed) == 72
    heavy = x[:, changed].float().numpy().ravel().astype(np.float64)
    normal = np.delete(x.float().numpy(), changed, axis=1).ravel().astype(np.float64)
    kurt = lambda v: np.mean((v - v.mean()) ** 4) / np.var(v) ** 2 - 3.0
    assert kurt(heavy) > 3.0 > 0.2 > abs(kurt(normal))   # t(3) tails vs a normal


def test_down_input_is_a_product_of_two_normal_draws():
    x = W.gated_activation(8, 256, 9)
    u, v = W.normal((8, 256), 9), W.normal((8, 256), 10)
    assert torch.equal(x, torch.from_numpy(u * v).to(torch.bfloat16))
    assert W.DRAFTER_DOWN.x_kind == "gated"


def test_spreads_of_weights_and_activations():
    w = W.weight(512, 1024, 3).float().numpy()
    assert abs(w.std() / 0.02 - 1.0) < 0.02 and abs(w.mean()) < 1e-3
    x = W.activation(256, 1024, 4).float().numpy()
    assert abs(x.std() - 1.0) < 0.02 and abs(x.mean()) < 0.01


def test_scaled_keeps_the_structure_at_a_smaller_size():
    g = W.scaled(W.LONG_O_PROJ, M=64, K=512)
    assert (g.M, g.N, g.K, g.x_kind) == (64, W.LONG_O_PROJ.N, 512, "t3")
    assert g.t3_channels == 32                     # at most one channel in 16
    k = W.scaled(W.KPROJ_M16, K=1024)
    assert k.outliers == 8 and k.zero_last_row
    x = k.make_x()
    assert x.shape == (16, 1024) and np.all(bf16_bits(x[-1]) == 0)
    assert W.scaled(W.PREFILL_QKV) == W.PREFILL_QKV  # no sizes given: unchanged
