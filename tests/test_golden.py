"""Layer geometry and block sizes printed on the pages (tests/golden/geometry.txt).

The fixture holds the pages' numbers as printed, each with its page and
section.  These tests check the printed numbers against one another (the
sidecar's parameter count, the fusion width), then check that the synthetic
workloads and the oracle's block layout follow from them.  CPU only.
"""
import pathlib

import numpy as np
import torch

import oracle
import workloads as W

GOLDEN = pathlib.Path(__file__).parent / "golden" / "geometry.txt"


def load() -> dict:
    out = {}
    for line in GOLDEN.read_text().splitlines():
        if not line.strip() or line.startswith("#"):
            continue
        name, value, source = line.split(None, 2)
        assert source.strip(), name                      # every value cites its page
        nums = tuple(int(v) for v in value.split(","))
        out[name] = nums if len(nums) > 1 else nums[0]
    return out


G = load()


def test_printed_numbers_agree_with_one_another():
    layers, kv, hidden = G["sidecar_weight_shape"]
    # one linear head per layer and KV head over the hidden state, with a bias each
    assert layers * kv * hidden + int(np.prod(G["sidecar_bias_shape"])) == G["sidecar_parameters"]
    assert (layers, kv) == (G["target_layers"], G["target_kv_heads"]) == G["sidecar_bias_shape"]
    # the query heads span the hidden width in both models
    assert G["target_query_heads"] * G["head_dim"] == hidden == G["drafter_hidden"]
    # the fusion concatenates the hidden state of each tapped target layer
    assert len(G["drafter_tap_layers"]) * hidden == G["fusion_in"]
    assert G["fusion_out"] == hidden
    assert max(G["drafter_tap_layers"]) < G["target_layers"]


def test_workload_shapes_follow_from_the_printed_geometry():
    hd, hidden = G["head_dim"], G["drafter_hidden"]
    q, kv = G["target_query_heads"], G["target_kv_heads"]
    assert (W.HIDDEN, W.MLP, W.FUSION_IN) == (hidden, G["drafter_mlp"], G["fusion_in"])
    assert W.QKV == (q + 2 * kv) * hd                   # fused Q, K, V rows
    assert W.KPROJ == kv * hd
    assert W.GATE_UP == 2 * G["drafter_mlp"]
    assert (W.PREFILL_QKV.N, W.PREFILL_QKV.K) == (W.QKV, hidden)
    o = [g for g in W.DECODE_SET if g.N == hidden]
    assert o and all(g.K == q * hd for g in o)          # o_proj maps the heads back


def test_oracle_blocks_are_the_printed_block_sizes():
    bn, bk = G["fp8_weight_block"]
    gk = G["fp8_act_group"]
    x = torch.zeros((3, 3 * gk), dtype=torch.bfloat16)
    x[1, gk + 5] = 2.0                                    # one nonzero group
    _, sa = oracle.quantize_act(x)
    assert sa.shape == (3, 3)
    assert np.count_nonzero(sa != 1.0) == 1 and sa[1, 1] == np.float32(2.0 / 448.0)
    w = torch.zeros((2 * bn, 3 * bk), dtype=torch.bfloat16)
    w[bn + 7, 2 * bk + 9] = -4.0                          # one nonzero block
    _, sw = oracle.quantize_weight(w)
    assert sw.shape == (2, 3)
    assert np.count_nonzero(sw != 1.0) == 1 and sw[1, 2] == np.float32(4.0 / 448.0)


def test_oracle_nvfp4_groups_are_the_printed_group_size():
    g = G["nvfp4_group"]
    w = torch.zeros((2, 4 * g), dtype=torch.bfloat16)
    w[1, 2 * g + 3] = 1.0
    packed, sb, _ = oracle.nvfp4_quantize(w)
    assert sb.shape == (2, 4) and packed.shape == (2, 2 * g)
    assert np.count_nonzero(sb) == 1
