"""GPU parity of the block-scaled GEMM and the fused linear layer.

The GEMM is fed the oracle's codes and scales; its BF16 output must satisfy
|y - ref| <= 1e-2 |ref| + 2e-3 rms(ref) against the oracle's FP64 sum of the
dequantized operands (tolerance of the library's accuracy contract; the page
"ProCreations/Nanbeige4.3-33B-FP8", "Compatibility and limitations", claims no
bit-exact equivalence across kernel geometry).  Shapes span several tiles with
ragged M tails on the decode path (every token tile: M <= 16, 32, 64, 128)
and the prefill path (M > 128); the full
workload shapes are checked on sampled rows.  In the exact-arithmetic regime
(small-integer codes, power-of-two scales) every partial sum is exact in FP32,
so the output must equal the BF16 rounding of the exact result bit for bit.
"""
import os
import subprocess
import sys

import numpy as np
import pytest
import torch

import fp8_block_scaled_09_b200 as fp8bq
import oracle
import workloads
from gpu_util import Guarded, bf16_to_f64, to_dev_codes, to_dev_f32, tolerance_report

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _device():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    fp8bq.lib()
    yield
    assert fp8bq.last_device_status() == 0


def operands(M, N, K, seed, x=None):
    if x is None:
        x = workloads.activation(M, K, seed, outliers=max(1, K // 1024))
    w = workloads.weight(N, K, seed + 1)
    qa, sa = oracle.quantize_act(x)
    qw, sw = oracle.quantize_weight(w)
    return x, qa, sa, qw, sw


def run_gemm(qa, sa, qw, sw):
    M, K = qa.shape
    N = qw.shape[0]
    y = Guarded((M, N), torch.bfloat16)
    ws = fp8bq.new_workspace(fp8bq.OP_GEMM, M, N, K, "cuda")
    fp8bq.gemm(to_dev_codes(qa), to_dev_f32(sa), to_dev_codes(qw), to_dev_f32(sw), out=y.t,
               workspace=ws)
    torch.cuda.synchronize()
    assert y.guards_intact()
    return y.t


def check(y, ref):
    ok, ratio, rms = tolerance_report(y, ref)
    assert ok, f"worst error / bound = {ratio:.3f} (rms(ref) = {rms:.4g})"


# Up to 148 n-blocks the decode kernel splits each n-block over a cluster of
# CTAs (sizes 1-8: e.g. 2 for QKV, 3 for (2, 256, 384), 5 for (7, 640, 640), 8
# for k_proj, (9, 2048, 2048) and (5, 1280, 1536)); beyond that it runs
# stream-K with the global split-K reduction ((4, 19200, 512), (3, 32768, 256)).
DECODE_SHAPES = [(1, 128, 128), (1, 1024, 7168), (2, 256, 384), (4, 9216, 7168),
                 (8, 7168, 7168), (15, 384, 1024), (16, 1024, 7168), (16, 128, 21504),
                 (3, 16384, 256), (7, 640, 640), (4, 19200, 512), (3, 32768, 256),
                 (9, 2048, 2048), (5, 1280, 1536)]


@pytest.mark.parametrize("M,N,K", DECODE_SHAPES)
def test_gemm_decode_path(M, N, K):
    _, qa, sa, qw, sw = operands(M, N, K, 100 + M)
    y = run_gemm(qa, sa, qw, sw)
    check(bf16_to_f64(y), oracle.gemm_ref(qa, sa, qw, sw))


# one or more shapes per token tile (17..32, 33..64, 65..128), with ragged M,
# several n-blocks split across CTAs and a K long enough that the staged scales
# cut the ring to four stages at M > 64
MIDM_SHAPES = [(17, 128, 128), (32, 256, 384), (33, 1024, 7168), (64, 384, 1024),
               (65, 2048, 896), (100, 1152, 7168), (127, 384, 1024), (128, 256, 256),
               (128, 512, 21504), (40, 20480, 256), (128, 19200, 384)]


@pytest.mark.parametrize("M,N,K", MIDM_SHAPES)
def test_gemm_mid_m_decode_path(M, N, K):
    _, qa, sa, qw, sw = operands(M, N, K, 300 + M)
    y = run_gemm(qa, sa, qw, sw)
    check(bf16_to_f64(y), oracle.gemm_ref(qa, sa, qw, sw))


# M > 128 (the 129..256 rows of the mid-size range included) runs on the prefill kernel
PREFILL_SHAPES = [(129, 384, 1024), (200, 2048, 7168), (255, 1152, 512), (256, 1024, 1024),
                  (255, 9216, 256), (300, 1152, 512),
                  (1000, 512, 896), (300, 128, 7168), (2048, 2048, 384), (8191, 384, 256)]


@pytest.mark.parametrize("M,N,K", PREFILL_SHAPES)
def test_gemm_prefill_path(M, N, K):
    _, qa, sa, qw, sw = operands(M, N, K, 200 + M)
    y = run_gemm(qa, sa, qw, sw)
    check(bf16_to_f64(y), oracle.gemm_ref(qa, sa, qw, sw))


def sample_rows(M, step, extra=()):
    rows = set(range(0, M, step)) | {M - 1} | set(r for r in extra if 0 <= r < M)
    return np.array(sorted(rows), dtype=np.int64)


@pytest.mark.parametrize("name", ["k_proj", "qkv_m8", "o_proj_m4", "qkv_m32", "o_proj_m128",
                                  "qkv_m128", "qkv_prefill", "fc", "gate_up", "down",
                                  "o_proj_long"])
def test_gemm_full_workloads_sampled(name):
    g = workloads.by_name(name)
    x = g.make_x()
    qa, sa = oracle.quantize_act(x)
    qw, sw = oracle.quantize_weight(g.make_w())
    y = run_gemm(qa, sa, qw, sw)
    step = 1 if g.M <= 128 else max(1, g.M // 48)
    rows = sample_rows(g.M, step, extra=(127, 128, g.M - 129))
    ref = oracle.gemm_ref(qa, sa, qw, sw, rows=rows)
    check(bf16_to_f64(y)[rows], ref)


@pytest.mark.parametrize("M,N,K", [(4, 256, 512), (40, 640, 1024), (128, 384, 2048),
                                   (300, 384, 640)])
def test_gemm_exact_arithmetic_regime_bit_exact(M, N, K):
    rng = np.random.default_rng(M)
    small = np.array([0x00, 0x38, 0x40, 0x44, 0x48, 0xB8, 0xC0, 0xC4], np.uint8)  # 0,+-1,+-2,+-3,4
    qa = rng.choice(small, size=(M, K))
    qw = rng.choice(small, size=(N, K))
    sa = np.ldexp(np.float32(1.0), rng.integers(-3, 3, size=(M, K // 128))).astype(np.float32)
    sw = np.ldexp(np.float32(1.0), rng.integers(-3, 3, size=(N // 128, K // 128))).astype(np.float32)
    y = run_gemm(qa, sa, qw, sw)
    ref = oracle.gemm_ref(qa, sa, qw, sw)            # exact: |sums| < 2^24 at these sizes
    expect = oracle.bf16_round(ref)
    got = y.cpu().view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(got, expect)


def test_gemm_identity_weight_closed_form():
    M = 200
    x = workloads.activation(M, 128, 21, outliers=1)
    qa, sa = oracle.quantize_act(x)
    qw, sw = oracle.quantize_weight(torch.eye(128, dtype=torch.bfloat16))
    y = run_gemm(qa, sa, qw, sw)
    # Y[m, n] = BF16(dq(qa[m, n]) * fl32(sa[m] * sw)) * 448 ... evaluated by the oracle in FP64
    check(bf16_to_f64(y), oracle.gemm_ref(qa, sa, qw, sw))


@pytest.mark.parametrize("M", [8, 96, 200, 600])
def test_gemm_deterministic(M):
    _, qa, sa, qw, sw = operands(M, 1024, 7168, 7)
    y1 = run_gemm(qa, sa, qw, sw).cpu()
    y2 = run_gemm(qa, sa, qw, sw).cpu()
    assert torch.equal(y1.view(torch.int16), y2.view(torch.int16))


def test_gemm_empty_m_is_noop():
    qa = torch.zeros((0, 256), dtype=torch.uint8, device="cuda")
    sa = torch.zeros((0, 2), dtype=torch.float32, device="cuda")
    qw = torch.zeros((128, 256), dtype=torch.uint8, device="cuda")
    sw = torch.ones((1, 2), dtype=torch.float32, device="cuda")
    y = fp8bq.gemm(qa, sa, qw, sw)
    assert y.shape == (0, 128)


# ------------------------------------------------------------------ fused linear

# decode-sized M on every plan of the decode kernel (cluster split with S = 8,
# 2, 1; stream-K with K ranges that wrap around K within a CTA; K so long that
# the scale table takes most of the shared memory), and larger M.
LINEAR_SHAPES = [(1, 1024, 7168), (16, 1024, 7168), (5, 384, 640), (1, 9216, 7168),
                 (8, 7168, 7168), (17, 1152, 512), (32, 2048, 2048), (31, 640, 7168),
                 (4, 19200, 512), (3, 32768, 256), (12, 16384, 1024), (20, 256, 128000),
                 (33, 256, 1024), (128, 1152, 7168), (192, 640, 2048), (700, 384, 7168),
                 (129, 256, 128), (2100, 512, 1024), (4096, 256, 384)]


@pytest.mark.parametrize("M,N,K", LINEAR_SHAPES)
def test_linear_matches_oracle_and_unfused_path(M, N, K):
    x, qa, sa, qw, sw = operands(M, N, K, 300 + M)
    xd = x.cuda()
    y = Guarded((M, N), torch.bfloat16)
    ws = fp8bq.new_workspace(fp8bq.OP_LINEAR, M, N, K, "cuda")
    fp8bq.linear(xd, to_dev_codes(qw), to_dev_f32(sw), out=y.t, workspace=ws)
    torch.cuda.synchronize()
    assert y.guards_intact()
    check(bf16_to_f64(y.t), oracle.linear_ref(x, qw, sw))
    # same codes and scales as the standalone quantizer feeding the standalone GEMM
    gq, gs = fp8bq.quantize_act(xd)
    y2 = fp8bq.gemm(gq, gs, to_dev_codes(qw), to_dev_f32(sw))
    assert torch.equal(y.t.view(torch.int16), y2.view(torch.int16))
    # the linear's scratch (behind the GEMM's part of a workspace of the
    # reported size) holds exactly those codes and scales
    up = lambda b: -(-b // 256) * 256
    off = ws.numel() - up(M * K) - up(M * (K // 128) * 4)
    assert torch.equal(ws[off:off + M * K].view(M, K), gq)
    so = off + up(M * K)
    assert torch.equal(ws[so:so + M * (K // 128) * 4].view(torch.float32).view(M, K // 128), gs)
    # and the split-K counters are back at zero
    assert int(ws[:16384].count_nonzero()) == 0


# ------------------------------------------------------------------ prefill split-K tail

# (M/128) x (N/256) = 160 or 150 tiles on a 148-SM grid with K >= 16384: the
# last wave's 12 or 2 tiles are split K-wise into parts whose FP32 partials the
# last part sums.  (Shorter K runs without the split; (1190, 4096, 7168) checks
# that path on the same tile count.)
@pytest.mark.parametrize("M,N,K", [(1280, 4096, 16384), (1190, 3840, 16384), (1190, 4096, 7168)])
def test_prefill_split_tail_matches_oracle(M, N, K):
    x, qa, sa, qw, sw = operands(M, N, K, 980 + M + K)
    y = run_gemm(qa, sa, qw, sw)
    rows = sample_rows(M, 24, extra=(127, 128, 1023, 1024, 1151, 1152, M - 129))
    check(bf16_to_f64(y)[rows], oracle.gemm_ref(qa, sa, qw, sw, rows=rows))


def test_prefill_split_tail_exact_and_without_workspace():
    # exact regime: the split sums are exact, so the tail split, a second call on
    # the same workspace (its counters back at zero) and a call without the
    # workspace (no split) all give the exact result bit for bit.  160 tiles: the
    # last 12 in raster order (m-tiles 8, 9 of n-tile 14, all of n-tile 15) are
    # split; rows 1024.. hold every split tile's rows.
    M, N, K = 1280, 4096, 16384
    rng = np.random.default_rng(77)
    small = np.array([0x00, 0x38, 0x40, 0x44, 0xB8, 0xC0], np.uint8)
    qa, qw = rng.choice(small, size=(M, K)), rng.choice(small, size=(N, K))
    # scales 2^-1..2^1: every partial sum is a multiple of 2^-2 below 2^20, exact
    sa = np.ldexp(np.float32(1.0), rng.integers(-1, 2, size=(M, K // 128))).astype(np.float32)
    sw = np.ldexp(np.float32(1.0), rng.integers(-1, 2, size=(N // 128, K // 128))).astype(np.float32)
    rows = np.arange(1024, M, dtype=np.int64)
    expect = oracle.bf16_round(oracle.gemm_ref(qa, sa, qw, sw, rows=rows))  # BF16 bit patterns
    dev = (to_dev_codes(qa), to_dev_f32(sa), to_dev_codes(qw), to_dev_f32(sw))
    ws = fp8bq.new_workspace(fp8bq.OP_GEMM, M, N, K, "cuda")
    assert ws.numel() > 8 << 20
    for workspace in (ws, ws, torch.zeros(256, dtype=torch.uint8, device="cuda")):
        y = fp8bq.gemm(*dev, workspace=workspace)
        torch.cuda.synchronize()
        assert np.array_equal(y.cpu().view(torch.int16).numpy().view(np.uint16)[rows], expect)
    assert int(ws[:64].sum()) == 0  # the tail counters are back at zero


# ------------------------------------------------------------------ CTA-pair prefill kernel

_PAIR_CHECK = r"""
import numpy as np, torch
import fp8_block_scaled_09_b200 as fp8bq, oracle, workloads
from gpu_util import bf16_to_f64, to_dev_codes, to_dev_f32, tolerance_report
for i, (M, N, K) in enumerate([(300, 512, 1024), (1000, 768, 2048), (256, 1152, 7168),
                               (129, 256, 256), (700, 384, 1024), (2100, 640, 512)]):
    x = workloads.activation(M, K, 960 + i, outliers=2)
    qa, sa = oracle.quantize_act(x)
    qw, sw = oracle.quantize_weight(workloads.weight(N, K, 970 + i))
    y = fp8bq.gemm(to_dev_codes(qa), to_dev_f32(sa), to_dev_codes(qw), to_dev_f32(sw))
    torch.cuda.synchronize()
    ok, ratio, _ = tolerance_report(bf16_to_f64(y), oracle.gemm_ref(qa, sa, qw, sw))
    assert ok, (M, N, K, ratio)
rng = np.random.default_rng(5)
small = np.array([0x00, 0x38, 0x40, 0x44, 0xB8, 0xC0], np.uint8)
M, N, K = 384, 512, 1024
qa, qw = rng.choice(small, size=(M, K)), rng.choice(small, size=(N, K))
sa = np.ldexp(np.float32(1.0), rng.integers(-2, 3, size=(M, K // 128))).astype(np.float32)
sw = np.ldexp(np.float32(1.0), rng.integers(-2, 3, size=(N // 128, K // 128))).astype(np.float32)
y = fp8bq.gemm(to_dev_codes(qa), to_dev_f32(sa), to_dev_codes(qw), to_dev_f32(sw))
torch.cuda.synchronize()
exp = oracle.bf16_round(oracle.gemm_ref(qa, sa, qw, sw))  # BF16 bit patterns
assert np.array_equal(y.cpu().view(torch.int16).numpy().view(np.uint16), exp)
assert fp8bq.last_device_status() == 0
print("pair prefill ok")
"""


def test_pair_prefill_kernel_when_selected():
    # The CTA-pair prefill kernel is off by default; FP8BQ_PREFILL_PAIRS=1 (read
    # once per device) selects it, so it runs in a process of its own.
    here = os.path.dirname(os.path.abspath(__file__))
    root = os.path.dirname(here)
    env = dict(os.environ, FP8BQ_PREFILL_PAIRS="1",
               PYTHONPATH=os.pathsep.join([root, here, os.environ.get("PYTHONPATH", "")]))
    r = subprocess.run([sys.executable, "-c", _PAIR_CHECK], env=env, capture_output=True,
                       text=True, timeout=900, cwd=root)
    assert r.returncode == 0, r.stdout[-2000:] + r.stderr[-4000:]
    assert "pair prefill ok" in r.stdout


# ------------------------------------------------------------------ descriptor cache

@pytest.mark.parametrize("M,N,K", [(8, 1024, 1024), (300, 512, 1024)])
def test_descriptor_cache_reuse_new_contents_and_clear(M, N, K):
    # Repeated calls on the same buffers reuse the cached TMA descriptors; a
    # descriptor names an address, not contents, so new data in the same
    # buffers must be read; clearing the cache changes nothing either.
    dev = [torch.empty((M, K), dtype=torch.uint8, device="cuda"),
           torch.empty((M, K // 128), dtype=torch.float32, device="cuda"),
           torch.empty((N, K), dtype=torch.uint8, device="cuda"),
           torch.empty((N // 128, K // 128), dtype=torch.float32, device="cuda")]
    y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    ws = fp8bq.new_workspace(fp8bq.OP_GEMM, M, N, K, "cuda")
    for i, clear in enumerate((False, False, True)):
        x, qa, sa, qw, sw = operands(M, N, K, 940 + 7 * i)
        for d, h in zip(dev, (qa, sa, qw, sw)):
            d.copy_(torch.from_numpy(np.ascontiguousarray(
                h, dtype=np.float32 if d.dtype == torch.float32 else np.uint8)))
        if clear:
            fp8bq.clear_cache()
        fp8bq.gemm(*dev, out=y, workspace=ws)
        torch.cuda.synchronize()
        check(bf16_to_f64(y), oracle.gemm_ref(qa, sa, qw, sw))


# ------------------------------------------------------------------ stream order

def test_weights_quantized_right_before_the_linear():
    # The decode linear requests weight blocks before its dependency wait.  The
    # weight quantizer just before it on the same stream never lets its
    # successor start early, so the linear must see the new weights, not the
    # zeros the buffers held before.
    M, N, K = 4, 9216, 7168
    x = workloads.activation(M, K, 910, outliers=7)
    w = workloads.weight(N, K, 911)
    qw_ref, sw_ref = oracle.quantize_weight(w)
    ref = oracle.linear_ref(x, qw_ref, sw_ref)
    xd, wd = x.cuda(), w.cuda()
    ws = fp8bq.new_workspace(fp8bq.OP_LINEAR, M, N, K, "cuda")
    for _ in range(3):
        qw = torch.zeros((N, K), dtype=torch.uint8, device="cuda")
        sw = torch.zeros((N // 128, K // 128), dtype=torch.float32, device="cuda")
        torch.cuda.synchronize()
        fp8bq.quantize_weight(wd, qw, sw)
        y = fp8bq.linear(xd, qw, sw, workspace=ws)
        torch.cuda.synchronize()
        check(bf16_to_f64(y), ref)


@pytest.mark.parametrize("M", [8, 200])
def test_linear_chain_reads_the_previous_output(M):
    # Each layer's input is the previous layer's output, all launched back to
    # back with one shared workspace and no host synchronisation: every
    # activation read and workspace write must wait for the kernels before it.
    K, layers = 1024, 6
    x0 = workloads.activation(M, K, 920)
    weights = [oracle.quantize_weight(workloads.weight(K, K, 921 + i)) for i in range(layers)]
    ws = fp8bq.new_workspace(fp8bq.OP_LINEAR, M, K, K, "cuda")
    cur, outs = x0.cuda(), []
    for qw, sw in weights:
        cur = fp8bq.linear(cur, to_dev_codes(qw), to_dev_f32(sw), workspace=ws)
        outs.append(cur)
    torch.cuda.synchronize()
    prev = x0
    for (qw, sw), y in zip(weights, outs):
        check(bf16_to_f64(y), oracle.linear_ref(prev, qw, sw))
        prev = y.cpu()


def test_linear_kproj_workload_with_zero_row():
    g = workloads.KPROJ_M16
    x = g.make_x()
    qw, sw = oracle.quantize_weight(g.make_w())
    y = fp8bq.linear(x.cuda(), to_dev_codes(qw), to_dev_f32(sw))
    torch.cuda.synchronize()
    yf = bf16_to_f64(y)
    check(yf, oracle.linear_ref(x, qw, sw))
    assert np.all(yf[g.M - 1] == 0.0)          # the all-zero activation row


def test_linear_prefill_qkv_sampled():
    g = workloads.PREFILL_QKV
    x = g.make_x()
    qw, sw = oracle.quantize_weight(g.make_w())
    y = fp8bq.linear(x.cuda(), to_dev_codes(qw), to_dev_f32(sw))
    torch.cuda.synchronize()
    rows = sample_rows(g.M, 256, extra=(128, 4095, 4096))
    check(bf16_to_f64(y)[rows], oracle.linear_ref(x, qw, sw, rows=rows))


def test_gemm_workspace_reused_across_calls():
    # split-K counters must be back at zero after every call for the next one to be right
    shapes = [(8, 9216, 7168), (100, 1152, 7168), (3, 16384, 256), (8, 9216, 7168),
              (64, 2048, 1024)]
    ws = torch.zeros(max(fp8bq.workspace_size(fp8bq.OP_GEMM, *s) for s in shapes),
                     dtype=torch.uint8, device="cuda")
    outs = []
    for i, (M, N, K) in enumerate(shapes):
        _, qa, sa, qw, sw = operands(M, N, K, 40 + (i % 3) + M)
        y = fp8bq.gemm(to_dev_codes(qa), to_dev_f32(sa), to_dev_codes(qw), to_dev_f32(sw),
                       workspace=ws)
        torch.cuda.synchronize()
        check(bf16_to_f64(y), oracle.gemm_ref(qa, sa, qw, sw))
        outs.append(y.cpu())
    assert torch.equal(outs[0].view(torch.int16), outs[3].view(torch.int16))


def test_one_workspace_serves_gemm_and_linear_of_any_shape():
    # The split-K counters sit at offset 0 of every workspace, and the fused
    # linear keeps its activation scratch behind them: one workspace serves a
    # mixed sequence of linear and gemm calls (stream-K decode, cluster decode,
    # mid-size M, the prefill split-K tail) in stream order.
    calls = [("linear", 4, 19200, 512), ("gemm", 3, 32768, 256), ("linear", 8, 9216, 7168),
             ("gemm", 4, 19200, 512), ("linear", 100, 1152, 7168), ("linear", 1280, 4096, 16384),
             ("gemm", 3, 32768, 256), ("gemm", 1280, 4096, 16384), ("linear", 4, 19200, 512)]
    op_of = {"linear": fp8bq.OP_LINEAR, "gemm": fp8bq.OP_GEMM}
    size = max(fp8bq.workspace_size(op_of[op], M, N, K) for op, M, N, K in calls)
    ws = torch.zeros(size, dtype=torch.uint8, device="cuda")
    first = {}
    for op, M, N, K in calls:
        x, qa, sa, qw, sw = operands(M, N, K, 500 + M + K)
        if op == "linear":
            y = fp8bq.linear(x.cuda(), to_dev_codes(qw), to_dev_f32(sw), workspace=ws)
        else:
            y = fp8bq.gemm(to_dev_codes(qa), to_dev_f32(sa), to_dev_codes(qw), to_dev_f32(sw),
                           workspace=ws)
        torch.cuda.synchronize()
        rows = sample_rows(M, 24, extra=(1024, 1151)) if M > 128 else np.arange(M, dtype=np.int64)
        ref = (oracle.linear_ref(x, qw, sw, rows=rows) if op == "linear"
               else oracle.gemm_ref(qa, sa, qw, sw, rows=rows))
        check(bf16_to_f64(y)[rows], ref)
        key = (op, M, N, K)
        if key in first:
            assert torch.equal(first[key].view(torch.int16), y.cpu().view(torch.int16))
        first.setdefault(key, y.cpu())
    assert fp8bq.last_device_status() == 0
    assert int(ws[:16384].sum()) == 0  # every counter back at zero


@pytest.mark.parametrize("M", [4, 333])
def test_device_chain_without_host_sync(M):
    # weight and activation quantization feed the GEMM on one stream with no host
    # synchronization in between: each kernel must see its predecessor's output
    N, K = 1152, 2048
    x = workloads.activation(M, K, 77, outliers=3)
    w = workloads.weight(N, K, 78)
    xd, wd = x.cuda(), w.cuda()
    torch.cuda.synchronize()
    qw_d, sw_d = fp8bq.quantize_weight(wd)
    qa_d, sa_d = fp8bq.quantize_act(xd)
    y = fp8bq.gemm(qa_d, sa_d, qw_d, sw_d)
    y2 = fp8bq.linear(xd, qw_d, sw_d)
    torch.cuda.synchronize()
    qw, sw = oracle.quantize_weight(w)
    qa, sa = oracle.quantize_act(x)
    assert np.array_equal(qw_d.cpu().numpy(), qw) and np.array_equal(qa_d.cpu().numpy(), qa)
    ref = oracle.gemm_ref(qa, sa, qw, sw)
    check(bf16_to_f64(y), ref)
    assert torch.equal(y.view(torch.int16), y2.view(torch.int16))


def test_decode_linear_near_ties_matches_unfused():
    # activation rows whose quotients sit next to E4M3 rounding midpoints: the
    # linear layer (quantizer + decode GEMM that streams weights early) must give
    # a bit-identical output to quantize_act followed by gemm
    from test_gpu_quantize import _near_tie_groups
    x = _near_tie_groups()[:16].contiguous()
    M, K = x.shape
    w = workloads.weight(256, K, 91)
    qw, sw = oracle.quantize_weight(w)
    xd = x.cuda()
    y = fp8bq.linear(xd, to_dev_codes(qw), to_dev_f32(sw))
    qa, sa = fp8bq.quantize_act(xd)
    y2 = fp8bq.gemm(qa, sa, to_dev_codes(qw), to_dev_f32(sw))
    torch.cuda.synchronize()
    assert torch.equal(y.view(torch.int16), y2.view(torch.int16))
    check(bf16_to_f64(y), oracle.linear_ref(x, qw, sw))


@pytest.mark.parametrize("M,N,K", [(1, 1024, 7168), (7, 640, 640), (16, 19200, 512), (9, 2048, 2048)])
def test_decode_linear_special_values_match_unfused(M, N, K):
    # The decode linear layer (cluster split and stream-K plans) must give an
    # output bit-identical to quantize_act followed by gemm, also for an
    # all-zero group (scale 1), BF16 subnormals (scales below 2^-92 take the
    # IEEE division) and large magnitudes, and within tolerance of the oracle.
    g = torch.Generator().manual_seed(500 + M)
    x = torch.randn((M, K), generator=g)
    x[0, :128] = 0.0
    x[M - 1, 128:256] *= 1e-39
    x[M // 2, 256:384] *= 1e30
    x = x.to(torch.bfloat16)
    w = workloads.weight(N, K, 600 + M)
    qw, sw = oracle.quantize_weight(w)
    xd, qw_d, sw_d = x.cuda(), to_dev_codes(qw), to_dev_f32(sw)
    ws = fp8bq.new_workspace(fp8bq.OP_LINEAR, M, N, K, "cuda")
    y = fp8bq.linear(xd, qw_d, sw_d, workspace=ws)
    qa, sa = fp8bq.quantize_act(xd)
    y2 = fp8bq.gemm(qa, sa, qw_d, sw_d)
    torch.cuda.synchronize()
    assert torch.equal(y.view(torch.int16), y2.view(torch.int16))
    check(bf16_to_f64(y), oracle.linear_ref(x, qw, sw))
    assert int(ws[:16384].count_nonzero()) == 0
