"""Host-side checks of the C ABI (no kernel is launched).

* the library builds and loads, and exports every function include/fp8bq.h declares;
* argument errors are reported synchronously with the documented status codes
  (shape, NULL, alignment, workspace), before any device work;
* workspace sizes and status strings are well defined.
On a machine without a GPU, a call with valid arguments reports
FP8BQ_ERR_NO_DEVICE; that check is skipped when a GPU is present (the
pointers used here are fake).
"""
import ctypes
import os
import re
import subprocess

import pytest
import torch

import fp8_block_scaled_09_b200 as fp8bq
from fp8_block_scaled_09_b200 import build as fp8bq_build

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include",
                      "fp8bq.h")

OK, INVALID, SHAPE, MISALIGNED, WORKSPACE, CUDA, TIMEOUT, NODEV, INDEX = range(9)


@pytest.fixture(scope="module")
def L():
    fp8bq_build.build()
    return fp8bq.lib()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(fp8bq_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_abi():
    names = declared_functions()
    for n in ("fp8bq_quantize_act", "fp8bq_quantize_weight", "fp8bq_gemm", "fp8bq_linear",
              "fp8bq_workspace_size", "fp8bq_last_device_status", "fp8bq_status_string",
              "fp8bq_kv_write_e4m3", "fp8bq_silu_mul_quantize", "fp8bq_gemm_silu_mul_quantize"):
        assert n in names


def test_library_exports_every_declared_symbol(L):
    out = subprocess.run(["nm", "-D", "--defined-only", fp8bq.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\bT (fp8bq_\w+)", out))
    missing = [n for n in declared_functions() if n not in exported]
    assert not missing, missing
    for n in declared_functions():
        assert getattr(L, n) is not None


def test_only_the_abi_is_exported(L):
    out = subprocess.run(["nm", "-D", "--defined-only", fp8bq.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    ours = set(re.findall(r"\bT (\w+)", out))
    extra = sorted(n for n in ours if not n.startswith("fp8bq_"))
    # cudart (linked statically) keeps its symbols hidden; nothing else leaks
    assert not [n for n in extra if "fp8bq" in n.lower()], extra


def test_status_strings(L):
    for code in range(9):
        assert len(fp8bq.status_string(code)) > 0
    assert fp8bq.status_string(99) == "unknown status"
    assert L.fp8bq_version() == 100


P = ctypes.c_void_p
GOOD = P(0x10000)       # fake, 16-byte aligned
ODD = P(0x10008)        # fake, misaligned


def test_quantize_act_argument_errors(L):
    f = L.fp8bq_quantize_act
    assert f(GOOD, 4, 100, GOOD, GOOD, None) == SHAPE       # K % 128
    assert f(GOOD, -1, 128, GOOD, GOOD, None) == SHAPE
    assert f(GOOD, 4, 0, GOOD, GOOD, None) == SHAPE
    assert f(GOOD, 4, 1 << 40, GOOD, GOOD, None) == SHAPE  # too large
    assert f(None, 0, 128, None, None, None) == OK           # M == 0 is a no-op
    assert f(None, 4, 128, GOOD, GOOD, None) == INVALID
    assert f(GOOD, 4, 128, None, GOOD, None) == INVALID
    assert f(GOOD, 4, 128, GOOD, None, None) == INVALID
    assert f(ODD, 4, 128, GOOD, GOOD, None) == MISALIGNED
    assert f(GOOD, 4, 128, ODD, GOOD, None) == MISALIGNED
    assert f(GOOD, 4, 128, GOOD, ODD, None) == MISALIGNED


def test_quantize_weight_argument_errors(L):
    f = L.fp8bq_quantize_weight
    assert f(GOOD, 100, 128, GOOD, GOOD, None) == SHAPE     # N % 128
    assert f(GOOD, 0, 128, GOOD, GOOD, None) == SHAPE
    assert f(GOOD, 128, 200, GOOD, GOOD, None) == SHAPE
    assert f(None, 128, 128, GOOD, GOOD, None) == INVALID
    assert f(GOOD, 128, 128, ODD, GOOD, None) == MISALIGNED


def test_gemm_argument_errors(L):
    f = L.fp8bq_gemm
    ws = fp8bq.workspace_size(fp8bq.OP_GEMM, 8, 256, 256)
    assert f(GOOD, GOOD, GOOD, GOOD, 8, 200, 256, GOOD, GOOD, ws, None) == SHAPE
    assert f(GOOD, GOOD, GOOD, GOOD, 8, 256, 250, GOOD, GOOD, ws, None) == SHAPE
    assert f(GOOD, GOOD, GOOD, GOOD, 8, 0, 256, GOOD, GOOD, ws, None) == SHAPE
    assert f(None, None, None, None, 0, 256, 256, None, None, 0, None) == OK
    assert f(GOOD, None, GOOD, GOOD, 8, 256, 256, GOOD, GOOD, ws, None) == INVALID
    assert f(GOOD, GOOD, GOOD, GOOD, 8, 256, 256, None, GOOD, ws, None) == INVALID
    assert f(GOOD, GOOD, ODD, GOOD, 8, 256, 256, GOOD, GOOD, ws, None) == MISALIGNED
    assert f(GOOD, GOOD, GOOD, GOOD, 8, 256, 256, GOOD, None, ws, None) == WORKSPACE
    assert f(GOOD, GOOD, GOOD, GOOD, 8, 256, 256, GOOD, GOOD, ws - 1, None) == WORKSPACE
    assert f(GOOD, GOOD, GOOD, GOOD, 8, 256, 256, GOOD, ODD, ws, None) == MISALIGNED


def test_linear_argument_errors(L):
    f = L.fp8bq_linear
    ws = fp8bq.workspace_size(fp8bq.OP_LINEAR, 300, 256, 256)
    assert f(GOOD, GOOD, GOOD, 300, 256, 100, GOOD, GOOD, ws, None) == SHAPE
    assert f(GOOD, GOOD, None, 300, 256, 256, GOOD, GOOD, ws, None) == INVALID
    assert f(ODD, GOOD, GOOD, 300, 256, 256, GOOD, GOOD, ws, None) == MISALIGNED
    # for M > 128: the 16 KB counter header (kept at offset 0 of every
    # workspace), then the activation codes and scales, all required (at this K
    # the prefill GEMM has no split-K tail to report)
    up = lambda b: -(-b // 256) * 256                # each part padded to 256 bytes
    assert ws == 16384 + up(300 * 256) + up(300 * 2 * 4)
    assert f(GOOD, GOOD, GOOD, 300, 256, 256, GOOD, GOOD, ws - 256, None) == WORKSPACE
    # at K >= 16384 the optional tail (header included) replaces the bare header
    ws_long = fp8bq.workspace_size(fp8bq.OP_LINEAR, 300, 256, 16384)
    tail = 16384 + 16 * 4 * 128 * 256 * 4
    assert ws_long == tail + up(300 * 16384) + up(300 * 128 * 4)
    assert f(GOOD, GOOD, GOOD, 300, 256, 16384, GOOD, GOOD, ws_long - tail + 16384 - 256,
             None) == WORKSPACE
    assert f(None, None, None, 0, 256, 256, None, None, 0, None) == OK


def test_kv_write_argument_errors(L):
    f = L.fp8bq_kv_write_e4m3
    #        k     v     rs    T  W     loc   kc    vc    slots sstride
    assert f(GOOD, GOOD, 1024, 0, 1024, None, None, None, 0, 1024, None) == OK      # T == 0
    assert f(GOOD, GOOD, 1024, -1, 1024, GOOD, GOOD, GOOD, 8, 1024, None) == INVALID
    assert f(GOOD, GOOD, 1000, 4, 1024, GOOD, GOOD, GOOD, 8, 1024, None) == INVALID  # row_stride < W
    assert f(GOOD, GOOD, 1024, 4, 1024, GOOD, GOOD, GOOD, 8, 1000, None) == INVALID  # slot < W
    assert f(GOOD, GOOD, 1028, 4, 1020, GOOD, GOOD, GOOD, 8, 1024, None) == SHAPE    # W % 8
    assert f(GOOD, GOOD, 1028, 4, 1024, GOOD, GOOD, GOOD, 8, 1024, None) == SHAPE    # stride % 8
    assert f(GOOD, GOOD, 1024, 4, 1024, GOOD, GOOD, GOOD, 8, 1032, None) == SHAPE    # slot % 16
    assert f(None, GOOD, 1024, 4, 1024, GOOD, GOOD, GOOD, 8, 1024, None) == INVALID
    assert f(GOOD, GOOD, 1024, 4, 1024, None, GOOD, GOOD, 8, 1024, None) == INVALID
    assert f(ODD, GOOD, 1024, 4, 1024, GOOD, GOOD, GOOD, 8, 1024, None) == MISALIGNED
    assert f(GOOD, GOOD, 1024, 4, 1024, P(0x10004), GOOD, GOOD, 8, 1024, None) == MISALIGNED


def test_silu_mul_quantize_argument_errors(L):
    f = L.fp8bq_silu_mul_quantize
    assert f(GOOD, 4, 100, GOOD, GOOD, None, None) == SHAPE     # I % 128
    assert f(GOOD, -1, 128, GOOD, GOOD, None, None) == SHAPE
    assert f(None, 0, 128, None, None, None, None) == OK         # M == 0
    assert f(None, 4, 128, GOOD, GOOD, None, None) == INVALID
    assert f(GOOD, 4, 128, GOOD, None, None, None) == INVALID
    assert f(GOOD, 4, 128, ODD, GOOD, None, None) == MISALIGNED
    assert f(GOOD, 4, 128, GOOD, GOOD, ODD, None) == MISALIGNED  # optional h, if given


def test_gemm_silu_mul_quantize_argument_errors(L):
    f = L.fp8bq_gemm_silu_mul_quantize
    #        qa    sa    qw    sw    M    I    K    q     s     h     ws    bytes
    assert f(GOOD, GOOD, GOOD, GOOD, 300, 100, 256, GOOD, GOOD, None, None, 0, None) == SHAPE
    assert f(GOOD, GOOD, GOOD, GOOD, 300, 128, 200, GOOD, GOOD, None, None, 0, None) == SHAPE
    assert f(GOOD, GOOD, GOOD, GOOD, -1, 128, 256, GOOD, GOOD, None, None, 0, None) == SHAPE
    assert f(None, None, None, None, 0, 128, 256, None, None, None, None, 0, None) == OK
    assert f(GOOD, GOOD, GOOD, GOOD, 300, 128, 256, None, GOOD, None, None, 0, None) == INVALID
    assert f(GOOD, GOOD, GOOD, GOOD, 300, 128, 256, GOOD, GOOD, ODD, None, 0, None) == MISALIGNED
    # decode-sized M needs its workspace (GEMM part + BF16 gate/up output)
    assert f(GOOD, GOOD, GOOD, GOOD, 8, 128, 256, GOOD, GOOD, None, None, 0, None) == WORKSPACE
    need = fp8bq.workspace_size(fp8bq.OP_GEMM_SILU, 8, 256, 256)
    assert f(GOOD, GOOD, GOOD, GOOD, 8, 128, 256, GOOD, GOOD, None, GOOD, need - 256,
             None) == WORKSPACE


def test_nvfp4_argument_errors(L):
    q = L.fp8bq_nvfp4_quantize_weight
    assert q(GOOD, 128, 100, GOOD, GOOD, GOOD, None) == SHAPE    # K % 16
    assert q(GOOD, 0, 128, GOOD, GOOD, GOOD, None) == SHAPE
    assert q(None, 128, 128, GOOD, GOOD, GOOD, None) == INVALID
    assert q(GOOD, 128, 128, GOOD, GOOD, P(0x10002), None) == MISALIGNED
    f = L.fp8bq_nvfp4_gemm_a16
    #        x     packed sb    g     M  N    K
    assert f(GOOD, GOOD, GOOD, GOOD, 4, 128, 128, GOOD, None) == SHAPE     # K % 256
    assert f(GOOD, GOOD, GOOD, GOOD, 4, 100, 256, GOOD, None) == SHAPE     # N % 128
    assert f(None, None, None, None, 0, 128, 256, None, None) == OK         # M == 0
    assert f(GOOD, GOOD, GOOD, None, 4, 128, 256, GOOD, None) == INVALID
    assert f(ODD, GOOD, GOOD, GOOD, 4, 128, 256, GOOD, None) == MISALIGNED


def test_workspace_sizes(L):
    g = lambda M, N, K: fp8bq.workspace_size(fp8bq.OP_GEMM, M, N, K)
    lin = lambda M, N, K: fp8bq.workspace_size(fp8bq.OP_LINEAR, M, N, K)
    up = lambda b: -(-b // 256) * 256
    assert g(0, 256, 256) == 0 and lin(0, 256, 256) == 0
    assert g(8, 200, 256) == 0 and g(8, 256, 200) == 0           # rejected shapes
    assert fp8bq.workspace_size(7, 8, 256, 256) == 0              # unknown op
    # prefill GEMM: nothing required; at K >= 16384 the optional split-K tail,
    # its counter header + 16 x 4 partial tiles
    tail = 16384 + 16 * 4 * 128 * 256 * 4
    assert g(8192, 9216, 7168) == 0 and g(32768, 7168, 7168) == 0
    assert g(4096, 7168, 21504) == g(1280, 4096, 16384) == tail
    assert g(1280, 4096, 16256) == 0
    d = g(16, 9216, 7168)
    assert d > 0 and d % 256 == 0
    # decode split-K: counters + (N/128 + 256) slots of 16 x 128 FP32 partials
    assert d >= (72 + 256) * 16 * 128 * 4
    # mid-size M uses the same path with a wider token tile (32, 64 or 128 rows)
    assert g(17, 9216, 7168) == 16384 + (72 + 256) * 32 * 128 * 4
    assert g(64, 9216, 7168) == 16384 + (72 + 256) * 64 * 128 * 4
    assert g(65, 9216, 7168) == g(128, 9216, 7168) == 16384 + (72 + 256) * 128 * 128 * 4
    assert g(129, 9216, 7168) == 0 and g(129, 9216, 16384) == tail
    # linear adds the activation codes and scales to the GEMM's part, which is
    # never less than the counter header
    assert lin(8192, 9216, 7168) == 16384 + 8192 * 7168 + 8192 * 56 * 4
    assert lin(16, 9216, 7168) == d + 16 * 7168 + up(16 * 56 * 4)
    assert lin(4096, 7168, 21504) == tail + 4096 * 21504 + 4096 * 168 * 4
    assert lin(300, 256, 1024) == 16384 + up(300 * 1024) + up(300 * 8 * 4)
    for args in ((1, 128, 128), (17, 384, 1024), (4096, 7168, 21504)):
        assert lin(*args) % 256 == 0 and g(*args) % 256 == 0
    # gate/up with the SiLU epilogue (N = 2I): nothing on the fused prefill path;
    # for M <= 128 the GEMM's part (at least the header) and the BF16 gate/up output
    gs = lambda M, N, K: fp8bq.workspace_size(fp8bq.OP_GEMM_SILU, M, N, K)
    assert gs(129, 16384, 7168) == 0 and gs(4096, 16384, 7168) == 0
    assert gs(8, 16384, 7168) == g(8, 16384, 7168) + 8 * 16384 * 2
    assert gs(1, 256, 128) == max(g(1, 256, 128), 16384) + up(256 * 2)
    assert gs(8, 384, 7168) == 0                                   # N = 2I needs I % 128 == 0


@pytest.mark.skipif(torch.cuda.is_available(), reason="valid calls would launch kernels on fake pointers")
def test_valid_call_without_device_reports_no_device(L):
    assert L.fp8bq_quantize_act(GOOD, 4, 128, GOOD, GOOD, None) == NODEV
    assert L.fp8bq_last_device_status(None) == NODEV
    assert L.fp8bq_selftest_timeout(20000, None) == NODEV
    assert L.fp8bq_kv_write_e4m3(GOOD, GOOD, 1024, 4, 1024, GOOD, GOOD, GOOD, 8, 1024, None) == NODEV
    assert L.fp8bq_silu_mul_quantize(GOOD, 4, 128, GOOD, GOOD, None, None) == NODEV
    assert L.fp8bq_gemm_silu_mul_quantize(GOOD, GOOD, GOOD, GOOD, 300, 128, 256, GOOD, GOOD, None,
                                          None, 0, None) == NODEV
    assert L.fp8bq_nvfp4_quantize_weight(GOOD, 128, 256, GOOD, GOOD, GOOD, None) == NODEV
    assert L.fp8bq_nvfp4_gemm_a16(GOOD, GOOD, GOOD, GOOD, 4, 128, 256, GOOD, None) == NODEV


def test_descriptor_cache_clears_without_a_device(L):
    # host-only: the cache of encoded TMA descriptors needs no GPU to be emptied
    fp8bq.clear_cache()
    fp8bq.clear_cache()


def test_selftest_limit_is_validated_on_the_host(L):
    assert L.fp8bq_selftest_timeout(0, None) == INVALID
    assert L.fp8bq_selftest_timeout(2000001, None) == INVALID


def test_binding_fails_loudly_without_cuda_tensors():
    x = torch.zeros(4, 128, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        fp8bq.quantize_act(x)


def test_header_compiles_as_c_and_cxx_and_links(L, tmp_path):
    # A C11 client: the header alone, strict warnings, every declared function
    # referenced and linked against the library, and calls that need no device.
    refs = "\n".join(f"    (void)&{n};" for n in declared_functions())
    src = tmp_path / "client.c"
    src.write_text(f"""#include "fp8bq.h"
#include <stdio.h>
#include <string.h>
int main(void) {{
{refs}
    if (fp8bq_version() <= 0) return 1;
    if (strcmp(fp8bq_status_string(FP8BQ_OK), "ok") != 0) return 2;
    if (fp8bq_workspace_size(FP8BQ_OP_GEMM, 16, 9216, 7168) == 0) return 3;
    if (fp8bq_gemm(NULL, NULL, NULL, NULL, 8, 200, 256, NULL, NULL, 0, NULL)
        != FP8BQ_ERR_UNSUPPORTED_SHAPE) return 4;
    if (fp8bq_quantize_act(NULL, 4, 128, NULL, NULL, NULL) != FP8BQ_ERR_INVALID_ARG) return 5;
    puts("client ok");
    return 0;
}}
""")
    libdir = os.path.dirname(fp8bq.LIB_PATH)
    exe = tmp_path / "client"
    subprocess.run(["gcc", "-std=c11", "-Wall", "-Wextra", "-Werror", "-pedantic",
                    "-I", os.path.dirname(HEADER), str(src), "-o", str(exe), f"-L{libdir}",
                    "-lfp8bq", f"-Wl,-rpath,{libdir}"], check=True)
    r = subprocess.run([str(exe)], capture_output=True, text=True)
    assert r.returncode == 0 and "client ok" in r.stdout, (r.returncode, r.stdout, r.stderr)
    # the same header in a C++ translation unit (extern "C" linkage)
    subprocess.run(["g++", "-std=c++17", "-Wall", "-Wextra", "-Werror", "-fsyntax-only",
                    "-x", "c++", HEADER], check=True)
