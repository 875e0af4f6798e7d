"""Plain CPU oracle for the W8A8 FP8 block-scaled linear layer.

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` use this package; the product library never
imports, links or runs it, and it imports nothing from the product package.

The arithmetic lives in ``oracle.c`` (plain C, FP64 GEMM accumulation, binary32
quantizer arithmetic); this module only builds it with gcc and marshals numpy
arrays through ctypes.  Functions and the passages they follow (page
"ProCreations/Nanbeige4.3-33B-FP8"):

* ``quantize_act``    -- dynamic per-token / group-128 activation scales
  (introduction; "Recipe and calibration").
* ``quantize_weight`` -- per-128x128-block E4M3 min-max weight scales
  ("Recipe and calibration": standard min-max, data independent).
* ``gemm_ref``        -- FP64 sum of the dequantized operands; the linear layer
  multiplies the quantized operands and emits BF16 (introduction: W8A8 FP8).
* ``e4m3_encode`` / ``e4m3_decode`` -- the E4M3 "fn" format the page names.

Every function is pinned by ``tests/test_oracle_pins.py`` against closed forms,
exhaustive brute force, library routines and exact rational arithmetic.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

GROUP = 128


def build(force: bool = False) -> str:
    """Compile oracle.c into liboracle.so next to it (gcc, -O2, OpenMP, no fast-math)."""
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    tmp = _LIB_PATH + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-fopenmp", "-fno-fast-math", "-ffp-contract=off", "-std=c11",
           "-Wall", "-shared", "-fPIC", _SRC, "-o", tmp, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        lib = ctypes.CDLL(build())
        P = ctypes.c_void_p
        I = ctypes.c_int64
        lib.oracle_e4m3_encode.argtypes = [ctypes.c_float]
        lib.oracle_e4m3_encode.restype = ctypes.c_uint8
        lib.oracle_e4m3_decode.argtypes = [ctypes.c_uint8]
        lib.oracle_e4m3_decode.restype = ctypes.c_double
        lib.oracle_e4m3_encode_array.argtypes = [P, I, P]
        lib.oracle_e4m3_decode_array.argtypes = [P, I, P]
        lib.oracle_quantize_act.argtypes = [P, I, I, P, P]
        lib.oracle_quantize_act_rows.argtypes = [P, I, I, P, I, P, P]
        lib.oracle_quantize_weight.argtypes = [P, I, I, P, P]
        lib.oracle_gemm_ref.argtypes = [P, P, P, P, I, I, I, P, I, P]
        lib.oracle_bf16_round.argtypes = [ctypes.c_double]
        lib.oracle_kv_write.argtypes = [P, P, I, I, I, P, I, I, P, P]
        lib.oracle_kv_write.restype = ctypes.c_int64
        lib.oracle_silu_mul.argtypes = [P, I, I, P]
        lib.oracle_bf16_round_array.argtypes = [P, I, P]
        lib.oracle_e2m1_decode.argtypes = [ctypes.c_uint8]
        lib.oracle_e2m1_decode.restype = ctypes.c_double
        lib.oracle_e2m1_encode.argtypes = [ctypes.c_float]
        lib.oracle_e2m1_encode.restype = ctypes.c_uint8
        lib.oracle_nvfp4_quantize.argtypes = [P, I, I, P, P, P]
        lib.oracle_nvfp4_gemm_ref.argtypes = [P, P, I, I, P, P, ctypes.c_float, I, P]
        lib.oracle_bf16_round.restype = ctypes.c_uint16
        _lib = lib
        return lib


def _ptr(a: np.ndarray) -> ctypes.c_void_p:
    assert a.flags["C_CONTIGUOUS"]
    return ctypes.c_void_p(a.ctypes.data)


def _bf16_bits(x) -> np.ndarray:
    """Accept BF16 bit patterns as uint16 numpy, or a torch bfloat16 CPU tensor."""
    if isinstance(x, np.ndarray):
        assert x.dtype == np.uint16
        return np.ascontiguousarray(x)
    import torch  # only for the tensor -> bit pattern view
    assert x.dtype == torch.bfloat16 and x.device.type == "cpu"
    return np.ascontiguousarray(x.contiguous().view(torch.int16).numpy().view(np.uint16))


def e4m3_encode(y: np.ndarray) -> np.ndarray:
    y = np.ascontiguousarray(y, dtype=np.float32)
    out = np.empty(y.shape, dtype=np.uint8)
    _load().oracle_e4m3_encode_array(_ptr(y), y.size, _ptr(out))
    return out


def e4m3_decode(codes: np.ndarray) -> np.ndarray:
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    out = np.empty(codes.shape, dtype=np.float64)
    _load().oracle_e4m3_decode_array(_ptr(codes), codes.size, _ptr(out))
    return out


def quantize_act(x) -> tuple[np.ndarray, np.ndarray]:
    """BF16 [M, K] -> (E4M3 codes uint8 [M, K], FP32 scales [M, K/128])."""
    xb = _bf16_bits(x)
    M, K = xb.shape
    assert K % GROUP == 0
    q = np.empty((M, K), dtype=np.uint8)
    s = np.empty((M, K // GROUP), dtype=np.float32)
    _load().oracle_quantize_act(_ptr(xb), M, K, _ptr(q), _ptr(s))
    return q, s


def quantize_act_rows(x, rows) -> tuple[np.ndarray, np.ndarray]:
    """quantize_act evaluated only on the listed rows (row r of the result = rows[r])."""
    xb = _bf16_bits(x)
    M, K = xb.shape
    rows = np.ascontiguousarray(rows, dtype=np.int64)
    assert rows.size == 0 or (rows.min() >= 0 and rows.max() < M)
    q = np.empty((rows.size, K), dtype=np.uint8)
    s = np.empty((rows.size, K // GROUP), dtype=np.float32)
    _load().oracle_quantize_act_rows(_ptr(xb), M, K, _ptr(rows), rows.size, _ptr(q), _ptr(s))
    return q, s


def quantize_weight(w) -> tuple[np.ndarray, np.ndarray]:
    """BF16 [N, K] -> (E4M3 codes uint8 [N, K], FP32 scales [N/128, K/128])."""
    wb = _bf16_bits(w)
    N, K = wb.shape
    assert N % GROUP == 0 and K % GROUP == 0
    q = np.empty((N, K), dtype=np.uint8)
    s = np.empty((N // GROUP, K // GROUP), dtype=np.float32)
    _load().oracle_quantize_weight(_ptr(wb), N, K, _ptr(q), _ptr(s))
    return q, s


def gemm_ref(qa, sa, qw, sw, rows=None) -> np.ndarray:
    """FP64 reference Y[rows, :] = dequant(A)[rows] @ dequant(W)^T."""
    qa = np.ascontiguousarray(qa, dtype=np.uint8)
    sa = np.ascontiguousarray(sa, dtype=np.float32)
    qw = np.ascontiguousarray(qw, dtype=np.uint8)
    sw = np.ascontiguousarray(sw, dtype=np.float32)
    M, K = qa.shape
    N = qw.shape[0]
    assert qw.shape[1] == K and sa.shape == (M, K // GROUP)
    assert sw.shape == (N // GROUP, K // GROUP)
    if rows is None:
        rows = np.arange(M, dtype=np.int64)
    rows = np.ascontiguousarray(rows, dtype=np.int64)
    out = np.empty((rows.size, N), dtype=np.float64)
    if rows.size and N:
        _load().oracle_gemm_ref(_ptr(qa), _ptr(sa), _ptr(qw), _ptr(sw), M, N, K,
                                _ptr(rows), rows.size, _ptr(out))
    return out


def linear_ref(x, qw, sw, rows=None) -> np.ndarray:
    """FP64 reference of the linear layer: quantize the activation rows, then gemm_ref."""
    xb = _bf16_bits(x)
    M, K = xb.shape
    if rows is None:
        rows = np.arange(M, dtype=np.int64)
    rows = np.ascontiguousarray(rows, dtype=np.int64)
    qa, sa = quantize_act_rows(xb, rows)
    return gemm_ref(qa, sa, qw, sw, rows=np.arange(rows.size, dtype=np.int64))


def bf16_round(v: np.ndarray) -> np.ndarray:
    """Nearest-even BF16 bit patterns of FP64 values (one rounding, from the exact value)."""
    v = np.ascontiguousarray(v, dtype=np.float64)
    out = np.empty(v.shape, dtype=np.uint16)
    _load().oracle_bf16_round_array(_ptr(v), v.size, _ptr(out))
    return out


def kv_write(k, v, loc, k_cache: np.ndarray, v_cache: np.ndarray) -> int:
    """FP8 E4M3 KV-cache write with unit scales, in place on the host caches.

    k, v: BF16 [T, width] (torch or numpy bit patterns; any row stride); loc:
    int64 [T]; k_cache, v_cache: uint8 [num_slots, slot_bytes] with slot_bytes
    >= width.  Returns the number of rows skipped for an out-of-range slot."""
    kb, vb = _bf16_strided(k), _bf16_strided(v)
    T, width = kb.shape[0], kb.shape[1]
    assert vb.shape == (T, width)
    row_stride = kb.strides[0] // 2
    assert vb.strides[0] // 2 == row_stride and kb.strides[1] == 2 and vb.strides[1] == 2
    loc = np.ascontiguousarray(loc, dtype=np.int64)
    assert k_cache.dtype == np.uint8 and k_cache.flags.c_contiguous and k_cache.shape == v_cache.shape
    num_slots, slot_bytes = k_cache.shape
    assert slot_bytes >= width
    # a strided row view: pass its first element's address with the row stride
    kp = ctypes.c_void_p(kb.ctypes.data)
    vp = ctypes.c_void_p(vb.ctypes.data)
    return int(_load().oracle_kv_write(kp, vp, row_stride, T, width, _ptr(loc), num_slots,
                                       slot_bytes, _ptr(k_cache), _ptr(v_cache)))


def silu_mul(gu) -> np.ndarray:
    """FP64 silu(gate) * up of a BF16 [M, 2I] gate/up tensor (gate first)."""
    g = _bf16_bits(gu)
    M, two_i = g.shape
    h = np.empty((M, two_i // 2), dtype=np.float64)
    _load().oracle_silu_mul(_ptr(g), M, two_i // 2, _ptr(h))
    return h


def _bf16_strided(x) -> np.ndarray:
    """BF16 bit patterns as a uint16 [rows, cols] array.  A numpy uint16 array is
    used as is (a column slice of a wider array keeps its row stride); a torch
    BF16 tensor is copied to a contiguous host array."""
    import torch
    if isinstance(x, torch.Tensor):
        assert x.dtype == torch.bfloat16 and x.dim() == 2
        return x.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)
    a = np.asarray(x)
    assert a.dtype == np.uint16 and a.ndim == 2 and a.strides[1] == 2
    return a


def e2m1_decode(code: int) -> float:
    return float(_load().oracle_e2m1_decode(int(code)))


def e2m1_encode(y: float) -> int:
    return int(_load().oracle_e2m1_encode(float(y)))


def nvfp4_quantize(w) -> tuple[np.ndarray, np.ndarray, float]:
    """Plain min-max NVFP4 quantization of BF16 W [N, K]: (packed uint8 [N, K/2],
    E4M3 block scales uint8 [N, K/16], global FP32 scale)."""
    wb = _bf16_bits(w)
    N, K = wb.shape
    packed = np.empty((N, K // 2), dtype=np.uint8)
    sb = np.empty((N, K // 16), dtype=np.uint8)
    g = np.zeros(1, dtype=np.float32)
    _load().oracle_nvfp4_quantize(_ptr(wb), N, K, _ptr(packed), _ptr(sb), _ptr(g))
    return packed, sb, float(g[0])


def nvfp4_gemm_ref(x, packed: np.ndarray, sb: np.ndarray, g: float, rows=None) -> np.ndarray:
    """FP64 X . dequant(W)^T for BF16 X [M, K] and NVFP4 W; rows of Y as in gemm_ref."""
    xb = _bf16_bits(x)
    M, K = xb.shape
    N = packed.shape[0]
    packed = np.ascontiguousarray(packed, dtype=np.uint8)
    sb = np.ascontiguousarray(sb, dtype=np.uint8)
    if rows is None:
        r = None
        n_rows = M
    else:
        r = np.ascontiguousarray(rows, dtype=np.int64)
        n_rows = r.size
    y = np.empty((n_rows, N), dtype=np.float64)
    _load().oracle_nvfp4_gemm_ref(_ptr(xb), _ptr(r) if r is not None else None, n_rows, K,
                                  _ptr(packed), _ptr(sb), ctypes.c_float(g), N, _ptr(y))
    return y
