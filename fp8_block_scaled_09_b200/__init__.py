"""W8A8 FP8 block-scaled linear layer for B200 (sm_100a).

Python binding of the C ABI in ``include/fp8bq.h`` (library ``libfp8bq.so``
built in this directory by ``build.py``).  This module only marshals torch
tensors (device memory and the current CUDA stream) into the C calls; every
step of the computation runs in the library's CUDA kernels.  There is no CPU
fallback: if the library is missing or no sm_100 device is current, the calls
raise.

Functions (names follow the C ABI without the ``fp8bq_`` prefix):

* ``quantize_act(x)``        BF16 [M, K] -> (E4M3 codes uint8 [M, K], FP32 [M, K/128])
* ``quantize_weight(w)``     BF16 [N, K] -> (E4M3 codes uint8 [N, K], FP32 [N/128, K/128])
* ``gemm(qa, sa, qw, sw)``   -> BF16 [M, N]
* ``linear(x, qw, sw)``      -> BF16 [M, N], activation quantization fused into the call
* ``kv_write_e4m3(k, v, loc, k_cache, v_cache)``  E4M3 unit-scale KV-cache write (in place)
* ``silu_mul_quantize(gu)``  BF16 [M, 2I] gate|up -> (codes [M, I], FP32 [M, I/128])
* ``nvfp4_quantize_weight(w)`` BF16 [N, K] -> (packed uint8 [N, K/2], E4M3 uint8 [N, K/16], FP32 [1])
* ``nvfp4_gemm_a16(x, packed, sb, g)`` BF16 [M, K] x NVFP4 W -> BF16 [M, N]
"""
from __future__ import annotations

import ctypes
import os
import threading

import torch

__all__ = [
    "Fp8bqError", "lib", "quantize_act", "quantize_weight", "gemm", "gemm_noalloc", "linear",
    "workspace_size", "new_workspace", "workspace_init", "last_device_status",
    "launch_count", "status_string", "selftest_timeout", "OP_GEMM", "OP_LINEAR", "OP_GEMM_SILU",
    "LIB_PATH", "kv_write_e4m3", "silu_mul_quantize", "gemm_silu_mul_quantize",
    "nvfp4_quantize_weight", "nvfp4_gemm_a16",
]

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libfp8bq.so")
OP_GEMM = 0
OP_LINEAR = 1
OP_GEMM_SILU = 2

STATUS_NAMES = {
    0: "FP8BQ_OK", 1: "FP8BQ_ERR_INVALID_ARG", 2: "FP8BQ_ERR_UNSUPPORTED_SHAPE",
    3: "FP8BQ_ERR_MISALIGNED", 4: "FP8BQ_ERR_WORKSPACE", 5: "FP8BQ_ERR_CUDA",
    6: "FP8BQ_ERR_TIMEOUT", 7: "FP8BQ_ERR_NO_DEVICE", 8: "FP8BQ_ERR_INDEX",
}

_lock = threading.Lock()
_lib = None


class Fp8bqError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {STATUS_NAMES.get(status, status)} ({status_string(status)})")


def lib() -> ctypes.CDLL:
    """Loads libfp8bq.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:  # loaded: no lock on the per-call path
        return _lib
    with _lock:
        if _lib is not None:
            return _lib
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m fp8_block_scaled_09_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        P, I, S = ctypes.c_void_p, ctypes.c_int64, ctypes.c_size_t
        st = ctypes.c_int
        L.fp8bq_quantize_act.argtypes = [P, I, I, P, P, P]
        L.fp8bq_quantize_weight.argtypes = [P, I, I, P, P, P]
        L.fp8bq_gemm.argtypes = [P, P, P, P, I, I, I, P, P, S, P]
        L.fp8bq_linear.argtypes = [P, P, P, I, I, I, P, P, S, P]
        L.fp8bq_gemm_noalloc.argtypes = [P, P, P, P, I, I, I, P, P]
        L.fp8bq_selftest_timeout.argtypes = [ctypes.c_uint32, P]
        L.fp8bq_kv_write_e4m3.argtypes = [P, P, I, I, I, P, P, P, I, I, P]
        L.fp8bq_silu_mul_quantize.argtypes = [P, I, I, P, P, P, P]
        L.fp8bq_gemm_silu_mul_quantize.argtypes = [P, P, P, P, I, I, I, P, P, P, P, S, P]
        L.fp8bq_nvfp4_quantize_weight.argtypes = [P, I, I, P, P, P, P]
        L.fp8bq_nvfp4_gemm_a16.argtypes = [P, P, P, P, I, I, I, P, P]
        L.fp8bq_workspace_size.argtypes = [ctypes.c_int, I, I, I]
        L.fp8bq_workspace_size.restype = S
        L.fp8bq_workspace_init.argtypes = [P, S, P]
        L.fp8bq_last_device_status.argtypes = [P]
        L.fp8bq_status_string.argtypes = [st]
        L.fp8bq_status_string.restype = ctypes.c_char_p
        L.fp8bq_launch_count.argtypes = []
        L.fp8bq_launch_count.restype = ctypes.c_uint64
        L.fp8bq_version.argtypes = []
        L.fp8bq_version.restype = ctypes.c_int
        L.fp8bq_clear_cache.argtypes = []
        L.fp8bq_clear_cache.restype = None
        for name in ("fp8bq_quantize_act", "fp8bq_quantize_weight", "fp8bq_gemm", "fp8bq_linear",
                     "fp8bq_workspace_init", "fp8bq_last_device_status", "fp8bq_gemm_noalloc",
                     "fp8bq_selftest_timeout", "fp8bq_kv_write_e4m3", "fp8bq_silu_mul_quantize",
                     "fp8bq_gemm_silu_mul_quantize",
                     "fp8bq_nvfp4_quantize_weight", "fp8bq_nvfp4_gemm_a16"):
            getattr(L, name).restype = st
        _lib = L
        return L


def status_string(status: int) -> str:
    return lib().fp8bq_status_string(int(status)).decode()


def _check(status: int, what: str) -> None:
    if status != 0:
        raise Fp8bqError(status, what)


_raw_stream = getattr(torch._C, "_cuda_getCurrentRawStream", None)


# Pointers and stream handles are passed as plain Python ints (or None for
# NULL): every argument is declared c_void_p, so ctypes converts them without a
# c_void_p object per argument (a few microseconds per call on the host).
def _stream(t: torch.Tensor) -> int:
    # the current stream's handle without building a torch.cuda.Stream object
    if _raw_stream is not None:
        return _raw_stream(t.get_device())
    return torch.cuda.current_stream(t.device).cuda_stream


def _ptr(t: torch.Tensor | None) -> int | None:
    return t.data_ptr() if t is not None else None


def _codes(t: torch.Tensor) -> torch.Tensor:
    if t.dtype == torch.float8_e4m3fn:
        return t.view(torch.uint8)
    if t.dtype != torch.uint8:
        raise TypeError(f"E4M3 codes must be uint8 or float8_e4m3fn, got {t.dtype}")
    return t


def _need(t: torch.Tensor, dtype: torch.dtype, name: str) -> None:
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous (row-major)")


def workspace_size(op: int, M: int, N: int, K: int) -> int:
    return int(lib().fp8bq_workspace_size(op, M, N, K))


def new_workspace(op: int, M: int, N: int, K: int, device) -> torch.Tensor:
    """A zero-filled (initial-state) workspace for this operation and shape."""
    return torch.zeros(max(workspace_size(op, M, N, K), 256), dtype=torch.uint8, device=device)


def workspace_init(ws: torch.Tensor) -> None:
    _check(lib().fp8bq_workspace_init(_ptr(ws), ws.numel(), _stream(ws)), "fp8bq_workspace_init")


def quantize_act(x: torch.Tensor, q: torch.Tensor | None = None, s: torch.Tensor | None = None):
    _need(x, torch.bfloat16, "x")
    M, K = x.shape
    if q is None:
        q = torch.empty((M, K), dtype=torch.uint8, device=x.device)
    if s is None:
        s = torch.empty((M, K // 128), dtype=torch.float32, device=x.device)
    _check(lib().fp8bq_quantize_act(_ptr(x), M, K, _ptr(q), _ptr(s), _stream(x)),
           "fp8bq_quantize_act")
    return q, s


def quantize_weight(w: torch.Tensor, q: torch.Tensor | None = None, s: torch.Tensor | None = None):
    _need(w, torch.bfloat16, "w")
    N, K = w.shape
    if q is None:
        q = torch.empty((N, K), dtype=torch.uint8, device=w.device)
    if s is None:
        s = torch.empty((N // 128, K // 128), dtype=torch.float32, device=w.device)
    _check(lib().fp8bq_quantize_weight(_ptr(w), N, K, _ptr(q), _ptr(s), _stream(w)),
           "fp8bq_quantize_weight")
    return q, s


def gemm(qa: torch.Tensor, sa: torch.Tensor, qw: torch.Tensor, sw: torch.Tensor,
         out: torch.Tensor | None = None, workspace: torch.Tensor | None = None) -> torch.Tensor:
    qa, qw = _codes(qa), _codes(qw)
    _need(qa, torch.uint8, "qa")
    _need(qw, torch.uint8, "qw")
    _need(sa, torch.float32, "sa")
    _need(sw, torch.float32, "sw")
    M, K = qa.shape
    N = qw.shape[0]
    if out is None:
        out = torch.empty((M, N), dtype=torch.bfloat16, device=qa.device)
    if workspace is None:
        workspace = new_workspace(OP_GEMM, M, N, K, qa.device)
    _check(lib().fp8bq_gemm(_ptr(qa), _ptr(sa), _ptr(qw), _ptr(sw), M, N, K, _ptr(out),
                            _ptr(workspace), workspace.numel(), _stream(qa)), "fp8bq_gemm")
    return out


def gemm_noalloc(qa: torch.Tensor, sa: torch.Tensor, qw: torch.Tensor, sw: torch.Tensor,
                 out: torch.Tensor) -> torch.Tensor:
    """fp8bq_gemm_noalloc: the GEMM with the library's built-in scratch instead of a
    workspace, for callers that cannot allocate device memory.  `out` must be given
    (this call allocates nothing); calls must not overlap on the GPU."""
    qa, qw = _codes(qa), _codes(qw)
    _need(qa, torch.uint8, "qa")
    _need(qw, torch.uint8, "qw")
    _need(sa, torch.float32, "sa")
    _need(sw, torch.float32, "sw")
    _need(out, torch.bfloat16, "out")
    M, K = qa.shape
    N = qw.shape[0]
    _check(lib().fp8bq_gemm_noalloc(_ptr(qa), _ptr(sa), _ptr(qw), _ptr(sw), M, N, K, _ptr(out),
                                    _stream(qa)), "fp8bq_gemm_noalloc")
    return out


def linear(x: torch.Tensor, qw: torch.Tensor, sw: torch.Tensor, out: torch.Tensor | None = None,
           workspace: torch.Tensor | None = None) -> torch.Tensor:
    qw = _codes(qw)
    _need(x, torch.bfloat16, "x")
    _need(qw, torch.uint8, "qw")
    _need(sw, torch.float32, "sw")
    M, K = x.shape
    N = qw.shape[0]
    if out is None:
        out = torch.empty((M, N), dtype=torch.bfloat16, device=x.device)
    if workspace is None:
        workspace = new_workspace(OP_LINEAR, M, N, K, x.device)
    _check(lib().fp8bq_linear(_ptr(x), _ptr(qw), _ptr(sw), M, N, K, _ptr(out), _ptr(workspace),
                              workspace.numel(), _stream(x)), "fp8bq_linear")
    return out


def last_device_status(device=None) -> int:
    """Synchronizes the current stream and returns/clears the device status word."""
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    s = ctypes.c_void_p(torch.cuda.current_stream(dev).cuda_stream)
    return int(lib().fp8bq_last_device_status(s))


def selftest_timeout(limit_us: int = 20000) -> None:
    """Enqueues the bounded-wait self-test (see fp8bq_selftest_timeout)."""
    dev = torch.device("cuda", torch.cuda.current_device())
    _check(lib().fp8bq_selftest_timeout(limit_us,
                                        ctypes.c_void_p(torch.cuda.current_stream(dev).cuda_stream)),
           "fp8bq_selftest_timeout")


def clear_cache() -> None:
    """Empties the library's cache of encoded TMA descriptors."""
    lib().fp8bq_clear_cache()


def launch_count() -> int:
    return int(lib().fp8bq_launch_count())


def kv_write_e4m3(k: torch.Tensor, v: torch.Tensor, loc: torch.Tensor, k_cache: torch.Tensor,
                  v_cache: torch.Tensor) -> None:
    """fp8bq_kv_write_e4m3: k_cache[loc[t], :W] = e4m3(k[t]) and the same for v, with
    unit scales.  k, v: BF16 [T, W] with unit column stride and a shared row stride (e.g.
    column slices of the fused QKV output); loc: int64 [T]; caches: uint8 or
    float8_e4m3fn [num_slots, slot_bytes], slot_bytes >= W.  Out-of-range slots are
    skipped on the device and reported through last_device_status()."""
    for t, name in ((k, "k"), (v, "v")):
        if t.dtype != torch.bfloat16 or t.device.type != "cuda" or t.dim() != 2 or t.stride(1) != 1:
            raise ValueError(f"{name} must be a 2-D CUDA BF16 tensor with unit column stride")
    if k.shape != v.shape or k.stride(0) != v.stride(0):
        raise ValueError("k and v must have the same shape and row stride")
    k_cache, v_cache = _codes(k_cache), _codes(v_cache)
    _need(k_cache, torch.uint8, "k_cache")
    _need(v_cache, torch.uint8, "v_cache")
    _need(loc, torch.int64, "loc")
    if k_cache.shape != v_cache.shape or k_cache.dim() != 2:
        raise ValueError("k_cache and v_cache must be [num_slots, slot_bytes] of the same shape")
    T, W = k.shape
    if loc.shape != (T,):
        raise ValueError("loc must be int64 [T]")
    _check(lib().fp8bq_kv_write_e4m3(_ptr(k), _ptr(v), k.stride(0), T, W, _ptr(loc),
                                     _ptr(k_cache), _ptr(v_cache), k_cache.shape[0],
                                     k_cache.shape[1], _stream(k)), "fp8bq_kv_write_e4m3")


def silu_mul_quantize(gu: torch.Tensor, q: torch.Tensor | None = None, s: torch.Tensor | None = None,
                      h: torch.Tensor | None = None) -> tuple[torch.Tensor, torch.Tensor]:
    """fp8bq_silu_mul_quantize: gu BF16 [M, 2I] (gate, then up) -> the group-128
    quantization of h = BF16(silu(gate) * up): (codes uint8 [M, I], scales FP32
    [M, I/128]).  Pass h (BF16 [M, I]) to also receive h itself."""
    _need(gu, torch.bfloat16, "gu")
    M, two_i = gu.shape
    if two_i % 2:
        raise ValueError("gu must have an even number of columns (gate | up)")
    I = two_i // 2
    if q is None:
        q = torch.empty((M, I), dtype=torch.uint8, device=gu.device)
    if s is None:
        s = torch.empty((M, I // 128 if I % 128 == 0 else 0), dtype=torch.float32, device=gu.device)
    q = _codes(q)
    _need(q, torch.uint8, "q")
    _need(s, torch.float32, "s")
    if h is not None:
        _need(h, torch.bfloat16, "h")
    _check(lib().fp8bq_silu_mul_quantize(_ptr(gu), M, I, _ptr(q), _ptr(s), _ptr(h), _stream(gu)),
           "fp8bq_silu_mul_quantize")
    return q, s


def gemm_silu_mul_quantize(qa: torch.Tensor, sa: torch.Tensor, qw: torch.Tensor, sw: torch.Tensor,
                           q: torch.Tensor | None = None, s: torch.Tensor | None = None,
                           h: torch.Tensor | None = None,
                           workspace: torch.Tensor | None = None) -> tuple[torch.Tensor, torch.Tensor]:
    """fp8bq_gemm_silu_mul_quantize: the gate/up GEMM (fused weight codes qw [2I, K],
    gate rows first) with the SiLU-gated product quantized in its epilogue ->
    (codes uint8 [M, I], scales FP32 [M, I/128]), the same as
    silu_mul_quantize(gemm(qa, sa, qw, sw)).  Pass h (BF16 [M, I]) to also receive h."""
    qa, qw = _codes(qa), _codes(qw)
    _need(qa, torch.uint8, "qa")
    _need(qw, torch.uint8, "qw")
    _need(sa, torch.float32, "sa")
    _need(sw, torch.float32, "sw")
    M, K = qa.shape
    two_i = qw.shape[0]
    if two_i % 2:
        raise ValueError("qw must have an even number of rows (gate | up)")
    I = two_i // 2
    if q is None:
        q = torch.empty((M, I), dtype=torch.uint8, device=qa.device)
    if s is None:
        s = torch.empty((M, I // 128 if I % 128 == 0 else 0), dtype=torch.float32, device=qa.device)
    q = _codes(q)
    _need(q, torch.uint8, "q")
    _need(s, torch.float32, "s")
    if h is not None:
        _need(h, torch.bfloat16, "h")
    if workspace is None:
        workspace = new_workspace(OP_GEMM_SILU, M, two_i, K, qa.device)
    _check(lib().fp8bq_gemm_silu_mul_quantize(_ptr(qa), _ptr(sa), _ptr(qw), _ptr(sw), M, I, K,
                                              _ptr(q), _ptr(s), _ptr(h), _ptr(workspace),
                                              workspace.numel(), _stream(qa)),
           "fp8bq_gemm_silu_mul_quantize")
    return q, s


def nvfp4_quantize_weight(w: torch.Tensor) -> tuple[torch.Tensor, torch.Tensor, torch.Tensor]:
    """fp8bq_nvfp4_quantize_weight: BF16 W [N, K] -> (packed E2M1 uint8 [N, K/2], E4M3
    block scales uint8 [N, K/16], global scale FP32 [1]), plain min-max."""
    _need(w, torch.bfloat16, "w")
    N, K = w.shape
    packed = torch.empty((N, K // 2), dtype=torch.uint8, device=w.device)
    sb = torch.empty((N, K // 16), dtype=torch.uint8, device=w.device)
    g = torch.empty(1, dtype=torch.float32, device=w.device)
    _check(lib().fp8bq_nvfp4_quantize_weight(_ptr(w), N, K, _ptr(packed), _ptr(sb), _ptr(g),
                                             _stream(w)), "fp8bq_nvfp4_quantize_weight")
    return packed, sb, g


def nvfp4_gemm_a16(x: torch.Tensor, packed: torch.Tensor, sb: torch.Tensor, g: torch.Tensor,
                   out: torch.Tensor | None = None) -> torch.Tensor:
    """fp8bq_nvfp4_gemm_a16: BF16 X [M, K] times the NVFP4 weight (packed [N, K/2], sb
    [N, K/16], g FP32 [1]) transposed -> BF16 [M, N]."""
    _need(x, torch.bfloat16, "x")
    _need(packed, torch.uint8, "packed")
    sb = _codes(sb)
    _need(sb, torch.uint8, "sb")
    _need(g, torch.float32, "g")
    M, K = x.shape
    N = packed.shape[0]
    if out is None:
        out = torch.empty((M, N), dtype=torch.bfloat16, device=x.device)
    _need(out, torch.bfloat16, "out")
    _check(lib().fp8bq_nvfp4_gemm_a16(_ptr(x), _ptr(packed), _ptr(sb), _ptr(g), M, N, K, _ptr(out),
                                      _stream(x)), "fp8bq_nvfp4_gemm_a16")
    return out
