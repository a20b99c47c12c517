"""ctypes wrappers around the C oracle (``dsqref.c``).

TEST INFRASTRUCTURE ONLY.  Every function takes and returns numpy arrays; the
arithmetic is entirely in the C file, single-threaded.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

Q8_0 = 8
Q4_K = 12

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "dsqref.c")
_HDR = os.path.join(_HERE, "dsqref.h")
_LIB = os.path.join(_HERE, "libdsqref.so")
_CFLAGS = ["-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math", "-fPIC",
           "-shared", "-Wall", "-Wextra", "-Werror"]

_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile ``libdsqref.so`` next to the sources (plain gcc, no GPU)."""
    newest = max(os.path.getmtime(_SRC), os.path.getmtime(_HDR))
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < newest:
        tmp = _LIB + f".{os.getpid()}.tmp"
        subprocess.check_call(["gcc", *_CFLAGS, "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def lib() -> ctypes.CDLL:
    """The loaded oracle.  DSQREF_LIB may name another build of the same
    source (the mutation test points it at copies with planted mistakes)."""
    global _lib
    with _lock:
        if _lib is None:
            _lib = ctypes.CDLL(os.environ.get("DSQREF_LIB") or build())
            _declare(_lib)
    return _lib


_P = ctypes.c_void_p
_I64 = ctypes.c_int64
_INT = ctypes.c_int


def _declare(L):
    sig = {
        "dsqref_f32_to_f16": (ctypes.c_uint16, [ctypes.c_float]),
        "dsqref_f16_to_f32": (ctypes.c_float, [ctypes.c_uint16]),
        "dsqref_f32_to_bf16": (ctypes.c_uint16, [ctypes.c_float]),
        "dsqref_bf16_to_f32": (ctypes.c_float, [ctypes.c_uint16]),
        "dsqref_row_bytes": (_I64, [_INT, _I64]),
        "dsqref_quantize_q8_0": (None, [_P, _I64, _I64, _P]),
        "dsqref_dequantize_q8_0": (None, [_P, _I64, _I64, _P]),
        "dsqref_q4k_get_scale_min": (None, [_P, _INT, _P, _P]),
        "dsqref_q4k_set_scale_min": (None, [_P, _INT, _INT, _INT]),
        "dsqref_quantize_q4_k": (None, [_P, _I64, _I64, _P]),
        "dsqref_dequantize_q4_k": (None, [_P, _I64, _I64, _P]),
        "dsqref_dequantize": (None, [_INT, _P, _I64, _I64, _P]),
        "dsqref_quantize_act_q8": (None, [_P, _I64, _I64, _P, _P, _P]),
        "dsqref_block_sums": (None, [_INT, _P, _I64, _I64, _P, _P]),
        "dsqref_gemv": (None, [_INT, _P, _I64, _I64, _P, _P, _P, _P, _P]),
        "dsqref_gemv_dequant_f64": (None, [_INT, _P, _I64, _I64, _P, _P, _P]),
        "dsqref_prefill_f64": (None, [_INT, _P, _I64, _I64, _P, _I64, _P]),
        "dsqref_row_shift": (_INT, [_P, _I64]),
        "dsqref_prefill_rounded": (None, [_INT, _INT, _P, _I64, _I64, _P, _I64, _P]),
        "dsqref_prefill_operands": (None, [_INT, _INT, _P, _I64, _I64, _P, _I64, _P, _P, _P]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(L, name)
        fn.restype = res
        fn.argtypes = args


def _ptr(a: np.ndarray) -> int:
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


# ---------------------------------------------------------------- scalars ---
def f32_to_f16(x: float) -> int:
    return lib().dsqref_f32_to_f16(x)


def f16_to_f32(h: int) -> float:
    return lib().dsqref_f16_to_f32(h)


def f32_to_bf16(x: float) -> int:
    return lib().dsqref_f32_to_bf16(x)


def bf16_to_f32(h: int) -> float:
    return lib().dsqref_bf16_to_f32(h)


def row_bytes(qtype: int, K: int) -> int:
    return lib().dsqref_row_bytes(qtype, K)


# ---------------------------------------------------------------- formats ---
def quantize(qtype: int, x: np.ndarray) -> np.ndarray:
    """Quantize fp32 rows [N, K] to packed bytes [N, row_bytes]."""
    x = _c(x, np.float32)
    N, K = x.shape
    rb = row_bytes(qtype, K)
    if rb == 0:
        raise ValueError(f"K={K} does not fit type {qtype}")
    out = np.zeros((N, rb), np.uint8)
    fn = lib().dsqref_quantize_q8_0 if qtype == Q8_0 else lib().dsqref_quantize_q4_k
    fn(_ptr(x), N, K, _ptr(out))
    return out


def dequantize(qtype: int, w: np.ndarray, K: int) -> np.ndarray:
    w = _c(w, np.uint8)
    N = w.shape[0]
    out = np.zeros((N, K), np.float32)
    lib().dsqref_dequantize(qtype, _ptr(w), N, K, _ptr(out))
    return out


def q4k_get_scale_min(scales12: np.ndarray, j: int) -> tuple[int, int]:
    s = _c(scales12, np.uint8)
    sc = ctypes.c_int()
    m = ctypes.c_int()
    lib().dsqref_q4k_get_scale_min(_ptr(s), j, ctypes.addressof(sc), ctypes.addressof(m))
    return sc.value, m.value


def q4k_set_scale_min(scales12: np.ndarray, j: int, sc: int, m: int) -> None:
    assert scales12.dtype == np.uint8 and scales12.flags["C_CONTIGUOUS"]
    lib().dsqref_q4k_set_scale_min(_ptr(scales12), j, sc, m)


def quantize_act_q8(x: np.ndarray):
    """x [M, K] fp32 -> (xq int8 [M, K], xd f32 [M, K/32], xs i32 [M, K/32])."""
    x = _c(x, np.float32)
    if x.ndim == 1:
        x = x[None, :]
    M, K = x.shape
    xq = np.zeros((M, K), np.int8)
    xd = np.zeros((M, K // 32), np.float32)
    xs = np.zeros((M, K // 32), np.int32)
    lib().dsqref_quantize_act_q8(_ptr(x), M, K, _ptr(xq), _ptr(xd), _ptr(xs))
    return xq, xd, xs


def block_sums(qtype: int, w: np.ndarray, K: int, xq: np.ndarray) -> np.ndarray:
    w = _c(w, np.uint8)
    xq = _c(xq, np.int8).reshape(-1)
    N = w.shape[0]
    out = np.zeros((N, K // 32), np.int32)
    lib().dsqref_block_sums(qtype, _ptr(w), N, K, _ptr(xq), _ptr(out))
    return out


def gemv(qtype: int, w: np.ndarray, K: int, xq, xd, xs=None):
    """Integer-form GEMV in fp64: returns (y, absum)."""
    w = _c(w, np.uint8)
    xq = _c(xq, np.int8).reshape(-1)
    xd = _c(xd, np.float32).reshape(-1)
    xs = _c(xs if xs is not None else np.zeros(K // 32, np.int32), np.int32).reshape(-1)
    N = w.shape[0]
    y = np.zeros(N, np.float64)
    a = np.zeros(N, np.float64)
    lib().dsqref_gemv(qtype, _ptr(w), N, K, _ptr(xq), _ptr(xd), _ptr(xs), _ptr(y), _ptr(a))
    return y, a


def gemv_dequant_f64(qtype: int, w: np.ndarray, K: int, xq, xd) -> np.ndarray:
    w = _c(w, np.uint8)
    xq = _c(xq, np.int8).reshape(-1)
    xd = _c(xd, np.float32).reshape(-1)
    N = w.shape[0]
    y = np.zeros(N, np.float64)
    lib().dsqref_gemv_dequant_f64(qtype, _ptr(w), N, K, _ptr(xq), _ptr(xd), _ptr(y))
    return y


def prefill_f64(qtype: int, w: np.ndarray, K: int, x: np.ndarray) -> np.ndarray:
    w = _c(w, np.uint8)
    x = _c(x, np.float32)
    M = x.shape[0]
    N = w.shape[0]
    y = np.zeros((M, N), np.float64)
    lib().dsqref_prefill_f64(qtype, _ptr(w), N, K, _ptr(x), M, _ptr(y))
    return y


def row_shift(row: np.ndarray) -> int:
    row = _c(row, np.float32).reshape(-1)
    return lib().dsqref_row_shift(_ptr(row), row.size)


def prefill_rounded(qtype: int, w: np.ndarray, K: int, x: np.ndarray, op16: str = "f16") -> np.ndarray:
    w = _c(w, np.uint8)
    x = _c(x, np.float32)
    M = x.shape[0]
    N = w.shape[0]
    y = np.zeros((M, N), np.float64)
    lib().dsqref_prefill_rounded(qtype, 0 if op16 == "f16" else 1, _ptr(w), N, K,
                                 _ptr(x), M, _ptr(y))
    return y


def prefill_operands(qtype: int, w: np.ndarray, K: int, x: np.ndarray, op16: str = "f16"):
    """(x16 bits [M, K], shift [M], w16 bits [N, K]) as the rounded reference forms them."""
    w = _c(w, np.uint8)
    x = _c(x, np.float32)
    M, N = x.shape[0], w.shape[0]
    x16 = np.zeros((M, K), np.uint16)
    sh = np.zeros(M, np.int32)
    w16 = np.zeros((N, K), np.uint16)
    lib().dsqref_prefill_operands(qtype, 0 if op16 == "f16" else 1, _ptr(w), N, K, _ptr(x), M,
                                  _ptr(x16), _ptr(sh), _ptr(w16))
    return x16, sh, w16
