"""libdsq Python binding: block-quantized projections on B200 (sm_100a).

Thin ctypes marshalling over the C ABI in ``include/dsq.h``; the functions
carry the C names and argument order.  Tensor arguments are torch CUDA
tensors (or raw device addresses as ints); outputs are caller-allocated.
Every step of the computation runs in libdsq's CUDA kernels -- there is no
Python or CPU fallback: if ``libdsq.so`` is missing or the call fails, a
``DsqError`` is raised.
"""
from __future__ import annotations

import ctypes
import os
import threading

__all__ = [
    "DSQ_Q8_0", "DSQ_Q4_K", "DsqError", "lib", "dsq_row_bytes", "dsq_quantize_act_q8",
    "dsq_gemv_q8_0", "dsq_gemv_q4_k", "dsq_gemv_paired", "dsq_gemv_grouped", "dsq_gemv_f32",
    "dsq_gemv_paired_f32", "dsq_gemv_grouped_f32", "dsq_gemv_tokens", "dsq_gemm_prefill",
    "dsq_gemm_prefill_grouped", "dsq_prefill_grouped_workspace_bytes",
    "dsq_prefill_workspace_bytes", "dsq_gemm_prefill_noalloc", "dsq_quantize_weights", "dsq_device_status", "dsq_last_error",
    "dsq_version", "dsq_launch_count", "dsq_test_block_sums", "dsq_test_set_wait_limit_ns",
    "dsq_test_prefill_operands", "dsq_test_block_sums_tokens", "LIB_PATH",
]

DSQ_Q8_0 = 8
DSQ_Q4_K = 12

STATUS = {0: "DSQ_OK", 1: "DSQ_ERR_INVALID_ARG", 2: "DSQ_ERR_ALIGNMENT", 3: "DSQ_ERR_SHAPE",
          4: "DSQ_ERR_UNSUPPORTED_DEVICE", 5: "DSQ_ERR_WORKSPACE", 6: "DSQ_ERR_LAUNCH",
          7: "DSQ_ERR_TIMEOUT", 8: "DSQ_ERR_CUDA", 9: "DSQ_ERR_RANGE"}

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libdsq.so")

_P = ctypes.c_void_p
_I64 = ctypes.c_int64
_INT = ctypes.c_int
_SZ = ctypes.c_size_t

# name -> (restype, argtypes); the order follows include/dsq.h and dsq_test.h
_SIGS = {
    "dsq_row_bytes": (_SZ, [_INT, _I64]),
    "dsq_quantize_act_q8": (_INT, [_P, _I64, _I64, _P, _P, _P, _P]),
    "dsq_gemv_q8_0": (_INT, [_P, _I64, _I64, _P, _P, _P, _P]),
    "dsq_gemv_q4_k": (_INT, [_P, _I64, _I64, _P, _P, _P, _P, _P]),
    "dsq_gemv_paired": (_INT, [_INT, _P, _I64, _P, _I64, _I64, _P, _P, _P, _P, _P, _P]),
    "dsq_gemv_grouped": (_INT, [_INT, _P, _I64, _I64, _I64, _P, _P, _P, _P, _P]),
    "dsq_gemv_f32": (_INT, [_INT, _P, _I64, _I64, _P, _P, _P]),
    "dsq_gemv_paired_f32": (_INT, [_INT, _P, _I64, _P, _I64, _I64, _P, _P, _P, _P]),
    "dsq_gemv_grouped_f32": (_INT, [_INT, _P, _I64, _I64, _I64, _P, _P, _P]),
    "dsq_gemv_tokens": (_INT, [_INT, _P, _I64, _P, _I64, _I64, _I64, _P, _P, _P, _P, _P, _P]),
    "dsq_gemm_prefill": (_INT, [_INT, _P, _I64, _I64, _P, _I64, _P, _P, _SZ, _P]),
    "dsq_prefill_workspace_bytes": (_SZ, [_INT, _I64, _I64, _I64]),
    "dsq_gemm_prefill_grouped": (_INT, [_INT, _I64, _P, _P, _I64, _P, _I64, _P, _P, _SZ, _P]),
    "dsq_prefill_grouped_workspace_bytes": (_SZ, [_INT, _I64, _P, _I64, _I64]),
    "dsq_gemm_prefill_noalloc": (_INT, [_INT, _P, _I64, _I64, _P, _I64, _P, _P]),
    "dsq_quantize_weights": (_INT, [_INT, _P, _I64, _I64, _P, _P]),
    "dsq_device_status": (_INT, [_P]),
    "dsq_last_error": (ctypes.c_char_p, []),
    "dsq_version": (ctypes.c_char_p, []),
    "dsq_launch_count": (ctypes.c_uint64, []),
    "dsq_test_block_sums": (_INT, [_INT, _P, _I64, _I64, _P, _P, _P, _P, _P, _P]),
    "dsq_test_set_wait_limit_ns": (_INT, [ctypes.c_uint64]),
    "dsq_test_prefill_operands": (_INT, [_INT, _P, _I64, _I64, _P, _I64, _P, _P, _P, _P]),
    "dsq_test_block_sums_tokens": (_INT, [_INT, _P, _I64, _I64, _I64, _P, _P, _P, _P, _P, _P]),
}

_lock = threading.Lock()
_lib = None


class DsqError(RuntimeError):
    def __init__(self, fn: str, status: int, msg: str):
        super().__init__(f"{fn}: {STATUS.get(status, status)}: {msg}")
        self.status = status


def lib() -> ctypes.CDLL:
    """The loaded libdsq.so (built in-tree by ``python -m block_quantized_dsq_b200.build``)."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise DsqError("lib", 8, f"{LIB_PATH} is not built; run "
                               "`python -m block_quantized_dsq_b200.build` (there is no fallback)")
            L = ctypes.CDLL(LIB_PATH)
            for name, (res, args) in _SIGS.items():
                fn = getattr(L, name)
                fn.restype = res
                fn.argtypes = args
            _lib = L
    return _lib


def _ptr(t) -> int | None:
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream) -> int | None:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(fn: str, rc: int) -> None:
    if rc != 0:
        raise DsqError(fn, rc, lib().dsq_last_error().decode())


# ------------------------------------------------------------------ API ----
def dsq_row_bytes(qtype: int, K: int) -> int:
    return lib().dsq_row_bytes(qtype, K)


def dsq_quantize_act_q8(x, M, K, xq, xd, xs=None, stream=None):
    _check("dsq_quantize_act_q8",
           lib().dsq_quantize_act_q8(_ptr(x), M, K, _ptr(xq), _ptr(xd), _ptr(xs), _stream(stream)))


def dsq_gemv_q8_0(w, N, K, xq, xd, y, stream=None):
    _check("dsq_gemv_q8_0", lib().dsq_gemv_q8_0(_ptr(w), N, K, _ptr(xq), _ptr(xd), _ptr(y), _stream(stream)))


def dsq_gemv_q4_k(w, N, K, xq, xd, xs, y, stream=None):
    _check("dsq_gemv_q4_k",
           lib().dsq_gemv_q4_k(_ptr(w), N, K, _ptr(xq), _ptr(xd), _ptr(xs), _ptr(y), _stream(stream)))


def dsq_gemv_paired(qtype, w0, N0, w1, N1, K, xq, xd, xs, y0, y1, stream=None):
    _check("dsq_gemv_paired",
           lib().dsq_gemv_paired(qtype, _ptr(w0), N0, _ptr(w1), N1, K, _ptr(xq), _ptr(xd), _ptr(xs),
                                 _ptr(y0), _ptr(y1), _stream(stream)))


def dsq_gemv_grouped(qtype, w, G, N, K, xq, xd, xs, y, stream=None):
    _check("dsq_gemv_grouped",
           lib().dsq_gemv_grouped(qtype, _ptr(w), G, N, K, _ptr(xq), _ptr(xd), _ptr(xs), _ptr(y),
                                  _stream(stream)))


def dsq_gemv_f32(qtype, w, N, K, x, y, stream=None):
    """Quantize the fp32 activation and run the GEMV in one launch."""
    _check("dsq_gemv_f32", lib().dsq_gemv_f32(qtype, _ptr(w), N, K, _ptr(x), _ptr(y), _stream(stream)))


def dsq_gemv_paired_f32(qtype, w0, N0, w1, N1, K, x, y0, y1, stream=None):
    _check("dsq_gemv_paired_f32",
           lib().dsq_gemv_paired_f32(qtype, _ptr(w0), N0, _ptr(w1), N1, K, _ptr(x), _ptr(y0), _ptr(y1),
                                     _stream(stream)))


def dsq_gemv_grouped_f32(qtype, w, G, N, K, x, y, stream=None):
    _check("dsq_gemv_grouped_f32",
           lib().dsq_gemv_grouped_f32(qtype, _ptr(w), G, N, K, _ptr(x), _ptr(y), _stream(stream)))


def dsq_gemv_tokens(qtype, w0, N0, w1, N1, K, M, xq, xd, xs, y0, y1, stream=None):
    """M = 1..8 prequantized tokens against one weight (N1 = 0) or two that
    share the input; every weight byte is read once for all M tokens."""
    _check("dsq_gemv_tokens",
           lib().dsq_gemv_tokens(qtype, _ptr(w0), N0, _ptr(w1), N1, K, M, _ptr(xq), _ptr(xd), _ptr(xs),
                                 _ptr(y0), _ptr(y1), _stream(stream)))


def dsq_gemm_prefill(qtype, w, N, K, x, M, y, workspace, workspace_bytes, stream=None):
    _check("dsq_gemm_prefill",
           lib().dsq_gemm_prefill(qtype, _ptr(w), N, K, _ptr(x), M, _ptr(y), _ptr(workspace),
                                  workspace_bytes, _stream(stream)))


def dsq_prefill_workspace_bytes(qtype: int, N: int, K: int, M: int) -> int:
    return lib().dsq_prefill_workspace_bytes(qtype, N, K, M)


def _host_array(ctype, values):
    return (ctype * len(values))(*values)


def dsq_gemm_prefill_grouped(qtype, ws, Ns, K, x, M, ys, workspace, workspace_bytes, stream=None):
    """G weights (lists ws, Ns, ys of equal length) sharing one activation X."""
    G = len(ws)
    _check("dsq_gemm_prefill_grouped",
           lib().dsq_gemm_prefill_grouped(qtype, G, _host_array(ctypes.c_void_p, [_ptr(w) for w in ws]),
                                          _host_array(ctypes.c_int64, list(Ns)), K, _ptr(x), M,
                                          _host_array(ctypes.c_void_p, [_ptr(y) for y in ys]), _ptr(workspace),
                                          workspace_bytes, _stream(stream)))


def dsq_prefill_grouped_workspace_bytes(qtype: int, Ns, K: int, M: int) -> int:
    return lib().dsq_prefill_grouped_workspace_bytes(qtype, len(Ns), _host_array(ctypes.c_int64, list(Ns)), K, M)


DSQ_PREFILL_NOALLOC_SCRATCH_BYTES = 32 * 1024 * 1024


def dsq_gemm_prefill_noalloc(qtype, w, N, K, x, M, y, stream=None):
    """dsq_gemm_prefill for callers that cannot allocate device memory at
    call time: scratch comes from a fixed 32 MiB array inside the library.
    The first call on a device does a one-time set-up (make it before any
    stream capture); calls that may overlap on the GPU race on the shared
    scratch and must be serialized by the caller."""
    _check("dsq_gemm_prefill_noalloc",
           lib().dsq_gemm_prefill_noalloc(qtype, _ptr(w), N, K, _ptr(x), M, _ptr(y), _stream(stream)))


def dsq_quantize_weights(qtype, x, N, K, w, stream=None):
    _check("dsq_quantize_weights", lib().dsq_quantize_weights(qtype, _ptr(x), N, K, _ptr(w), _stream(stream)))


def dsq_device_status(stream=None) -> int:
    """Synchronizes the stream; returns (and clears) the device status code."""
    return lib().dsq_device_status(_stream(stream))


def dsq_last_error() -> str:
    return lib().dsq_last_error().decode()


def dsq_version() -> str:
    return lib().dsq_version().decode()


def dsq_launch_count() -> int:
    return lib().dsq_launch_count()


# -------------------------------------------------------------- test-only --
def dsq_test_block_sums(qtype, w, N, K, xq, xd, xs, y, isum, stream=None):
    _check("dsq_test_block_sums",
           lib().dsq_test_block_sums(qtype, _ptr(w), N, K, _ptr(xq), _ptr(xd), _ptr(xs), _ptr(y), _ptr(isum),
                                     _stream(stream)))


def dsq_test_set_wait_limit_ns(ns: int) -> None:
    lib().dsq_test_set_wait_limit_ns(ns)


def dsq_test_prefill_operands(qtype, w, N, K, x, M, x16, shift, w16, stream=None):
    _check("dsq_test_prefill_operands",
           lib().dsq_test_prefill_operands(qtype, _ptr(w), N, K, _ptr(x), M, _ptr(x16), _ptr(shift), _ptr(w16),
                                           _stream(stream)))


def dsq_test_block_sums_tokens(qtype, w, N, K, M, xq, xd, xs, y, isum, stream=None):
    _check("dsq_test_block_sums_tokens",
           lib().dsq_test_block_sums_tokens(qtype, _ptr(w), N, K, M, _ptr(xq), _ptr(xd), _ptr(xs), _ptr(y),
                                            _ptr(isum), _stream(stream)))
