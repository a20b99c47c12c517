"""The C-ABI library builds, loads and exports every declared entry point;
host-side argument checks return the documented status and launch nothing
(no GPU needed: each case fails before any CUDA call)."""
import ctypes
import os
import re

import pytest

from conftest import ROOT

HEADERS = [os.path.join(ROOT, "include", "dsq.h"), os.path.join(ROOT, "include", "dsq_test.h")]


def declared_functions():
    names = []
    for h in HEADERS:
        text = open(h).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        names += re.findall(r"\b(dsq_\w+)\s*\(", text)
    return sorted(set(names))


@pytest.fixture(scope="module")
def dsq():
    from block_quantized_dsq_b200 import build
    build.build()
    import block_quantized_dsq_b200 as dsq
    return dsq


def test_every_declared_symbol_is_exported(dsq):
    names = declared_functions()
    assert len(names) >= 16
    raw = ctypes.CDLL(dsq.LIB_PATH)
    missing = [n for n in names if not hasattr(raw, n)]
    assert not missing, missing
    # the binding exposes the same names
    assert not [n for n in names if not hasattr(dsq, n)]


def test_row_bytes_and_version(dsq):
    assert dsq.dsq_row_bytes(dsq.DSQ_Q8_0, 4096) == 4352
    assert dsq.dsq_row_bytes(dsq.DSQ_Q4_K, 4096) == 2304
    assert dsq.dsq_row_bytes(dsq.DSQ_Q4_K, 4000) == 0
    assert dsq.dsq_row_bytes(dsq.DSQ_Q8_0, 33) == 0
    assert dsq.dsq_row_bytes(7, 4096) == 0
    assert "sm_100a" in dsq.dsq_version()


def _status(fn, *args):
    from block_quantized_dsq_b200 import DsqError
    try:
        fn(*args)
    except DsqError as e:
        return e.status
    return 0


A16 = 1 << 20        # a fake, 16-byte aligned device address (never dereferenced)


def test_host_side_validation(dsq):
    L = dsq.lib()
    before = dsq.dsq_launch_count()
    # unsupported type
    assert L.dsq_gemv_paired(7, A16, 8, A16, 8, 256, A16, A16, A16, A16, A16, None) == 1
    # K not a multiple of the block size
    assert L.dsq_gemv_q8_0(A16, 8, 48, A16, A16, A16, None) == 3
    assert L.dsq_gemv_q4_k(A16, 8, 288, A16, A16, A16, A16, None) == 3
    assert L.dsq_quantize_act_q8(A16, 1, 40, A16, A16, A16, None) == 3
    assert L.dsq_gemm_prefill(8, A16, 128, 96, A16, 4, A16, A16, 1 << 30, None) == 3
    # null pointers
    assert L.dsq_gemv_q8_0(None, 8, 256, A16, A16, A16, None) == 1
    assert L.dsq_gemv_q4_k(A16, 8, 256, A16, A16, None, A16, None) == 1   # Q4_K needs xs
    assert L.dsq_quantize_act_q8(None, 1, 32, A16, A16, A16, None) == 1
    # misaligned pointers
    assert L.dsq_gemv_q8_0(A16 + 8, 8, 256, A16, A16, A16, None) == 2
    assert L.dsq_gemv_q8_0(A16, 8, 256, A16 + 4, A16, A16, None) == 2
    assert L.dsq_quantize_act_q8(A16 + 4, 1, 32, A16, A16, A16, None) == 2
    assert L.dsq_gemm_prefill(12, A16 + 2, 128, 256, A16, 4, A16, A16, 1 << 30, None) == 2
    # negative and out-of-range sizes
    assert L.dsq_gemv_q8_0(A16, -1, 256, A16, A16, A16, None) == 1
    assert L.dsq_gemv_grouped(8, A16, -2, 8, 256, A16, A16, A16, A16, None) == 1
    assert L.dsq_gemm_prefill(8, A16, 0, 256, A16, 4, A16, A16, 1 << 30, None) == 1
    assert L.dsq_gemm_prefill(8, A16, 128, 256, A16, 0, A16, A16, 1 << 30, None) == 1
    assert L.dsq_gemv_q8_0(A16, 8, 1 << 21, A16, A16, A16, None) == 3
    # empty problems are a no-op that touches nothing (no device needed)
    assert L.dsq_gemv_q8_0(None, 0, 256, None, None, None, None) == 0
    assert L.dsq_gemv_paired(8, None, 0, None, 0, 256, None, None, None, None, None, None) == 0
    assert L.dsq_quantize_act_q8(None, 0, 32, None, None, None, None) == 0
    # the fp32-activation (fused) forms
    assert L.dsq_gemv_f32(7, A16, 8, 256, A16, A16, None) == 1                 # unsupported type
    assert L.dsq_gemv_f32(8, A16, 8, 96, A16, A16, None) == 3                  # K % 256 != 0: no fused form
    assert L.dsq_gemv_f32(8, A16, 8, 256, A16 + 4, A16, None) == 2             # misaligned x
    assert L.dsq_gemv_f32(8, A16, 8, 256, None, A16, None) == 1                # null x
    assert L.dsq_gemv_grouped_f32(8, A16, 16, 8, 8192, A16, A16, None) == 3    # activations beyond 64 KB
    assert L.dsq_gemv_grouped_f32(8, A16, -1, 8, 256, A16, A16, None) == 1
    assert L.dsq_gemv_paired_f32(12, A16, 8, A16, 8, 256, A16 + 8, A16, A16, None) == 2
    assert L.dsq_gemv_paired_f32(8, None, 0, None, 0, 256, None, None, None, None) == 0   # empty: no-op
    # the multi-token GEMV: token count, activation area, K, pointers
    assert L.dsq_gemv_tokens(8, A16, 8, None, 0, 4096, 9, A16, A16, None, A16, None, None) == 3
    assert L.dsq_gemv_tokens(8, A16, 8, None, 0, 4096, 0, A16, A16, None, A16, None, None) == 3
    assert L.dsq_gemv_tokens(8, A16, 8, None, 0, 8192, 8, A16, A16, None, A16, None, None) == 3
    assert L.dsq_gemv_tokens(12, A16, 8, None, 0, 288, 2, A16, A16, A16, A16, None, None) == 3
    assert L.dsq_gemv_tokens(12, A16, 8, None, 0, 256, 2, A16, A16, None, A16, None, None) == 1
    assert L.dsq_gemv_tokens(8, A16 + 8, 8, None, 0, 256, 2, A16, A16, None, A16, None, None) == 2
    assert L.dsq_gemv_tokens(8, A16, 8, A16, 4, 256, 2, A16, A16, None, A16, None, None) == 1   # null y1
    assert L.dsq_gemv_tokens(8, None, 0, None, 0, 256, 2, None, None, None, None, None, None) == 0
    # the grouped prefill: weight count, sizes, host arrays
    arr_p = (ctypes.c_void_p * 5)(*([A16] * 5))
    arr_n = (ctypes.c_int64 * 5)(*([128] * 5))
    assert L.dsq_gemm_prefill_grouped(8, 0, arr_p, arr_n, 256, A16, 4, arr_p, A16, 1 << 30, None) == 1
    assert L.dsq_gemm_prefill_grouped(8, 5, arr_p, arr_n, 256, A16, 4, arr_p, A16, 1 << 30, None) == 1
    assert L.dsq_gemm_prefill_grouped(8, 2, None, arr_n, 256, A16, 4, arr_p, A16, 1 << 30, None) == 1
    assert L.dsq_gemm_prefill_grouped(8, 2, arr_p, arr_n, 96, A16, 4, arr_p, A16, 1 << 30, None) == 3
    bad_n = (ctypes.c_int64 * 2)(128, 0)
    assert L.dsq_gemm_prefill_grouped(8, 2, arr_p, bad_n, 256, A16, 4, arr_p, A16, 1 << 30, None) == 1
    assert L.dsq_prefill_grouped_workspace_bytes(8, 2, bad_n, 256, 4) == 0
    assert L.dsq_prefill_grouped_workspace_bytes(8, 5, arr_n, 256, 4) == 0
    # the allocation-free prefill names a bad argument before it looks at the
    # scratch size, even for a problem too large for its scratch
    big_m = 8192                                    # 8192 x 8192 x 2 B of fp16 activations > 32 MiB
    assert L.dsq_gemm_prefill_noalloc(8, None, 256, 8192, A16, big_m, A16, None) == 1
    assert L.dsq_gemm_prefill_noalloc(8, A16, 256, 8192, A16 + 4, big_m, A16, None) == 2
    assert L.dsq_gemm_prefill_noalloc(8, A16, 256, 8192, A16, big_m, None, None) == 1
    assert L.dsq_gemm_prefill_noalloc(8, A16, 256, 96, A16, 4, A16, None) == 3
    assert L.dsq_gemm_prefill_noalloc(7, A16, 256, 256, A16, 4, A16, None) == 1
    # nothing was launched
    assert dsq.dsq_launch_count() == before
    assert "multiple" in dsq.dsq_last_error() or dsq.dsq_last_error()


def test_binding_raises_with_status(dsq):
    from block_quantized_dsq_b200 import DsqError
    with pytest.raises(DsqError) as ei:
        dsq.dsq_gemv_q8_0(A16, 8, 48, A16, A16, A16, stream=0)
    assert ei.value.status == 3 and "multiple of 32" in str(ei.value)
