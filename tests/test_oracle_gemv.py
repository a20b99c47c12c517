"""Pins for the oracle's block dots and decode GEMV (no GPU).

The integer form the method uses (per-block int32 dots, then scaling) is
checked against: the plain fp64 definition (dequantize, then dot), numpy
float64/int64 matmuls, and closed forms on hand-built blocks.
"""
import numpy as np
import pytest

import oracle
from block_quantized_dsq_b200 import synth


def _q8_0_bytes(d_f16: int, q: np.ndarray) -> np.ndarray:
    """Hand-assembled Q8_0 rows: q [N, K] int codes, one shared fp16 scale."""
    N, K = q.shape
    out = np.zeros((N, K // 32, 34), np.uint8)
    out[:, :, 0] = d_f16 & 0xFF
    out[:, :, 1] = d_f16 >> 8
    out[:, :, 2:] = q.reshape(N, K // 32, 32).astype(np.int8).view(np.uint8)
    return out.reshape(N, -1)


def _q4k_unit_rows(N, K, q=None):
    """Hand-assembled Q4_K rows with d = 1, dmin = 0, every sc = 1, m = 0."""
    nsb = K // 256
    out = np.zeros((N, nsb, 144), np.uint8)
    out[:, :, 0:2] = np.array([0x3C00], np.uint16).view(np.uint8)   # d = 1.0
    out[:, :, 4:8] = 0x01       # sc_0..3 = 1
    out[:, :, 8:12] = 0x00      # m_0..3 = 0
    out[:, :, 12:16] = 0x01     # sc_4..7 low nibble 1, m_4..7 = 0
    if q is None:
        out[:, :, 16:] = 0x11   # every code 1
    else:
        qq = q.reshape(N, nsb, 8, 32)
        for c in range(4):
            out[:, :, 16 + 32 * c:16 + 32 * c + 32] = (qq[:, :, 2 * c] | (qq[:, :, 2 * c + 1] << 4)).astype(np.uint8)
    return out.reshape(N, -1)


@pytest.mark.parametrize("qtype", [8, 12])
@pytest.mark.parametrize("K", [256, 512])
def test_integer_form_equals_plain_definition(ref, qtype, K):
    N = 9
    w = ref.quantize(qtype, synth.weights(11, N, K))
    x = synth.activations(12, 1, K)
    xq, xd, xs = ref.quantize_act_q8(x)
    y, absum = ref.gemv(qtype, w, K, xq, xd, xs)
    y_plain = ref.gemv_dequant_f64(qtype, w, K, xq, xd)
    assert np.all(np.abs(y - y_plain) <= 1e-13 * absum)
    assert np.all(absum > 0)


@pytest.mark.parametrize("qtype", [8, 12])
def test_plain_definition_matches_numpy_matmul(ref, qtype):
    N, K = 13, 512
    w = ref.quantize(qtype, synth.weights(13, N, K))
    xq, xd, _ = ref.quantize_act_q8(synth.activations(14, 1, K))
    wf = ref.dequantize(qtype, w, K).astype(np.float64)     # fp32 dequant
    xf = (xd[0].astype(np.float64).repeat(32) * xq[0].astype(np.float64))
    y_np = wf @ xf
    y = ref.gemv_dequant_f64(qtype, w, K, xq, xd)
    scale = np.abs(wf) @ np.abs(xf)
    # Q8_0's fp32 dequant is exact; Q4_K's rounds once per element
    tol = 1e-13 if qtype == 8 else 2.0 ** -23
    assert np.all(np.abs(y - y_np) <= tol * scale)


@pytest.mark.parametrize("qtype", [8, 12])
def test_block_sums_bruteforce(ref, qtype):
    rng = np.random.default_rng(7)
    N, K = 6, 512
    if qtype == 8:
        q = rng.integers(-127, 128, (N, K))
        w = _q8_0_bytes(0x3C00, q)          # d = 1 -> dequant == code
    else:
        q = rng.integers(0, 16, (N, K))
        w = _q4k_unit_rows(N, K, q)         # d = 1, sc = 1, m = 0 -> dequant == code
    codes = ref.dequantize(qtype, w, K).astype(np.int64)
    assert np.array_equal(codes, q)
    xq = rng.integers(-127, 128, K).astype(np.int8)
    want = (codes.reshape(N, K // 32, 32) * xq.astype(np.int64).reshape(1, K // 32, 32)).sum(-1)
    got = ref.block_sums(qtype, w, K, xq)
    assert np.array_equal(got, want)


def test_block_sum_extremes_q8_0(ref):
    K = 64
    q = np.full((2, K), 127)
    q[1] = -127
    w = _q8_0_bytes(0x3C00, q)
    xq = np.full(K, -127, np.int8)
    s = ref.block_sums(8, w, K, xq)
    assert s.tolist() == [[-516128, -516128], [516128, 516128]]


@pytest.mark.parametrize("qtype", [8, 12])
def test_unit_weights_closed_form(ref, qtype):
    """All codes 1 and unit scales: y_n = sum_b xd_b * xs_b for every row."""
    N, K = 5, 512
    w = _q8_0_bytes(0x3C00, np.ones((N, K), int)) if qtype == 8 else _q4k_unit_rows(N, K)
    xq, xd, xs = ref.quantize_act_q8(synth.activations(15, 1, K))
    y, _ = ref.gemv(qtype, w, K, xq, xd, xs)
    want = float(np.sum(xd[0].astype(np.float64) * xs[0].astype(np.float64)))
    assert np.allclose(y, want, rtol=1e-14, atol=0)


def test_q4k_min_term_closed_form(ref):
    """Codes 0, d = 0, dmin = 1, m_j = j+1: y = -sum_j (j+1) * xd_j * xs_j."""
    K = 256
    blk = np.zeros(144, np.uint8)
    blk[2:4] = np.array([0x3C00], np.uint16).view(np.uint8)     # dmin = 1.0
    for j in range(8):
        ref.q4k_set_scale_min(blk[4:16], j, 0, j + 1)
    xq, xd, xs = ref.quantize_act_q8(synth.activations(16, 1, K))
    y, _ = ref.gemv(12, blk[None, :], K, xq, xd, xs)
    want = -sum((j + 1) * float(xd[0, j]) * float(xs[0, j]) for j in range(8))
    assert abs(y[0] - want) <= 1e-14 * abs(want)


@pytest.mark.parametrize("qtype", [8, 12])
def test_one_hot_activation_picks_one_column(ref, qtype):
    N, K = 7, 512
    w = ref.quantize(qtype, synth.weights(17, N, K))
    k0 = 300
    x = np.zeros((1, K), np.float32)
    x[0, k0] = 2.54
    xq, xd, xs = ref.quantize_act_q8(x)
    assert xq[0, k0] == 127 and np.count_nonzero(xq) == 1
    y, _ = ref.gemv(qtype, w, K, xq, xd, xs)
    col = ref.gemv_dequant_f64(qtype, w, K, xq, xd)
    # with an exact dequant: y_n = w^[n, k0] * 127 * xd
    wf = ref.dequantize(qtype, w, K).astype(np.float64)
    want = wf[:, k0] * 127.0 * float(xd[0, k0 // 32])
    tol = 1e-14 if qtype == 8 else 2.0 ** -22
    assert np.all(np.abs(y - want) <= tol * np.abs(want) + 1e-300)
    assert np.all(np.abs(col - want) <= tol * np.abs(want) + 1e-300)


def test_textbook_integer_matvec(ref):
    """d_w = d_x = 1 reduces the method to an integer matrix-vector product."""
    rng = np.random.default_rng(8)
    N, K = 11, 1024
    q = rng.integers(-127, 128, (N, K))
    w = _q8_0_bytes(0x3C00, q)
    xq = rng.integers(-127, 128, K).astype(np.int8)
    xd = np.ones(K // 32, np.float32)
    y, _ = ref.gemv(8, w, K, xq, xd)
    assert np.array_equal(y, (q @ xq.astype(np.int64)).astype(np.float64))


def test_paired_and_grouped_are_independent_gemvs(ref):
    """Paired: (W0 x, W1 x); grouped: W_g x_g -- checked on the flat layout."""
    K, N, G = 256, 4, 3
    w = ref.quantize(8, synth.weights(18, G * N, K))          # [G*N, row] = [K, N, G]
    x = synth.activations(19, G, K)
    xq, xd, xs = ref.quantize_act_q8(x)
    flat = np.concatenate([ref.gemv(8, w[g * N:(g + 1) * N], K, xq[g], xd[g], xs[g])[0] for g in range(G)])
    wf = ref.dequantize(8, w, K).astype(np.float64).reshape(G, N, K)
    xf = (xd.astype(np.float64).repeat(32, axis=1) * xq.astype(np.float64))
    want = np.einsum("gnk,gk->gn", wf, xf).reshape(-1)
    assert np.allclose(flat, want, rtol=1e-12, atol=1e-15)


def _q4k_rows_const(N, K, d_f16, dmin_f16, sc, m, code):
    """Hand-assembled Q4_K rows: one fp16 d / dmin, every (sc_j, m_j) equal,
    every 4-bit code equal (scale field packed by the pinned setter)."""
    nsb = K // 256
    blk = np.zeros(144, np.uint8)
    blk[0:2] = np.array([d_f16], np.uint16).view(np.uint8)
    blk[2:4] = np.array([dmin_f16], np.uint16).view(np.uint8)
    s = np.zeros(12, np.uint8)
    for j in range(8):
        oracle.q4k_set_scale_min(s, j, sc, m)
    blk[4:16] = s
    blk[16:] = (code | (code << 4)) & 0xFF
    return np.tile(blk, (N, nsb))


def test_absum_closed_forms_q8_0(ref):
    """absum is the sum of the magnitudes of the block terms d_w * xd_b * isum_b.
    Unit codes make isum_b = xs_b, so with block signs s_b and scale d:
    y = d * sum_b s_b xd_b xs_b and absum = |d| * sum_b |xd_b xs_b|."""
    K = 1024
    nb = K // 32
    xq, xd, xs = ref.quantize_act_q8(synth.activations(21, 1, K))
    base = np.abs(xd[0].astype(np.float64) * xs[0].astype(np.float64))
    signs = np.where(np.arange(nb) % 2 == 0, 1, -1)
    rows = [(0x3C00, np.ones(K, int)),                       # d = 1, all +1
            (0x3C00, np.repeat(signs, 32)),                  # alternating block signs
            (0x4000, -np.ones(K, int))]                      # d = 2, all -1
    w = np.concatenate([_q8_0_bytes(d, q[None, :]) for d, q in rows])
    y, absum = ref.gemv(8, w, K, xq, xd, xs)
    want_abs = np.array([base.sum(), base.sum(), 2.0 * base.sum()])
    signed = xd[0].astype(np.float64) * xs[0].astype(np.float64)
    want_y = np.array([signed.sum(), (signs * signed).sum(), -2.0 * signed.sum()])
    assert np.allclose(absum, want_abs, rtol=1e-14, atol=0)
    assert np.allclose(y, want_y, rtol=1e-12, atol=1e-12 * base.sum())
    # the mixed-sign row cancels: |y| is well below the condition scale
    assert abs(y[1]) < 0.5 * absum[1]


def test_absum_counts_both_q4_k_terms(ref):
    """Q4_K forms two products per sub-block, (d sc) xd isum and (dmin m) xd xs,
    and absum adds both magnitudes.  With d = dmin = 1, sc = m = 1 and every
    code 1 the weights dequantize to exactly 0, so y = 0 while each product
    is xd_b xs_b: absum = 2 sum_b |xd_b xs_b|.  With codes 0 only the min
    term is left: absum = m sum_b |xd_b xs_b|."""
    K = 512
    xq, xd, xs = ref.quantize_act_q8(synth.activations(22, 1, K))
    base = float(np.sum(np.abs(xd[0].astype(np.float64) * xs[0].astype(np.float64))))
    w_cancel = _q4k_rows_const(1, K, 0x3C00, 0x3C00, 1, 1, 1)
    assert np.all(ref.dequantize(12, w_cancel, K) == 0.0)
    y, absum = ref.gemv(12, w_cancel, K, xq, xd, xs)
    assert y[0] == 0.0
    assert abs(absum[0] - 2.0 * base) <= 1e-14 * base
    w_min = _q4k_rows_const(1, K, 0x3C00, 0x3C00, 5, 3, 0)
    y, absum = ref.gemv(12, w_min, K, xq, xd, xs)
    assert abs(absum[0] - 3.0 * base) <= 1e-14 * base
    signed = float(np.sum(xd[0].astype(np.float64) * xs[0].astype(np.float64)))
    assert abs(y[0] + 3.0 * signed) <= 1e-13 * base


@pytest.mark.parametrize("qtype", [8, 12])
def test_absum_bounds_the_result(ref, qtype):
    """Triangle inequality on seeded data: |y_n| <= absum_n, and absum_n is at
    least the magnitude of the largest single block contribution."""
    N, K = 16, 1024
    w = ref.quantize(qtype, synth.weights(23, N, K))
    xq, xd, xs = ref.quantize_act_q8(synth.activations(24, 1, K))
    y, absum = ref.gemv(qtype, w, K, xq, xd, xs)
    assert np.all(np.abs(y) <= absum * (1 + 1e-14))
    wf = ref.dequantize(qtype, w, K).astype(np.float64)
    xf = xd[0].astype(np.float64).repeat(32) * xq[0].astype(np.float64)
    per_block = np.abs((wf * xf).reshape(N, K // 32, 32).sum(-1)).max(-1)
    assert np.all(absum >= per_block * (1 - 1e-6))
