"""Prefill dequant-GEMM parity on the GPU.

Three checks per case: the rounded operands (binary16 bits of the scaled
activations and of the dequantized weights, plus the row shifts) are
bit-exact with the oracle; the output is within PREFILL_ROUNDED_TOL relative
L2 of the oracle's operand-rounded fp64 sum (only accumulation error is
left); and within PREFILL_TOL of the fp64 dequantized reference.  Sizes span
several tiles, ragged token and row counts, K-split, one token, and the full
workload sizes (sampled rows/columns computed one by one by the oracle).
"""
import numpy as np
import pytest
import torch

from block_quantized_dsq_b200 import synth
from conftest import PREFILL_ROUNDED_TOL, PREFILL_TOL, to_dev

pytestmark = pytest.mark.gpu


def rel_l2(y, y_ref):
    return float(np.linalg.norm(np.asarray(y, np.float64) - y_ref) / np.linalg.norm(y_ref))


def run_prefill(dsq, qtype, wg, N, K, xg, M):
    y = torch.full((M, N), float("nan"), dtype=torch.float32, device="cuda")
    nbytes = dsq.dsq_prefill_workspace_bytes(qtype, N, K, M)
    ws = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    dsq.dsq_gemm_prefill(qtype, wg, N, K, xg, M, y, ws, nbytes)
    torch.cuda.synchronize()
    return y.cpu().numpy()


CASES = [(8, 128, 256, 1), (8, 256, 512, 5), (12, 300, 512, 33), (8, 128, 4096, 128), (12, 384, 1024, 200),
         (8, 640, 2048, 70), (12, 128, 768, 257), (8, 200, 256, 513), (12, 4096, 4096, 3), (8, 1024, 512, 1100),
         # M = 1 takes the CUDA-core small-M kernel, up to 8 the
         # mma.sync kernel (when its activations fit), then the narrowest
         # tensor-core tile
         (8, 4096, 4096, 8), (12, 1000, 2048, 3), (8, 33, 16384, 2), (12, 300, 512, 9), (8, 256, 512, 17),
         (8, 700, 1024, 2), (12, 64, 256, 1),
         (12, 4096, 4096, 4), (12, 517, 2048, 6), (12, 100, 4096, 8), (8, 95, 1024, 4), (8, 1000, 3072, 6),
         (12, 64, 16384, 8)]   # K = 16384: the mma.sync kernel's activations do not fit


@pytest.mark.parametrize("qtype,N,K,M", CASES)
def test_prefill_parity(dsq, ref, qtype, N, K, M):
    w = ref.quantize(qtype, synth.weights(300 + N, N, K))
    x = synth.activations(301 + M, M, K)
    if M > 2:
        x[1] *= 1e3          # rows with different power-of-two shifts
        x[2] *= 1e-4
    y = run_prefill(dsq, qtype, to_dev(w), N, K, to_dev(x), M)
    assert np.isfinite(y).all()
    y_rounded = ref.prefill_rounded(qtype, w, K, x, "f16")
    assert rel_l2(y, y_rounded) <= PREFILL_ROUNDED_TOL
    y64 = ref.prefill_f64(qtype, w, K, x)
    assert rel_l2(y, y64) <= PREFILL_TOL


@pytest.mark.parametrize("qtype,N,K,M", [(8, 130, 512, 7), (12, 64, 1024, 3)])
def test_prefill_operands_bit_exact(dsq, ref, qtype, N, K, M):
    w = ref.quantize(qtype, synth.weights(310, N, K))
    x = synth.activations(311, M, K)
    x[0] *= 7e4              # beyond binary16 range before scaling
    x[1, :17] = 0.0
    x16_r, sh_r, w16_r = ref.prefill_operands(qtype, w, K, x, "f16")
    x16 = torch.empty((M, K), dtype=torch.int16, device="cuda")
    sh = torch.empty(M, dtype=torch.int32, device="cuda")
    w16 = torch.empty((N, K), dtype=torch.int16, device="cuda")
    dsq.dsq_test_prefill_operands(qtype, to_dev(w), N, K, to_dev(x), M, x16, sh, w16)
    torch.cuda.synchronize()
    assert np.array_equal(sh.cpu().numpy(), sh_r)
    assert np.array_equal(x16.cpu().numpy().view(np.uint16), x16_r)
    assert np.array_equal(w16.cpu().numpy().view(np.uint16), w16_r)


@pytest.mark.parametrize("qtype,N,M", [(12, 4096, 128), (12, 4096, 512), (12, 4096, 2048),
                                       (8, 8192, 128), (8, 8192, 512), (8, 8192, 2048), (12, 4096, 3), (8, 8192, 2)])
def test_prefill_workload_sampled(dsq, ref, qtype, N, M):
    """Full workload sizes (K = 4096), in the configuration the bench times;
    the oracle recomputes a sample of 48 tokens x 256 weight rows."""
    K = 4096
    seeds = synth.SEEDS["prefill"]
    w = ref.quantize(qtype, synth.weights(seeds["w_q4_k"] if qtype == 12 else seeds["w_q8_0"], N, K))
    x = synth.activations(seeds["x_base"] + M, M, K)
    y = run_prefill(dsq, qtype, to_dev(w), N, K, to_dev(x), M)
    assert np.isfinite(y).all()
    rng = np.random.default_rng(M + N)
    ms = np.sort(rng.choice(M, size=min(48, M), replace=False))
    ns = np.sort(rng.choice(N, size=256, replace=False))
    ys = y[np.ix_(ms, ns)]
    assert rel_l2(ys, ref.prefill_rounded(qtype, w[ns], K, x[ms], "f16")) <= PREFILL_ROUNDED_TOL
    assert rel_l2(ys, ref.prefill_f64(qtype, w[ns], K, x[ms])) <= PREFILL_TOL


def test_prefill_workspace_is_checked(dsq, ref):
    w = ref.quantize(8, synth.weights(320, 128, 256))
    x = synth.activations(321, 4, 256)
    need = dsq.dsq_prefill_workspace_bytes(8, 128, 256, 4)
    assert need > 0
    ws = torch.empty(need, dtype=torch.uint8, device="cuda")
    y = torch.empty((4, 128), dtype=torch.float32, device="cuda")
    from block_quantized_dsq_b200 import DsqError
    with pytest.raises(DsqError) as ei:
        dsq.dsq_gemm_prefill(8, to_dev(w), 128, 256, to_dev(x), 4, y, ws, need - 1)
    assert ei.value.status == 5
    with pytest.raises(DsqError) as ei:
        dsq.dsq_gemm_prefill(8, to_dev(w), 128, 256, to_dev(x), 4, y, None, need)
    assert ei.value.status == 5


def _operands_and_status(dsq, ref, qtype, w, K, x):
    """The kernels' rounded operands and the device status they leave, with
    the oracle's operands for the same inputs."""
    N, M = w.shape[0], x.shape[0]
    x16 = torch.empty((M, K), dtype=torch.int16, device="cuda")
    sh = torch.empty(M, dtype=torch.int32, device="cuda")
    w16 = torch.empty((N, K), dtype=torch.int16, device="cuda")
    assert dsq.dsq_device_status() == 0
    dsq.dsq_test_prefill_operands(qtype, to_dev(w), N, K, to_dev(x), M, x16, sh, w16)
    status = dsq.dsq_device_status()
    got = (x16.cpu().numpy().view(np.uint16), sh.cpu().numpy(), w16.cpu().numpy().view(np.uint16))
    x16_r, sh_r, w16_r = ref.prefill_operands(qtype, w, K, x, "f16")
    return got, (x16_r, sh_r, w16_r), status


@pytest.mark.parametrize("qtype", [8, 12])
@pytest.mark.parametrize("sigma_scale", [5e-5, 1e-3])
def test_prefill_operands_tiny_weights_and_extreme_rows(dsq, ref, qtype, sigma_scale):
    """Weights of sigma 1e-6 and 2e-5 (binary16 subnormals, and values around
    the smallest normal 2^-14) and activation rows at the ends of the shift
    range: max |x| near FLT_MAX (shift -113), 2^-118 (shift clamped at 126),
    fp32 subnormals.  The operand bits must still equal the oracle's."""
    N, K, M = 96, 512, 6
    w = ref.quantize(qtype, synth.weights(330, N, K) * np.float32(sigma_scale))
    x = synth.activations(331, M, K)
    x[0] *= np.float32(3.0e38 / np.abs(x[0]).max())
    x[1] *= np.float32(2.0 ** -118 / np.abs(x[1]).max())
    x[2] = (x[2] * np.float32(1e-40)).astype(np.float32)          # fp32 subnormals
    x[3, ::2] = 0.0
    x[4] = 0.0
    got, want, status = _operands_and_status(dsq, ref, qtype, w, K, x)
    assert status == 0
    assert want[1][0] == -113 and want[1][1] == 126 and want[1][4] == 0
    for g, r in zip(got, want):
        assert np.array_equal(g, r)
    # at least some weights landed in the binary16 subnormal range
    if sigma_scale == 5e-5:
        mag = want[2] & 0x7FFF
        assert np.any((mag > 0) & (mag < 0x0400))


def test_prefill_extreme_rows_parity(dsq, ref):
    """Rows near FLT_MAX and near 2^-118 go through the whole GEMM: each row
    within the rounded-reference tolerance of its own norm."""
    qtype, N, K, M = 8, 256, 256, 40
    w = ref.quantize(qtype, synth.weights(332, N, K))
    x = synth.activations(333, M, K)
    x[0] *= np.float32(1.0e37 / np.abs(x[0]).max())
    x[1] *= np.float32(2.0 ** -118 / np.abs(x[1]).max())
    x[2] *= np.float32(2.0 ** 100)
    y = run_prefill(dsq, qtype, to_dev(w), N, K, to_dev(x), M)
    assert np.isfinite(y).all()
    y_rounded = ref.prefill_rounded(qtype, w, K, x, "f16")
    y64 = ref.prefill_f64(qtype, w, K, x)
    for m in range(M):
        assert rel_l2(y[m], y_rounded[m]) <= PREFILL_ROUNDED_TOL, m
        assert rel_l2(y[m], y64[m]) <= PREFILL_TOL, m


def _q8_0_row_with_block(ref, N, K, d_bits, code):
    """Seeded Q8_0 rows; row 5's first block gets scale bits d_bits and
    codes alternating +code / -code."""
    w = ref.quantize(8, synth.weights(334, N, K))
    blk = w[5, 0:34]
    blk[0:2] = np.array([d_bits], np.uint16).view(np.uint8)
    blk[2:] = np.array([code, -code] * 16, np.int8).view(np.uint8)
    return w


def _q4_k_row_with_subblock(ref, N, K, d_bits, dmin_bits, sc, m, codes):
    """Seeded Q4_K rows; row 5's first super-block gets d / dmin bits, sub-block
    0 the scale pair (sc, m) and the given codes, the others (0, 0)."""
    w = ref.quantize(12, synth.weights(335, N, K))
    blk = w[5, 0:144]
    blk[0:2] = np.array([d_bits], np.uint16).view(np.uint8)
    blk[2:4] = np.array([dmin_bits], np.uint16).view(np.uint8)
    sc12 = np.zeros(12, np.uint8)
    ref.q4k_set_scale_min(sc12, 0, sc, m)
    blk[4:16] = sc12
    blk[16:48] = (np.array(codes, np.uint8) & 0x0F) | (blk[16:48] & 0xF0)
    return w


RANGE_CASES = [
    # (type, builder args, out of range?)
    (8, (0x6007, 127), False),          # |d| = 515.5: 515.5 * 127 = 65468.5 -> 65472, finite
    (8, (0x6008, 127), True),           # |d| = 516:   516 * 127 = 65532 -> inf
    (8, (0xE008, 127), True),           # d = -516
    (12, (0x5450, 0x0000, 63, 0, [15, 0] * 16), False),   # 15 * 69 * 63 = 65205 -> 65216, finite
    (12, (0x5460, 0x0000, 63, 0, [15, 0] * 16), True),    # 15 * 70 * 63 = 66150 -> inf
    (12, (0x0000, 0x6410, 0, 63, [0, 1] * 16), True),     # -dmin * m = -65520 -> -inf
]


@pytest.mark.parametrize("M", [1, 2, 6, 40])      # the small-M, mma.sync and tensor-core kernels
@pytest.mark.parametrize("qtype,args,bad", RANGE_CASES)
def test_prefill_weight_range_fails_closed(dsq, ref, qtype, args, bad, M):
    """A weight block whose dequantized values leave the binary16 range makes
    the kernels record DSQ_ERR_RANGE; a block just inside the bound does not.
    Either way the operand bits equal the oracle's (inf where it overflows)."""
    N, K = 128, 256
    w = _q8_0_row_with_block(ref, N, K, *args) if qtype == 8 else _q4_k_row_with_subblock(ref, N, K, *args)
    x = synth.activations(336, M, K)
    got, want, status = _operands_and_status(dsq, ref, qtype, w, K, x)
    assert np.array_equal(got[2], want[2])
    w16 = want[2]
    has_inf = bool(np.any((w16 & 0x7FFF) == 0x7C00))
    assert has_inf == bad
    assert status == (9 if bad else 0)
    y = run_prefill(dsq, qtype, to_dev(w), N, K, to_dev(x), M)
    assert dsq.dsq_device_status() == (9 if bad else 0)
    assert np.isfinite(np.delete(y, 5, axis=1)).all()
    assert np.isfinite(y[:, 5]).all() != bad


@pytest.mark.parametrize("qtype,N,K,M", [(8, 129, 4096, 9), (12, 255, 2048, 11), (8, 33, 1024, 13)])
def test_prefill_split_k_ragged_outputs(dsq, ref, qtype, N, K, M):
    """K split across many pair tiles with M x N not a multiple of 4: every
    split's partials must be summed from the right place."""
    w = ref.quantize(qtype, synth.weights(340 + N, N, K))
    x = synth.activations(341 + M, M, K)
    y = run_prefill(dsq, qtype, to_dev(w), N, K, to_dev(x), M)
    assert (M * N) % 4 != 0
    assert rel_l2(y, ref.prefill_rounded(qtype, w, K, x, "f16")) <= PREFILL_ROUNDED_TOL
    assert rel_l2(y, ref.prefill_f64(qtype, w, K, x)) <= PREFILL_TOL


def _grouped(dsq, qtype, wgs, Ns, K, xg, M):
    ys = [torch.full((M, n), float("nan"), dtype=torch.float32, device="cuda") for n in Ns]
    nb = dsq.dsq_prefill_grouped_workspace_bytes(qtype, Ns, K, M)
    ws = torch.empty(nb, dtype=torch.uint8, device="cuda")
    dsq.dsq_gemm_prefill_grouped(qtype, wgs, Ns, K, xg, M, ys, ws, nb)
    torch.cuda.synchronize()
    return ys


@pytest.mark.parametrize("qtype,Ns,K,M", [(12, [300, 129, 256], 1024, 7), (8, [512, 64], 512, 40),
                                          (8, [128, 200, 256, 77], 256, 300), (12, [1536], 1024, 33),
                                          (12, [300, 129, 256], 1024, 19), (8, [64, 1000], 4096, 2)])
def test_prefill_grouped_parity(dsq, ref, qtype, Ns, K, M):
    """Several weights sharing X in one launch (grouped attention-A prefill):
    each output against the oracle's references for that weight."""
    ws = [ref.quantize(qtype, synth.weights(350 + g, n, K)) for g, n in enumerate(Ns)]
    x = synth.activations(351 + M, M, K)
    x[min(1, M - 1)] *= 1e3
    ys = _grouped(dsq, qtype, [to_dev(w) for w in ws], Ns, K, to_dev(x), M)
    for w, y in zip(ws, ys):
        yc = y.cpu().numpy()
        assert np.isfinite(yc).all()
        assert rel_l2(yc, ref.prefill_rounded(qtype, w, K, x, "f16")) <= PREFILL_ROUNDED_TOL
        assert rel_l2(yc, ref.prefill_f64(qtype, w, K, x)) <= PREFILL_TOL


@pytest.mark.parametrize("qtype", [8, 12])
def test_prefill_grouped_equals_single_calls(dsq, ref, qtype):
    """With the same split plan a weight computed in a group gets exactly the
    bits it gets alone: at M = 2048 neither 2048 rows (64 pair tiles) nor 2304
    rows (72) nor both together split K on 74 SM pairs.  A sample is also
    checked against the oracle."""
    K, M, Ns = 4096, 2048, [2048, 2304]
    ws = [ref.quantize(qtype, synth.weights(360 + g, n, K)) for g, n in enumerate(Ns)]
    x = synth.activations(361, M, K)
    wgs, xg = [to_dev(w) for w in ws], to_dev(x)
    ys = _grouped(dsq, qtype, wgs, Ns, K, xg, M)
    rng = np.random.default_rng(362)
    ms = np.sort(rng.choice(M, size=24, replace=False))
    for g, (w, n) in enumerate(zip(ws, Ns)):
        y1 = torch.from_numpy(run_prefill(dsq, qtype, wgs[g], n, K, xg, M)).cuda()
        assert torch.equal(ys[g], y1)
        ns = np.sort(rng.choice(n, size=128, replace=False))
        ys_c = ys[g].cpu().numpy()[np.ix_(ms, ns)]
        assert rel_l2(ys_c, ref.prefill_rounded(qtype, w[ns], K, x[ms], "f16")) <= PREFILL_ROUNDED_TOL


def test_prefill_grouped_refusals(dsq):
    from block_quantized_dsq_b200 import DsqError
    t = torch.zeros(1 << 16, dtype=torch.uint8, device="cuda")
    before = dsq.dsq_launch_count()
    for ws, Ns, status in [([t] * 5, [128] * 5, 1), ([t, t], [128, 0], 1), ([t], [128], 5)]:
        with pytest.raises(DsqError) as ei:
            dsq.dsq_gemm_prefill_grouped(8, ws, Ns, 256, t, 4, [t] * len(ws), t, 0)
        assert ei.value.status == status
    assert dsq.dsq_launch_count() == before


@pytest.mark.parametrize("qtype,N,K,M", [(12, 4000, 1024, 300), (8, 2000, 2048, 700)])
def test_prefill_two_way_split_is_deterministic(dsq, ref, qtype, N, K, M):
    """K split in two: the partials are summed in split order, so two calls
    give the same bits."""
    tiles = -(-M // 256) * -(-N // 256)
    assert 2 * tiles <= 74 < 4 * tiles          # the planner splits K in two on 74 SM pairs
    w = ref.quantize(qtype, synth.weights(370 + N, N, K))
    x = synth.activations(371 + M, M, K)
    y1 = run_prefill(dsq, qtype, to_dev(w), N, K, to_dev(x), M)
    y2 = run_prefill(dsq, qtype, to_dev(w), N, K, to_dev(x), M)
    assert np.array_equal(y1, y2)
    assert rel_l2(y1, ref.prefill_rounded(qtype, w, K, x, "f16")) <= PREFILL_ROUNDED_TOL
    assert rel_l2(y1, ref.prefill_f64(qtype, w, K, x)) <= PREFILL_TOL


@pytest.mark.parametrize("qtype", [8, 12])
@pytest.mark.parametrize("M", [4, 300])          # the mma.sync bridge and the CTA-pair kernel
def test_prefill_sees_weights_written_just_before(dsq, ref, qtype, M):
    """Weights quantized on the same stream immediately before the call, with
    no synchronization between, are the ones multiplied: the kernels that
    read weights wait for their predecessors before their first weight
    load."""
    N, K = 1024, 2048
    w32 = synth.weights(400 + M, N, K)
    x = synth.activations(401 + M, M, K)
    w_ref = ref.quantize(qtype, w32)
    w = torch.zeros(w_ref.shape, dtype=torch.uint8, device="cuda")
    w32g, xg = to_dev(w32), to_dev(x)
    y = torch.full((M, N), float("nan"), dtype=torch.float32, device="cuda")
    nb = dsq.dsq_prefill_workspace_bytes(qtype, N, K, M)
    ws = torch.empty(nb, dtype=torch.uint8, device="cuda")
    torch.cuda.synchronize()
    dsq.dsq_quantize_weights(qtype, w32g, N, K, w)
    dsq.dsq_gemm_prefill(qtype, w, N, K, xg, M, y, ws, nb)
    torch.cuda.synchronize()
    assert np.array_equal(w.cpu().numpy(), w_ref)
    assert rel_l2(y.cpu().numpy(), ref.prefill_rounded(qtype, w_ref, K, x, "f16")) <= PREFILL_ROUNDED_TOL


@pytest.mark.parametrize("qtype,N,K,M", [(12, 10000, 4096, 300), (8, 10000, 2048, 300)])
def test_prefill_last_wave_split(dsq, ref, qtype, N, K, M):
    """40 weight tiles x 2 token tiles = 80 pair tiles on 74 SM pairs: the
    last wave's 6 tiles (weight rows 9472 .. 9999, the last tile ragged, and
    both token tiles, the second ragged at 300 tokens) are split in K into
    one wave of pieces whose partials a second kernel sums in split order.
    Every row of those tiles and a sample of the others against the oracle;
    two calls give the same bits."""
    m_pad = -(-M // 256) * 256
    unsplit = m_pad * K * 2 + -(-m_pad * 4 // 1024) * 1024
    assert dsq.dsq_prefill_workspace_bytes(qtype, N, K, M) > unsplit   # the plan holds last-wave partials
    w = ref.quantize(qtype, synth.weights(380 + N, N, K))
    x = synth.activations(381 + M, M, K)
    x[1] *= 1e3
    y1 = run_prefill(dsq, qtype, to_dev(w), N, K, to_dev(x), M)
    y2 = run_prefill(dsq, qtype, to_dev(w), N, K, to_dev(x), M)
    assert np.isfinite(y1).all()
    assert np.array_equal(y1, y2)
    rng = np.random.default_rng(382)
    ns = np.concatenate([np.sort(rng.choice(9472, size=128, replace=False)), np.arange(9472, N)])
    ys = y1[:, ns]
    assert rel_l2(ys[:, 128:], ref.prefill_rounded(qtype, w[ns[128:]], K, x, "f16")) <= PREFILL_ROUNDED_TOL
    assert rel_l2(ys, ref.prefill_rounded(qtype, w[ns], K, x, "f16")) <= PREFILL_ROUNDED_TOL
    assert rel_l2(ys, ref.prefill_f64(qtype, w[ns], K, x)) <= PREFILL_TOL


def test_prefill_grouped_last_wave_split(dsq, ref):
    """Q4_K weights of 4096 and 1024 rows sharing 2048 tokens: 160 pair tiles
    = 2 waves of 74 and a last wave of 12 tiles (the second weight's rows
    512 .. 1023 for tokens from 1024 on, and rows 768 .. 1023 for all), split
    in K.  Those rows and a sample of the rest against the oracle."""
    qtype, K, M, Ns = 12, 4096, 2048, [4096, 1024]
    ws = [ref.quantize(qtype, synth.weights(390 + g, n, K)) for g, n in enumerate(Ns)]
    x = synth.activations(397, M, K)
    ys = _grouped(dsq, qtype, [to_dev(w) for w in ws], Ns, K, to_dev(x), M)
    rng = np.random.default_rng(392)
    ms = np.sort(np.concatenate([rng.choice(1024, size=16, replace=False),
                                 1024 + rng.choice(1024, size=32, replace=False)]))
    for g, (w, y) in enumerate(zip(ws, ys)):
        yc = y.cpu().numpy()
        assert np.isfinite(yc).all()
        ns = np.arange(512, 1024) if g == 1 else np.sort(rng.choice(Ns[g], size=128, replace=False))
        ys_c = yc[np.ix_(ms, ns)]
        assert rel_l2(ys_c, ref.prefill_rounded(qtype, w[ns], K, x[ms], "f16")) <= PREFILL_ROUNDED_TOL
        assert rel_l2(ys_c, ref.prefill_f64(qtype, w[ns], K, x[ms])) <= PREFILL_TOL
