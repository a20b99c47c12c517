"""Decode GEMV parity on the GPU (regular, paired, grouped; Q8_0 and Q4_K).

Per-block int32 dot sums are compared bit-exactly (same device code as the
GEMV, through dsq_test_block_sums); outputs against the oracle's fp64
integer-form GEMV within GEMV_TOL (see conftest.gemv_error).  The four decode
workloads run at full size; edge shapes cover a single row, ragged row
counts, the smallest K, K that is not a multiple of 256 (the row-wise Q8_0
kernel) and K large enough that a lane handles several units per row.
"""
import numpy as np
import pytest
import torch

from block_quantized_dsq_b200 import synth
from conftest import GEMV_TOL, gemv_error, plain_rel_error, to_dev

pytestmark = pytest.mark.gpu


def _prep(ref, qtype, N, K, wseed, xseed, M=1):
    w = ref.quantize(qtype, synth.weights(wseed, N, K))
    x = synth.activations(xseed, M, K)
    xq, xd, xs = ref.quantize_act_q8(x)
    return w, xq, xd, xs


def _check(ref, qtype, w, K, xq, xd, xs, y):
    y_ref, absum = ref.gemv(qtype, w, K, xq, xd, xs)
    err = gemv_error(y, y_ref, absum, K // 32)
    assert err <= GEMV_TOL, err
    assert plain_rel_error(y, y_ref) <= GEMV_TOL


EDGE = [(8, 1, 256), (8, 1001, 1024), (8, 37, 32), (8, 50, 96), (8, 129, 12288), (8, 17, 16384),
        (8, 300, 3072), (12, 1, 256), (12, 515, 4096), (12, 33, 12288), (12, 9, 768)]


@pytest.mark.parametrize("qtype,N,K", EDGE)
def test_block_sums_bit_exact_and_gemv(dsq, ref, qtype, N, K):
    w, xq, xd, xs = _prep(ref, qtype, N, K, 60 + N, 61 + K)
    isum = torch.zeros((N, K // 32), dtype=torch.int32, device="cuda")
    y = torch.zeros(N, dtype=torch.float32, device="cuda")
    dsq.dsq_test_block_sums(qtype, to_dev(w), N, K, to_dev(xq), to_dev(xd), to_dev(xs), y, isum)
    torch.cuda.synchronize()
    assert np.array_equal(isum.cpu().numpy(), ref.block_sums(qtype, w, K, xq))
    _check(ref, qtype, w, K, xq, xd, xs, y.cpu().numpy())


@pytest.mark.parametrize("qtype,N,K", EDGE)
def test_regular_gemv(dsq, ref, qtype, N, K):
    w, xq, xd, xs = _prep(ref, qtype, N, K, 70 + N, 71 + K)
    y = torch.full((N,), float("nan"), dtype=torch.float32, device="cuda")
    if qtype == 8:
        dsq.dsq_gemv_q8_0(to_dev(w), N, K, to_dev(xq), to_dev(xd), y)
    else:
        dsq.dsq_gemv_q4_k(to_dev(w), N, K, to_dev(xq), to_dev(xd), to_dev(xs), y)
    torch.cuda.synchronize()
    _check(ref, qtype, w, K, xq, xd, xs, y.cpu().numpy())


def test_gemv_q8_0_1024_workload(dsq, ref):
    """Q8_0 GEMV 1024 x 1024, weights seed 0, activation seed 100."""
    s = synth.SEEDS["gemv_q8_0_1024"]
    w, xq, xd, xs = _prep(ref, 8, 1024, 1024, s["w"], s["x"])
    y = torch.empty(1024, dtype=torch.float32, device="cuda")
    dsq.dsq_gemv_q8_0(to_dev(w), 1024, 1024, to_dev(xq), to_dev(xd), y)
    torch.cuda.synchronize()
    _check(ref, 8, w, 1024, xq, xd, xs, y.cpu().numpy())


def test_gemv_q4_k_4096_workload(dsq, ref):
    s = synth.SEEDS["gemv_q4_k_4096"]
    w, xq, xd, xs = _prep(ref, 12, 4096, 4096, s["w"], s["x"])
    isum = torch.empty((4096, 128), dtype=torch.int32, device="cuda")
    y = torch.empty(4096, dtype=torch.float32, device="cuda")
    dsq.dsq_test_block_sums(12, to_dev(w), 4096, 4096, to_dev(xq), to_dev(xd), to_dev(xs), y, isum)
    y2 = torch.empty(4096, dtype=torch.float32, device="cuda")
    dsq.dsq_gemv_q4_k(to_dev(w), 4096, 4096, to_dev(xq), to_dev(xd), to_dev(xs), y2)
    torch.cuda.synchronize()
    assert np.array_equal(isum.cpu().numpy(), ref.block_sums(12, w, 4096, xq))
    assert torch.equal(y, y2)            # the hook does not change the result
    _check(ref, 12, w, 4096, xq, xd, xs, y2.cpu().numpy())


def test_paired_workload_64_calls(dsq, ref):
    """Two Q8_0 8192 x 4096 weights sharing one activation; 64 back-to-back
    calls with fresh seeded activations, each quantized on the GPU."""
    s = synth.SEEDS["paired_q8_0_2x8192x4096"]
    N, K = 8192, 4096
    w0 = ref.quantize(8, synth.weights(s["w0"], N, K))
    w1 = ref.quantize(8, synth.weights(s["w1"], N, K))
    w0g, w1g = to_dev(w0), to_dev(w1)
    X = np.concatenate([synth.activations(s["x_base"] + i, 1, K) for i in range(64)])
    xg = to_dev(X)
    xq = torch.empty((64, K), dtype=torch.int8, device="cuda")
    xd = torch.empty((64, K // 32), dtype=torch.float32, device="cuda")
    xs = torch.empty((64, K // 32), dtype=torch.int32, device="cuda")
    y = torch.empty((64, 2, N), dtype=torch.float32, device="cuda")
    for i in range(64):
        dsq.dsq_quantize_act_q8(xg[i], 1, K, xq[i], xd[i], xs[i])
        dsq.dsq_gemv_paired(8, w0g, N, w1g, N, K, xq[i], xd[i], xs[i], y[i, 0], y[i, 1])
    torch.cuda.synchronize()
    yc = y.cpu().numpy()
    xq_c, xd_c, xs_c = xq.cpu().numpy(), xd.cpu().numpy(), xs.cpu().numpy()
    for i in range(64):                 # the oracle over every one of the 64 calls
        q, d, sm = ref.quantize_act_q8(X[i:i + 1])
        assert np.array_equal(q[0], xq_c[i]) and np.array_equal(d[0], xd_c[i]) and np.array_equal(sm[0], xs_c[i])
        _check(ref, 8, w0, K, q, d, sm, yc[i, 0])
        _check(ref, 8, w1, K, q, d, sm, yc[i, 1])


@pytest.mark.parametrize("qtype,N0,N1,K", [(8, 100, 37, 1024), (12, 256, 513, 4096), (8, 0, 64, 256),
                                           (8, 5, 0, 96), (12, 1, 1, 256)])
def test_paired_edges(dsq, ref, qtype, N0, N1, K):
    w0 = ref.quantize(qtype, synth.weights(80, max(N0, 1), K))[:N0]
    w1 = ref.quantize(qtype, synth.weights(81, max(N1, 1), K))[:N1]
    xq, xd, xs = ref.quantize_act_q8(synth.activations(82, 1, K))
    y0 = torch.full((max(N0, 1),), float("nan"), device="cuda")
    y1 = torch.full((max(N1, 1),), float("nan"), device="cuda")
    w0g = to_dev(w0) if N0 else None
    w1g = to_dev(w1) if N1 else None
    dsq.dsq_gemv_paired(qtype, w0g, N0, w1g, N1, K, to_dev(xq), to_dev(xd), to_dev(xs), y0, y1)
    torch.cuda.synchronize()
    if N0:
        _check(ref, qtype, w0, K, xq, xd, xs, y0.cpu().numpy()[:N0])
    if N1:
        _check(ref, qtype, w1, K, xq, xd, xs, y1.cpu().numpy()[:N1])


def test_grouped_workload(dsq, ref):
    """8 groups of Q8_0 1024 x 4096, each with its own activation, one launch
    (ggml layout [4096, 1024, 8])."""
    s = synth.SEEDS["grouped_q8_0_8x1024x4096"]
    G, N, K = 8, 1024, 4096
    w = np.concatenate([ref.quantize(8, synth.weights(s["w_base"] + g, N, K)) for g in range(G)])
    X = np.concatenate([synth.activations(s["x_base"] + g, 1, K) for g in range(G)])
    xq, xd, xs = ref.quantize_act_q8(X)
    y = torch.empty((G, N), dtype=torch.float32, device="cuda")
    dsq.dsq_gemv_grouped(8, to_dev(w), G, N, K, to_dev(xq), to_dev(xd), to_dev(xs), y)
    torch.cuda.synchronize()
    yc = y.cpu().numpy()
    for g in range(G):
        _check(ref, 8, w[g * N:(g + 1) * N], K, xq[g], xd[g], xs[g], yc[g])


@pytest.mark.parametrize("qtype,G,N,K", [(8, 1, 64, 256), (8, 3, 37, 1024), (12, 4, 129, 512), (8, 5, 11, 96),
                                         (12, 16, 8, 4096)])
def test_grouped_edges(dsq, ref, qtype, G, N, K):
    w = ref.quantize(qtype, synth.weights(90 + G, G * N, K))
    X = synth.activations(91 + G, G, K)
    xq, xd, xs = ref.quantize_act_q8(X)
    y = torch.empty((G, N), dtype=torch.float32, device="cuda")
    dsq.dsq_gemv_grouped(qtype, to_dev(w), G, N, K, to_dev(xq), to_dev(xd), to_dev(xs), y)
    torch.cuda.synchronize()
    yc = y.cpu().numpy()
    for g in range(G):
        _check(ref, qtype, w[g * N:(g + 1) * N], K, xq[g], xd[g], xs[g], yc[g])


def test_results_are_deterministic(dsq, ref):
    w, xq, xd, xs = _prep(ref, 8, 2048, 4096, 95, 96)
    ys = []
    for _ in range(3):
        y = torch.empty(2048, dtype=torch.float32, device="cuda")
        dsq.dsq_gemv_q8_0(to_dev(w), 2048, 4096, to_dev(xq), to_dev(xd), y)
        ys.append(y)
    torch.cuda.synchronize()
    assert torch.equal(ys[0], ys[1]) and torch.equal(ys[1], ys[2])


@pytest.mark.parametrize("N", [148 * 200 + 7, 148 * 306 + 7])   # 200 and 306 rows per SM: 12 and 16 warps
def test_gemv_q4_k_long_matrix_takes_the_wide_launch(dsq, ref, N):
    """Q4_K matrices of K = 4096 long enough for the 12- and 16-warp launches
    (ragged row counts).  Each row is still reduced by one warp in the same
    order, so the first 4096 rows equal a 4096-row call (the 8-warp launch)
    bit for bit; all rows against the oracle."""
    K = 4096
    w, xq, xd, xs = _prep(ref, 12, N, K, 64, 65)
    wg, xqg, xdg, xsg = to_dev(w), to_dev(xq), to_dev(xd), to_dev(xs)
    y = torch.empty(N, dtype=torch.float32, device="cuda")
    dsq.dsq_gemv_q4_k(wg, N, K, xqg, xdg, xsg, y)
    y_head = torch.empty(4096, dtype=torch.float32, device="cuda")
    dsq.dsq_gemv_q4_k(wg, 4096, K, xqg, xdg, xsg, y_head)
    torch.cuda.synchronize()
    assert torch.equal(y[:4096], y_head)
    _check(ref, 12, w, K, xq, xd, xs, y.cpu().numpy())


@pytest.mark.parametrize("N", [1024, 8192])   # below and above the multi-token kernel's range
def test_gemv_q4_k_overlapped_launches_back_to_back(dsq, ref, N):
    """Shorter Q4_K GEMVs take the overlapped launch: a call starts loading its
    weights before its launch-dependency wait, beside the previous call.
    Weights quantized on the stream just before, and three back-to-back
    calls on different weights, activations and outputs with no host
    synchronization between them, each equal the same call made alone."""
    K = 4096
    w32 = [synth.weights(70 + i, N, K) for i in range(3)]
    acts = [_prep(ref, 12, 1, K, 80, 81 + i)[1:] for i in range(3)]
    wq = [torch.zeros((N, K // 256 * 144), dtype=torch.uint8, device="cuda") for _ in range(3)]
    ys = [torch.full((N,), float("nan"), dtype=torch.float32, device="cuda") for _ in range(3)]
    dev = [(to_dev(xq), to_dev(xd), to_dev(xs)) for xq, xd, xs in acts]
    w32g = [to_dev(w) for w in w32]
    torch.cuda.synchronize()
    for i in range(3):
        dsq.dsq_quantize_weights(12, w32g[i], N, K, wq[i])
    for i in range(3):
        dsq.dsq_gemv_q4_k(wq[i], N, K, *dev[i], ys[i])
    torch.cuda.synchronize()
    for i in range(3):
        y1 = torch.empty(N, dtype=torch.float32, device="cuda")
        dsq.dsq_gemv_q4_k(wq[i], N, K, *dev[i], y1)
        torch.cuda.synchronize()
        assert torch.equal(ys[i], y1)
        w_ref = ref.quantize(12, w32[i])
        assert np.array_equal(wq[i].cpu().numpy(), w_ref)
        _check(ref, 12, w_ref, K, *acts[i], ys[i].cpu().numpy())


@pytest.mark.parametrize("qtype,N,K", [(8, 3000, 4096), (12, 2500, 4096), (8, 148 * 32, 4096),
                                       (12, 148 * 32 + 1, 4096), (8, 2047, 4096),
                                       (8, 2048, 36864)])   # K above the multi-token kernel's activation area
def test_gemv_mid_length_single_token_routes_bit_exactly(dsq, ref, qtype, N, K):
    """From 2048 rows up to one 32-row group per SM (4736 rows on 148 SMs), and
    K up to 32768, a single-token GEMV runs the multi-token kernel; outside
    that range the GEMV kernel.  Either way the outputs equal, bit for bit, those of the
    block-sum hook (always the GEMV kernel), and the oracle's within 1e-5."""
    w, xq, xd, xs = _prep(ref, qtype, N, K, 90 + N, 91)
    wg, xqg, xdg, xsg = to_dev(w), to_dev(xq), to_dev(xd), to_dev(xs)
    y = torch.empty(N, dtype=torch.float32, device="cuda")
    if qtype == 8:
        dsq.dsq_gemv_q8_0(wg, N, K, xqg, xdg, y)
    else:
        dsq.dsq_gemv_q4_k(wg, N, K, xqg, xdg, xsg, y)
    y_hook = torch.empty(N, dtype=torch.float32, device="cuda")
    isum = torch.empty((N, K // 32), dtype=torch.int32, device="cuda")
    dsq.dsq_test_block_sums(qtype, wg, N, K, xqg, xdg, xsg, y_hook, isum)
    torch.cuda.synchronize()
    assert torch.equal(y, y_hook)
    _check(ref, qtype, w, K, xq, xd, xs, y.cpu().numpy())
