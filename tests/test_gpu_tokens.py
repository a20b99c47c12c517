"""Multi-token decode GEMV (dsq_gemv_tokens) on the GPU.

M = 1..8 prequantized tokens against one weight or two weights that share the
input (the paired Q / KV projections).  Every token's outputs must equal bit
for bit the single-token entry points' outputs for that token (the kernel
keeps their block terms and reduction order), the per-block int32 sums are
compared bit-exactly with the oracle, and every output is within GEMV_TOL of
the oracle's fp64 integer-form GEMV.  Shapes cover one unit per row (G = 1),
three units (G = 4, idle virtual lanes), several units per virtual lane
(K = 12288), row counts below and across the 32-row groups, one weight empty,
and the paired decode workload's full size, on both kernels: the CUDA-core one
and, from 4 (Q8_0) or 5 (Q4_K) tokens, the tensor-core one.
"""
import numpy as np
import pytest
import torch

from block_quantized_dsq_b200 import synth
from conftest import GEMV_TOL, gemv_error, plain_rel_error, to_dev

pytestmark = pytest.mark.gpu


def _acts(ref, seed, M, K):
    X = synth.activations(seed, M, K)
    return ref.quantize_act_q8(X)


def _single(dsq, qtype, wg, N, K, xq, xd, xs, m):
    y = torch.empty(N, dtype=torch.float32, device="cuda")
    if qtype == 8:
        dsq.dsq_gemv_q8_0(wg, N, K, xq[m], xd[m], y)
    else:
        dsq.dsq_gemv_q4_k(wg, N, K, xq[m], xd[m], xs[m], y)
    return y


def _oracle_check(ref, qtype, w, K, xq, xd, xs, y):
    y_ref, absum = ref.gemv(qtype, w, K, xq, xd, xs)
    assert gemv_error(y, y_ref, absum, K // 32) <= GEMV_TOL
    assert plain_rel_error(y, y_ref) <= GEMV_TOL


CASES = [(8, 1, 256, 1), (8, 7, 256, 3), (12, 33, 768, 2), (8, 100, 1024, 8), (12, 1000, 1024, 5),
         (8, 515, 4096, 8), (12, 4096, 4096, 8), (8, 129, 12288, 4), (12, 64, 12288, 2), (8, 64, 2048, 6),
         (12, 200, 4096, 7), (8, 8192, 4096, 3), (12, 6000, 2048, 5),   # several row groups per CTA
         (12, 300, 6144, 7),    # tensor-core form, 24 units: four virtual lanes per warp, some idle
         (8, 300, 7168, 5),     # 8 padded tokens would not fit: the CUDA-core form takes M = 5
         (12, 700, 4096, 4)]    # below the Q4_K threshold: the CUDA-core form


@pytest.mark.parametrize("qtype,N,K,M", CASES)
def test_tokens_equal_single_token_calls_and_oracle(dsq, ref, qtype, N, K, M):
    w = ref.quantize(qtype, synth.weights(700 + N, N, K))
    xq, xd, xs = _acts(ref, 701 + M, M, K)
    wg, xqg, xdg, xsg = to_dev(w), to_dev(xq), to_dev(xd), to_dev(xs)
    y = torch.full((M, N), float("nan"), dtype=torch.float32, device="cuda")
    isum = torch.zeros((M, N, K // 32), dtype=torch.int32, device="cuda")
    dsq.dsq_test_block_sums_tokens(qtype, wg, N, K, M, xqg, xdg, xsg, y, isum)
    y2 = torch.full((M, N), float("nan"), dtype=torch.float32, device="cuda")
    dsq.dsq_gemv_tokens(qtype, wg, N, None, 0, K, M, xqg, xdg, xsg if qtype == 12 else None, y2, None)
    singles = [_single(dsq, qtype, wg, N, K, xqg, xdg, xsg, m) for m in range(M)]
    torch.cuda.synchronize()
    assert torch.equal(y, y2)                 # the test hook does not change the result
    isum_c = isum.cpu().numpy()
    yc = y.cpu().numpy()
    for m in range(M):
        assert torch.equal(y[m], singles[m]), f"token {m} differs from the single-token GEMV"
        assert np.array_equal(isum_c[m], ref.block_sums(qtype, w, K, xq[m]))
        _oracle_check(ref, qtype, w, K, xq[m], xd[m], xs[m], yc[m])


@pytest.mark.parametrize("qtype,N0,N1,K,M", [(8, 100, 37, 1024, 4), (12, 256, 513, 4096, 8), (8, 0, 64, 256, 2),
                                             (12, 5, 0, 512, 3), (8, 31, 33, 4096, 8)])
def test_tokens_paired(dsq, ref, qtype, N0, N1, K, M):
    w0 = ref.quantize(qtype, synth.weights(710, max(N0, 1), K))[:N0]
    w1 = ref.quantize(qtype, synth.weights(711, max(N1, 1), K))[:N1]
    xq, xd, xs = _acts(ref, 712, M, K)
    xqg, xdg, xsg = to_dev(xq), to_dev(xd), to_dev(xs)
    w0g = to_dev(w0) if N0 else None
    w1g = to_dev(w1) if N1 else None
    y0 = torch.full((M, max(N0, 1)), float("nan"), device="cuda")
    y1 = torch.full((M, max(N1, 1)), float("nan"), device="cuda")
    dsq.dsq_gemv_tokens(qtype, w0g, N0, w1g, N1, K, M, xqg, xdg, xsg, y0, y1)
    p0 = torch.full((max(N0, 1),), float("nan"), device="cuda")
    p1 = torch.full((max(N1, 1),), float("nan"), device="cuda")
    for m in range(M):
        dsq.dsq_gemv_paired(qtype, w0g, N0, w1g, N1, K, xqg[m], xdg[m], xsg[m], p0, p1)
        torch.cuda.synchronize()
        if N0:
            assert torch.equal(y0[m, :N0], p0[:N0])
            _oracle_check(ref, qtype, w0, K, xq[m], xd[m], xs[m], y0[m, :N0].cpu().numpy())
        if N1:
            assert torch.equal(y1[m, :N1], p1[:N1])
            _oracle_check(ref, qtype, w1, K, xq[m], xd[m], xs[m], y1[m, :N1].cpu().numpy())


def test_tokens_paired_workload_8_tokens(dsq, ref):
    """The paired decode workload's weights (2 x Q8_0 8192 x 4096, seeds 1/2)
    against 8 of its activations at once."""
    s = synth.SEEDS["paired_q8_0_2x8192x4096"]
    N, K, M = 8192, 4096, 8
    w0 = ref.quantize(8, synth.weights(s["w0"], N, K))
    w1 = ref.quantize(8, synth.weights(s["w1"], N, K))
    X = np.concatenate([synth.activations(s["x_base"] + i, 1, K) for i in range(M)])
    xq, xd, xs = ref.quantize_act_q8(X)
    y0 = torch.empty((M, N), device="cuda")
    y1 = torch.empty((M, N), device="cuda")
    dsq.dsq_gemv_tokens(8, to_dev(w0), N, to_dev(w1), N, K, M, to_dev(xq), to_dev(xd), None, y0, y1)
    torch.cuda.synchronize()
    y0c, y1c = y0.cpu().numpy(), y1.cpu().numpy()
    for m in range(M):
        _oracle_check(ref, 8, w0, K, xq[m], xd[m], xs[m], y0c[m])
        _oracle_check(ref, 8, w1, K, xq[m], xd[m], xs[m], y1c[m])


def test_tokens_refusals_launch_nothing(dsq):
    from block_quantized_dsq_b200 import DsqError
    A = torch.zeros(1 << 16, dtype=torch.uint8, device="cuda")
    p = A.data_ptr()
    before = dsq.dsq_launch_count()
    for args, status in [((8, p, 64, None, 0, 4096, 9, p, p, None, p, None), 3),     # M > 8
                         ((8, p, 64, None, 0, 4096, 0, p, p, None, p, None), 3),     # M < 1
                         ((8, p, 64, None, 0, 8192, 8, p, p, None, p, None), 3),     # activations > 64 KB
                         ((8, p, 64, None, 0, 96, 2, p, p, None, p, None), 3),       # K % 256
                         ((12, p, 64, None, 0, 256, 2, p, p, None, p, None), 1),     # Q4_K needs xs
                         ((8, p + 8, 64, None, 0, 256, 2, p, p, None, p, None), 2)]: # weight alignment
        with pytest.raises(DsqError) as ei:
            dsq.dsq_gemv_tokens(*args)
        assert ei.value.status == status, args
    dsq.dsq_gemv_tokens(8, None, 0, None, 0, 256, 3, None, None, None, None, None)   # empty: no-op
    assert dsq.dsq_launch_count() == before
