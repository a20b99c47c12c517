"""Decode GEMVs that take the fp32 activation and quantize it in the kernel
(dsq_gemv_f32, dsq_gemv_paired_f32, dsq_gemv_grouped_f32).

The fused call performs the same arithmetic as dsq_quantize_act_q8 followed by
the two-call GEMV -- the same Q8 codes, the same dot order -- so its outputs
must equal the two-call path bit for bit; they are also checked against the
oracle (activation quantization, then the fp64 integer-form GEMV) within
GEMV_TOL.  All four decode workloads run at full size, plus ragged and
multi-unit shapes and the shapes the fused form refuses.
"""
import numpy as np
import pytest
import torch

from block_quantized_dsq_b200 import DsqError, synth
from conftest import GEMV_TOL, gemv_error, plain_rel_error, to_dev

pytestmark = pytest.mark.gpu


def _two_call(dsq, qtype, wd, N, K, x_dev, M=1):
    xq = torch.empty((M, K), dtype=torch.int8, device="cuda")
    xd = torch.empty((M, K // 32), dtype=torch.float32, device="cuda")
    xs = torch.empty((M, K // 32), dtype=torch.int32, device="cuda")
    dsq.dsq_quantize_act_q8(x_dev, M, K, xq, xd, xs)
    return xq, xd, xs


def _oracle_check(ref, qtype, w, K, x, y):
    xq, xd, xs = ref.quantize_act_q8(x)
    y_ref, absum = ref.gemv(qtype, w, K, xq, xd, xs)
    assert gemv_error(y, y_ref, absum, K // 32) <= GEMV_TOL
    assert plain_rel_error(y, y_ref) <= GEMV_TOL


@pytest.mark.parametrize("qtype,N,K", [(8, 1024, 1024), (12, 4096, 4096), (8, 1, 256), (8, 777, 4096),
                                       (12, 33, 12288), (8, 129, 16384), (12, 300, 768)])
def test_single(dsq, ref, qtype, N, K):
    w = ref.quantize(qtype, synth.weights(300 + N, N, K))
    x = synth.activations(301 + K, 1, K)
    wd, xd_ = to_dev(w), to_dev(x)
    y_f = torch.full((N,), float("nan"), dtype=torch.float32, device="cuda")
    dsq.dsq_gemv_f32(qtype, wd, N, K, xd_, y_f)
    xq, xdd, xs = _two_call(dsq, qtype, wd, N, K, xd_)
    y_2 = torch.full((N,), float("nan"), dtype=torch.float32, device="cuda")
    if qtype == 8:
        dsq.dsq_gemv_q8_0(wd, N, K, xq, xdd, y_2)
    else:
        dsq.dsq_gemv_q4_k(wd, N, K, xq, xdd, xs, y_2)
    torch.cuda.synchronize()
    a, b = y_f.cpu().numpy(), y_2.cpu().numpy()
    assert np.array_equal(a.view(np.uint32), b.view(np.uint32))
    _oracle_check(ref, qtype, w, K, x, a)


def test_paired_workload_64_calls(dsq, ref):
    """2 x Q8_0 8192 x 4096 sharing one activation, 64 calls with fresh activations."""
    s = synth.SEEDS["paired_q8_0_2x8192x4096"]
    N, K = 8192, 4096
    w0 = ref.quantize(8, synth.weights(s["w0"], N, K))
    w1 = ref.quantize(8, synth.weights(s["w1"], N, K))
    w0d, w1d = to_dev(w0), to_dev(w1)
    X = np.stack([synth.activations(s["x_base"] + c, 1, K)[0] for c in range(64)])
    Xd = to_dev(X)
    Y = torch.full((64, 2, N), float("nan"), dtype=torch.float32, device="cuda")
    for c in range(64):
        dsq.dsq_gemv_paired_f32(8, w0d, N, w1d, N, K, Xd[c], Y[c, 0], Y[c, 1])
    torch.cuda.synchronize()
    Yh = Y.cpu().numpy()
    for c in (0, 1, 31, 63):
        xq, xd, xs = _two_call(dsq, 8, None, N, K, Xd[c])
        y0 = torch.empty(N, dtype=torch.float32, device="cuda")
        y1 = torch.empty(N, dtype=torch.float32, device="cuda")
        dsq.dsq_gemv_paired(8, w0d, N, w1d, N, K, xq, xd, xs, y0, y1)
        torch.cuda.synchronize()
        assert np.array_equal(Yh[c, 0].view(np.uint32), y0.cpu().numpy().view(np.uint32))
        assert np.array_equal(Yh[c, 1].view(np.uint32), y1.cpu().numpy().view(np.uint32))
        _oracle_check(ref, 8, w0, K, X[c:c + 1], Yh[c, 0])
        _oracle_check(ref, 8, w1, K, X[c:c + 1], Yh[c, 1])
    assert dsq.dsq_device_status() == 0


@pytest.mark.parametrize("qtype,N0,N1,K", [(12, 300, 77, 1024), (8, 0, 500, 2048), (8, 513, 0, 4096)])
def test_paired_ragged(dsq, ref, qtype, N0, N1, K):
    w0 = ref.quantize(qtype, synth.weights(310 + N0, max(N0, 1), K))[:N0]
    w1 = ref.quantize(qtype, synth.weights(311 + N1, max(N1, 1), K))[:N1]
    x = synth.activations(312, 1, K)
    y0 = torch.full((max(N0, 1),), float("nan"), dtype=torch.float32, device="cuda")
    y1 = torch.full((max(N1, 1),), float("nan"), dtype=torch.float32, device="cuda")
    w0d = to_dev(w0) if N0 else to_dev(np.zeros((1, 16), np.uint8))
    w1d = to_dev(w1) if N1 else to_dev(np.zeros((1, 16), np.uint8))
    dsq.dsq_gemv_paired_f32(qtype, w0d, N0, w1d, N1, K, to_dev(x), y0, y1)
    torch.cuda.synchronize()
    if N0:
        _oracle_check(ref, qtype, w0, K, x, y0.cpu().numpy()[:N0])
    if N1:
        _oracle_check(ref, qtype, w1, K, x, y1.cpu().numpy()[:N1])


@pytest.mark.parametrize("qtype,G,N,K", [(8, 8, 1024, 4096), (12, 3, 129, 2048), (8, 1, 64, 256)])
def test_grouped(dsq, ref, qtype, G, N, K):
    if (qtype, G, N, K) == (8, 8, 1024, 4096):
        s = synth.SEEDS["grouped_q8_0_8x1024x4096"]
        wseed, xseed = s["w_base"], s["x_base"]
    else:
        wseed, xseed = 320 + G, 330 + G
    Ws = [ref.quantize(qtype, synth.weights(wseed + g, N, K)) for g in range(G)]
    X = np.stack([synth.activations(xseed + g, 1, K)[0] for g in range(G)])
    wd = to_dev(np.concatenate(Ws, axis=0))
    Xd = to_dev(X)
    y_f = torch.full((G, N), float("nan"), dtype=torch.float32, device="cuda")
    dsq.dsq_gemv_grouped_f32(qtype, wd, G, N, K, Xd, y_f)
    xq, xd, xs = _two_call(dsq, qtype, wd, N, K, Xd, M=G)
    y_2 = torch.full((G, N), float("nan"), dtype=torch.float32, device="cuda")
    dsq.dsq_gemv_grouped(qtype, wd, G, N, K, xq, xd, xs, y_2)
    torch.cuda.synchronize()
    a, b = y_f.cpu().numpy(), y_2.cpu().numpy()
    assert np.array_equal(a.view(np.uint32), b.view(np.uint32))
    for g in range(G):
        _oracle_check(ref, qtype, Ws[g], K, X[g:g + 1], a[g])


def test_refused_shapes_launch_nothing(dsq):
    w = torch.zeros((64, dsq.dsq_row_bytes(8, 96)), dtype=torch.uint8, device="cuda")
    x = torch.zeros((16, 8192), dtype=torch.float32, device="cuda")
    y = torch.zeros((16, 64), dtype=torch.float32, device="cuda")
    before = dsq.dsq_launch_count()
    with pytest.raises(DsqError) as ei:   # K % 256 != 0: no fused form
        dsq.dsq_gemv_f32(8, w, 64, 96, x, y)
    assert ei.value.status == 3
    w2 = torch.zeros((16 * 64, dsq.dsq_row_bytes(8, 8192)), dtype=torch.uint8, device="cuda")
    with pytest.raises(DsqError) as ei:   # 16 x 8192 activations exceed the shared-memory area
        dsq.dsq_gemv_grouped_f32(8, w2, 16, 64, 8192, x, y)
    assert ei.value.status == 3 and "shared memory" in str(ei.value)
    with pytest.raises(DsqError) as ei:   # misaligned x
        dsq.dsq_gemv_f32(8, w2, 64, 8192, x.data_ptr() + 4, y)
    assert ei.value.status == 2
    with pytest.raises(DsqError) as ei:   # null x
        dsq.dsq_gemv_f32(8, w2, 64, 8192, None, y)
    assert ei.value.status == 1
    assert dsq.dsq_launch_count() == before
