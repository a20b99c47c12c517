"""Failure detection without a GPU fault: every pipeline wait in the kernels
is bounded.  With the test limit set to 0 each wait expires at once; the
kernels must record DSQ_ERR_TIMEOUT in the device status word, drain their
own copies, free TMEM and return -- after which the context is still usable
and a normal call gives correct results."""
import numpy as np
import pytest
import torch

from block_quantized_dsq_b200 import synth
from conftest import GEMV_TOL, PREFILL_TOL, gemv_error, to_dev

pytestmark = pytest.mark.gpu


def test_expired_waits_report_timeout_and_context_survives(dsq, ref):
    K, N, M = 1024, 512, 64
    w8 = ref.quantize(8, synth.weights(400, N, K))
    xq, xd, xs = ref.quantize_act_q8(synth.activations(401, 1, K))
    x = synth.activations(402, M, K)
    wg, xqg, xdg, xsg, xg = to_dev(w8), to_dev(xq), to_dev(xd), to_dev(xs), to_dev(x)
    y = torch.empty(N, dtype=torch.float32, device="cuda")
    Y = torch.empty((M, N), dtype=torch.float32, device="cuda")
    nbytes = dsq.dsq_prefill_workspace_bytes(8, N, K, M)
    ws = torch.empty(nbytes, dtype=torch.uint8, device="cuda")

    assert dsq.dsq_device_status() == 0
    try:
        dsq.dsq_test_set_wait_limit_ns(0)
        dsq.dsq_gemv_q8_0(wg, N, K, xqg, xdg, y)
        assert dsq.dsq_device_status() == 7            # DSQ_ERR_TIMEOUT
        dsq.dsq_gemm_prefill(8, wg, N, K, xg, M, Y, ws, nbytes)
        assert dsq.dsq_device_status() == 7
        dsq.dsq_gemm_prefill(8, wg, N, K, xg, 2, Y, ws, nbytes)      # the small-M kernel
        assert dsq.dsq_device_status() == 7
        dsq.dsq_gemv_paired(8, wg, N, wg, N, K, xqg, xdg, xsg, y, y)
        assert dsq.dsq_device_status() == 7
        dsq.dsq_gemv_tokens(8, wg, N, None, 0, K, 1, xqg, xdg, None, y, None)
        assert dsq.dsq_device_status() == 7
    finally:
        dsq.dsq_test_set_wait_limit_ns(2 ** 64 - 1)   # back to the default limit
    assert dsq.dsq_device_status() == 0                # the word was cleared

    dsq.dsq_gemv_q8_0(wg, N, K, xqg, xdg, y)
    y_tok = torch.empty(N, dtype=torch.float32, device="cuda")
    dsq.dsq_gemv_tokens(8, wg, N, None, 0, K, 1, xqg, xdg, None, y_tok, None)
    Y4 = torch.empty((2, N), dtype=torch.float32, device="cuda")
    dsq.dsq_gemm_prefill(8, wg, N, K, xg, 2, Y4, ws, nbytes)
    dsq.dsq_gemm_prefill(8, wg, N, K, xg, M, Y, ws, nbytes)
    assert dsq.dsq_device_status() == 0
    assert torch.equal(y, y_tok)
    Y64_4 = ref.prefill_f64(8, w8, K, x[:2])
    assert np.linalg.norm(Y4.cpu().numpy() - Y64_4) / np.linalg.norm(Y64_4) <= PREFILL_TOL
    y_ref, absum = ref.gemv(8, w8, K, xq, xd, xs)
    assert gemv_error(y.cpu().numpy(), y_ref, absum, K // 32) <= GEMV_TOL
    Y64 = ref.prefill_f64(8, w8, K, x)
    assert np.linalg.norm(Y.cpu().numpy() - Y64) / np.linalg.norm(Y64) <= PREFILL_TOL


def test_launch_counter_counts_kernels(dsq, ref):
    K, N = 256, 64
    w = to_dev(ref.quantize(8, synth.weights(403, N, K)))
    x = to_dev(synth.activations(404, 1, K))
    xq = torch.empty(K, dtype=torch.int8, device="cuda")
    xd = torch.empty(K // 32, dtype=torch.float32, device="cuda")
    y = torch.empty(N, dtype=torch.float32, device="cuda")
    before = dsq.dsq_launch_count()
    dsq.dsq_quantize_act_q8(x, 1, K, xq, xd, None)
    dsq.dsq_gemv_q8_0(w, N, K, xq, xd, y)
    torch.cuda.synchronize()
    assert dsq.dsq_launch_count() - before == 2
