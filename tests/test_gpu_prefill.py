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
         (8, 640, 2048, 70), (12, 128, 768, 257), (8, 200, 256, 513), (12, 4096, 4096, 3), (8, 1024, 512, 1100)]


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
                                       (8, 8192, 128), (8, 8192, 512), (8, 8192, 2048)])
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
