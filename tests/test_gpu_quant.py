"""Activation prequantization and weight quantizers on the GPU: bit-exact
with the CPU oracle (codes, scales and block sums compared byte by byte)."""
import numpy as np
import pytest
import torch

from block_quantized_dsq_b200 import synth
from conftest import to_dev

pytestmark = pytest.mark.gpu


def _act_cases():
    rng = np.random.default_rng(31)
    cases = {
        "decode_k1024": synth.activations(100, 1, 1024),
        "decode_k4096": synth.activations(1000, 1, 4096),
        "grouped_8x4096": np.concatenate([synth.activations(140 + g, 1, 4096) for g in range(8)]),
        "tiny_k32": synth.activations(5, 3, 32),
        "ragged_k96": synth.activations(6, 5, 96),
        "prefill_512x4096": synth.activations(712, 512, 4096),
    }
    special = rng.standard_normal((4, 256)).astype(np.float32)
    special[0, :32] = 0.0                                          # all-zero block
    special[0, 32:64] = np.float32(2.5) * (np.arange(32) - 16)      # exact ties at d = 2.5*16/127?
    special[1, :32] = (np.arange(32, dtype=np.float32) - 15.5) * 2.0 ** -130   # subnormal inputs
    special[1, 32:64] = 3e38 * np.sign(rng.standard_normal(32))     # near fp32 max
    special[2, :] *= 1e-20
    special[3, :32] = 127.0 * (rng.integers(-2, 3, 32) / 2.0)       # half-integers with d = 1
    special[3, 0] = 127.0
    cases["special_values"] = special
    return cases


@pytest.mark.parametrize("name", list(_act_cases()))
def test_act_q8_bit_exact(dsq, ref, name):
    x = _act_cases()[name]
    M, K = x.shape
    xq_r, xd_r, xs_r = ref.quantize_act_q8(x)
    xg = to_dev(x)
    xq = torch.empty((M, K), dtype=torch.int8, device="cuda")
    xd = torch.empty((M, K // 32), dtype=torch.float32, device="cuda")
    xs = torch.empty((M, K // 32), dtype=torch.int32, device="cuda")
    dsq.dsq_quantize_act_q8(xg, M, K, xq, xd, xs)
    torch.cuda.synchronize()
    assert np.array_equal(xq.cpu().numpy(), xq_r)
    assert np.array_equal(xd.cpu().numpy().view(np.uint32), xd_r.view(np.uint32))
    assert np.array_equal(xs.cpu().numpy(), xs_r)


def test_act_q8_without_block_sums(dsq, ref):
    x = synth.activations(9, 2, 512)
    xq_r, xd_r, _ = ref.quantize_act_q8(x)
    xq = torch.empty((2, 512), dtype=torch.int8, device="cuda")
    xd = torch.empty((2, 16), dtype=torch.float32, device="cuda")
    dsq.dsq_quantize_act_q8(to_dev(x), 2, 512, xq, xd, None)
    torch.cuda.synchronize()
    assert np.array_equal(xq.cpu().numpy(), xq_r)
    assert np.array_equal(xd.cpu().numpy(), xd_r)


@pytest.mark.parametrize("qtype,N,K", [(8, 64, 4096), (8, 33, 96), (8, 1, 32), (12, 64, 4096), (12, 7, 256),
                                       (12, 3, 768)])
def test_weight_quantizer_bit_exact(dsq, ref, qtype, N, K):
    x = synth.weights(50 + N, N, K)
    x[0, :256] = 0.0                       # a zero super-block / zero blocks
    if N > 2:
        x[1] = np.abs(x[1])                # all non-negative row (m = 0)
        x[2] = -np.abs(x[2])               # all non-positive row
    want = ref.quantize(qtype, x)
    w = torch.empty((N, want.shape[1]), dtype=torch.uint8, device="cuda")
    dsq.dsq_quantize_weights(qtype, to_dev(x), N, K, w)
    torch.cuda.synchronize()
    assert np.array_equal(w.cpu().numpy(), want)
