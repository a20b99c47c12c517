"""The allocation-free prefill entry point (dsq_gemm_prefill_noalloc).

Some callers cannot allocate device memory when they call into the library:
they run under a device-memory budget reserved up front, or are handed only
their input and output buffers by a host framework, or sit in a region where
cudaMalloc is not allowed.  For them, the library offers one entry point that
takes its scratch from a fixed 32 MiB array built into the library.  This
file checks, through the C ABI, that two calls in a row give what the regular
workspace entry point gives, and that a problem too large for the built-in
scratch is refused cleanly.  It sits last in collection order so that a run
that stops at the first failure has already run every other test; it also
passes on its own in a fresh process.
"""
import numpy as np
import pytest
import torch

from block_quantized_dsq_b200 import synth
from conftest import PREFILL_TOL, to_dev

pytestmark = pytest.mark.gpu


def _with_workspace(dsq, qtype, wg, N, K, xg, M):
    y = torch.full((M, N), float("nan"), dtype=torch.float32, device="cuda")
    nbytes = dsq.dsq_prefill_workspace_bytes(qtype, N, K, M)
    ws = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    dsq.dsq_gemm_prefill(qtype, wg, N, K, xg, M, y, ws, nbytes)
    return y


def test_noalloc_matches_workspace_entry_point_on_two_calls(dsq, ref):
    cases = [(8, 512, 1024, 64),      # K-split: the scratch also holds fp32 partials
             (12, 384, 2048, 300)]    # two token tiles, no split
    for qtype, N, K, M in cases:      # two calls in a row share the one scratch array
        w = ref.quantize(qtype, synth.weights(500 + M, N, K))
        x = synth.activations(501 + M, M, K)
        wg, xg = to_dev(w), to_dev(x)
        y_na = torch.full((M, N), float("nan"), dtype=torch.float32, device="cuda")
        dsq.dsq_gemm_prefill_noalloc(qtype, wg, N, K, xg, M, y_na)
        y_ws = _with_workspace(dsq, qtype, wg, N, K, xg, M)
        torch.cuda.synchronize()
        a = y_na.cpu().numpy()
        assert np.isfinite(a).all()
        # the same plan and kernels on the same inputs: identical bits
        assert torch.equal(y_na, y_ws)
        y64 = ref.prefill_f64(qtype, w, K, x)
        assert np.linalg.norm(a.astype(np.float64) - y64) / np.linalg.norm(y64) <= PREFILL_TOL
    assert dsq.dsq_device_status() == 0


def test_noalloc_refuses_problems_beyond_its_scratch(dsq):
    from block_quantized_dsq_b200 import DsqError
    N, K, M = 256, 8192, 4096                     # fp16 activations alone: 64 MiB
    assert dsq.dsq_prefill_workspace_bytes(8, N, K, M) > dsq.DSQ_PREFILL_NOALLOC_SCRATCH_BYTES
    w = torch.zeros((N, dsq.dsq_row_bytes(8, K)), dtype=torch.uint8, device="cuda")
    x = torch.zeros((M, K), dtype=torch.float32, device="cuda")
    y = torch.zeros((M, N), dtype=torch.float32, device="cuda")
    before = dsq.dsq_launch_count()
    with pytest.raises(DsqError) as ei:
        dsq.dsq_gemm_prefill_noalloc(8, w, N, K, x, M, y)
    assert ei.value.status == 5 and "scratch" in str(ei.value)
    assert dsq.dsq_launch_count() == before
