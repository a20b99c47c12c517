import json
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

GOLDEN = os.path.join(ROOT, "tests", "golden")


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) and the built libdsq")
    config.addinivalue_line("markers", "slow: full-size parity cases")


def load_golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


@pytest.fixture(scope="session")
def ref():
    import oracle
    oracle.lib()
    return oracle


@pytest.fixture(scope="session")
def dsq():
    """libdsq on a real device.  Skips only when no CUDA device exists; a
    missing or broken library is an error (there is no fallback)."""
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from block_quantized_dsq_b200 import build
    build.build()
    import block_quantized_dsq_b200 as dsq
    dsq.lib()
    torch.cuda.init()
    return dsq


def to_dev(a):
    import numpy as np
    import torch
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def gemv_error(y, y_ref, absum, nterms):
    """max_n |y - y_ref| / max(|y_ref|, absum / sqrt(nterms)): relative error
    with the summation's condition scale as the floor of the denominator."""
    import numpy as np
    y = np.asarray(y, np.float64)
    denom = np.maximum(np.abs(y_ref), absum / np.sqrt(nterms))
    denom = np.where(denom > 0, denom, 1.0)
    return float(np.max(np.abs(y - y_ref) / denom)) if y.size else 0.0


def plain_rel_error(y, y_ref):
    """max relative error over outputs with |y_ref| >= 0.1 * rms(y_ref)."""
    import numpy as np
    y = np.asarray(y, np.float64)
    if y.size == 0:
        return 0.0
    rms = np.sqrt(np.mean(y_ref ** 2))
    sel = np.abs(y_ref) >= 0.1 * rms
    if not sel.any():
        return 0.0
    return float(np.max(np.abs(y[sel] - y_ref[sel]) / np.abs(y_ref[sel])))


GEMV_TOL = 1e-5       # max relative error (GEMV), see gemv_error
PREFILL_TOL = 2e-3    # relative L2 vs the fp64 dequantized reference
PREFILL_ROUNDED_TOL = 1e-5   # relative L2 vs the operand-rounded reference
