import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


@pytest.fixture(scope="session")
def oracle():
    from oracle import oracle as O
    O.build()
    return O


def has_gpu():
    import torch
    return torch.cuda.is_available()


@pytest.fixture(scope="session")
def lib():
    """The CUDA binding; GPU tests only."""
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from bit_quantized_attention_smoothing_b200 import qattn as Q
    Q.load()
    return Q


def np16(t):
    """fp16 torch tensor (any device) -> contiguous numpy uint16 bit patterns."""
    import numpy as np
    return t.detach().contiguous().cpu().numpy().view(np.uint16)


def out_errors(gpu_out_rows, ref64_rows):
    """(max-abs, mean-abs) error of fp16 GPU rows against the oracle's unrounded float64 rows."""
    import numpy as np
    g = gpu_out_rows.astype(np.float64)
    e = np.abs(g - ref64_rows)
    return float(e.max()), float(e.mean())


# Output tolerances of the forward against the oracle's unrounded float64 output.
MAX_ABS_TOL = 2e-3
MEAN_ABS_TOL = 2e-4


def check_output(gpu_out_rows, ref64_rows):
    """Applies the output tolerance; returns (ok, message).

    mean |O_gpu - O64| <= 2e-4 over all elements, and max |O_gpu - O64| <= 2e-3 for every
    element with |O64| < 4.  The output is fp16, whose own rounding (half the spacing of the fp16
    grid) is 1.95e-3 for |O| in [4, 8): there the budget is 2e-3 on top of that half-spacing."""
    import numpy as np
    g = gpu_out_rows.astype(np.float64)
    r = np.asarray(ref64_rows, dtype=np.float64)
    e = np.abs(g - r)
    half_ulp = np.spacing(np.abs(r).astype(np.float16)).astype(np.float64) / 2
    big = np.abs(r) >= 4.0
    allow = np.where(big, MAX_ABS_TOL + half_ulp, MAX_ABS_TOL)
    excess = e - allow
    i = int(np.argmax(excess))
    mean = float(e.mean())
    msg = (f"max-abs {e.max():.3e} (|O|={abs(r.flat[int(np.argmax(e))]):.3f}), worst vs allowance "
           f"{e.flat[i]:.3e} <= {allow.flat[i]:.3e} at |O|={abs(r.flat[i]):.3f}, mean-abs "
           f"{mean:.3e}, elements with |O|>=4: {int(big.sum())}")
    return bool(excess.max() <= 0 and mean <= MEAN_ABS_TOL), msg
