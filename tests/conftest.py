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


# Output tolerances of the forward against the oracle's unrounded float64 output: max-abs 2e-3
# and mean-abs 2e-4, flat, over every compared element.
MAX_ABS_TOL = 2e-3
MEAN_ABS_TOL = 2e-4


def check_output(gpu_out_rows, ref64_rows):
    """Applies the output tolerance; returns (ok, message).

    max |O_gpu - O64| <= 2e-3 and mean |O_gpu - O64| <= 2e-4 over all compared elements, O_gpu
    the fp16 output and O64 the oracle's unrounded float64 output.  The message also reports, for
    information, the floor the fp16 output type alone sets: max and mean |fp16(O64) - O64|."""
    import numpy as np
    g = gpu_out_rows.astype(np.float64)
    r = np.asarray(ref64_rows, dtype=np.float64)
    e = np.abs(g - r)
    floor = np.abs(r.astype(np.float16).astype(np.float64) - r)
    i = int(np.argmax(e))
    mx, mean = float(e.flat[i]), float(e.mean())
    msg = (f"max-abs {mx:.3e} at |O|={abs(r.flat[i]):.3f} (fp16 floor there {floor.flat[i]:.3e}), "
           f"mean-abs {mean:.3e}; fp16 rounding floor max {floor.max():.3e} mean {floor.mean():.3e}; "
           f"elements {e.size}, over 2e-3: {int((e > MAX_ABS_TOL).sum())}")
    return bool(mx <= MAX_ABS_TOL and mean <= MEAN_ABS_TOL), msg
