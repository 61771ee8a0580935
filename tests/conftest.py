import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

GOLDEN = os.path.join(ROOT, "tests", "golden")


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


def read_golden(name):
    """Rows of whitespace-separated fields from tests/golden/<name>, comments dropped."""
    rows = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if line:
                rows.append(line.split())
    return rows


@pytest.fixture(scope="session")
def cuda_device():
    import torch

    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch.device("cuda:0")


# bf16 configurations: max-abs <= 2e-2 and mean-abs <= 2e-3 against the float64 oracle;
# fp32 configuration: max-abs <= 1e-4.
BF16_MAX_ABS, BF16_MEAN_ABS = 2e-2, 2e-3
F32_MAX_ABS = 1e-4


# (what, elements, max-abs, mean-abs) of the comparisons made with report=True, printed at
# the end of the session (also under -q) so that the log carries the measured errors.
PARITY_REPORT = []


def pytest_terminal_summary(terminalreporter):
    if not PARITY_REPORT:
        return
    terminalreporter.write_sep("-", "parity against the float64 oracle (whole outputs)")
    for what, n, mx, mean in PARITY_REPORT:
        terminalreporter.write_line(f"{what}: {n} elements, max-abs {mx:.3e}, mean-abs {mean:.3e}")


def assert_parity(got, ref, dtype="bf16", what="", report=False):
    """Element-by-element comparison of a GPU result with the float64 oracle."""
    import numpy as np

    g = got.detach().to("cpu").double().numpy() if hasattr(got, "detach") else np.asarray(got, dtype=np.float64)
    r = np.asarray(ref, dtype=np.float64)
    assert g.shape == r.shape, (g.shape, r.shape)
    assert np.all(np.isfinite(g)), f"{what}: non-finite output"
    err = np.abs(g - r)
    mx, mean = float(err.max()) if err.size else 0.0, float(err.mean()) if err.size else 0.0
    if report:
        PARITY_REPORT.append((what, int(err.size), mx, mean))
    if dtype == "bf16":
        assert mx <= BF16_MAX_ABS and mean <= BF16_MEAN_ABS, f"{what}: max-abs {mx:.3e} mean-abs {mean:.3e}"
    else:
        assert mx <= F32_MAX_ABS, f"{what}: max-abs {mx:.3e}"
    return mx, mean
