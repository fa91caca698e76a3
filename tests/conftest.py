import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (sm_100a) and the built library")
    config.addinivalue_line("markers", "slow: larger CPU cases")


@pytest.fixture(scope="session")
def cuda_device():
    import torch
    if not torch.cuda.is_available():
        pytest.fail("GPU test collected on a machine without CUDA")
    return torch.device("cuda:0")


def pytest_terminal_summary(terminalreporter):
    """Worst tolerance margins of the GPU parity comparisons (1.0 = at the
    tolerance: atol 1e-2 + rtol 1e-2 |ref| for outputs, 1e-4 max(1, |lse|) for
    LSE), grouped by the first word of each comparison's label."""
    helpers = sys.modules.get("_pkv_helpers")
    if helpers is None or not getattr(helpers, "MARGINS", None):
        return
    terminalreporter.write_sep("-", "worst tolerance margins (error / tolerance)")
    for key, (mo, ml) in sorted(helpers.MARGINS.items()):
        terminalreporter.write_line(f"{key:>24}: out {mo:.3f}  lse {ml:.3f}")
