import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) GPU and the built CUDA library")


@pytest.fixture(scope="session")
def oracle():
    import oracle as O
    O.build()
    return O


def pytest_terminal_summary(terminalreporter, exitstatus, config):
    """The strict (unrounded fp32 output) GEMM errors of the session, one line per check."""
    mod = sys.modules.get("gpu_util")
    rows = getattr(mod, "STRICT_RESULTS", None) if mod else None
    if not rows:
        return
    tr = terminalreporter
    tr.write_sep("-", "strict GEMM bound (fp32 output vs fp64 oracle): rel_fro <= 2e-3, "
                      "max_abs/rms <= 1e-2")
    for what, rel, mar in rows:
        tr.write_line(f"{what}: rel_fro={rel:.3e} max_abs/rms={mar:.3e}")
