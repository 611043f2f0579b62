import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


@pytest.fixture(scope="session")
def golden():
    import json

    def load(name):
        with open(os.path.join(ROOT, "tests", "golden", name), encoding="utf-8") as f:
            return json.load(f)
    return load


def pytest_terminal_summary(terminalreporter):
    """The fp32 parity checks' literal relative errors next to the 1e-5 * mag reading."""
    try:
        import tolerances
    except ImportError:
        return
    if not tolerances.REPORTS:
        return
    tr = terminalreporter
    tr.write_line("fp32 parity: max |gpu-ref|/mag (bound 1e-5) | max |gpu-ref|/|ref| where |ref| >= 1e-2 mag")
    for what, c21, lit, n in tolerances.REPORTS:
        tr.write_line(f"  {what}: {c21:.3g} | {lit:.3g} over {n} outputs")
