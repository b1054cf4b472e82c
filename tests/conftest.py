import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: takes more than a few seconds")


@pytest.fixture(scope="session", autouse=True)
def _built_libs():
    """Build the generator libraries once (host parts are needed on CPU)."""
    import synth
    synth.build()


def pytest_terminal_summary(terminalreporter):
    """Elementwise median and maximum relative errors of every parity
    comparison that recorded them, beside the normwise metric."""
    import sys
    mod = sys.modules.get("tests.gpu_util")
    lines = mod.report_lines() if mod is not None else []
    if lines:
        terminalreporter.section("parity errors (y against the oracle)")
        for line in lines:
            terminalreporter.write_line(line)
