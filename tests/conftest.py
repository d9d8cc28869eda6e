import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (B200) and the built engine")
    config.addinivalue_line("markers", "slow: minutes of CPU oracle work")


@pytest.fixture(scope="session")
def tiny():
    from oracle.model import OracleModel
    from workload import CONFIGS, WeightSet

    wl = CONFIGS["tiny_d4"]
    ws = WeightSet(wl.shape, seed=0, gain_std=0.1).materialize()
    return wl, ws, OracleModel(wl.shape, ws)


def pytest_terminal_summary(terminalreporter, exitstatus, config):
    """List every parity comparison with its flagged positions and divergences."""
    try:
        from _parity import REPORT
    except ImportError:
        return
    if REPORT:
        terminalreporter.section("engine vs oracle parity (flagged near-tie positions listed)")
        for line in REPORT:
            terminalreporter.write_line(line)
