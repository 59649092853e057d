import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long-running CPU test")


@pytest.fixture(scope="session")
def oracle_mod():
    import oracle
    oracle.build()
    return oracle


def pytest_terminal_summary(terminalreporter):
    """Print the errors the parity comparisons measured (what, max-abs, rel-F)."""
    try:
        from parity import MEASURED
    except ImportError:
        return
    if not MEASURED:
        return
    terminalreporter.write_sep("-", "measured errors (max-abs, rel-F)")
    for what, max_abs, rel_f in MEASURED:
        terminalreporter.write_line(f"{what}: max-abs {max_abs:.3e}  rel-F {rel_f:.3e}")
