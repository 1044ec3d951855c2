import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long-running CPU check")


@pytest.fixture(scope="session")
def oracle_mod():
    import oracle
    oracle.build()
    return oracle


def pytest_terminal_summary(terminalreporter, exitstatus, config):
    """Draft parity of the session: positions compared, oracle near ties, mismatches."""
    try:
        from helpers import PARITY_LOG
    except Exception:
        return
    if not PARITY_LOG:
        return
    tr = terminalreporter
    tr.write_sep("-", "draft parity (every position, oracle teacher-forced on the GPU's tokens)")
    for name, c in PARITY_LOG:
        tr.write_line(f"{name}: compared {c.compared}, near ties {c.near_ties}, "
                      f"hard mismatches {c.hard_mismatch}, max |logit err| {c.max_logit_err:.2e}")
