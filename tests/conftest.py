import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: CPU test that takes tens of seconds")


@pytest.fixture(scope="session")
def root():
    return ROOT


# Near-threshold report: every kept-set comparison records how many blocks the oracle marked
# near the selection threshold and how many of them the GPU decided the other way; the counts are
# printed at the end of the run.
KEPT_REPORT = []


def pytest_terminal_summary(terminalreporter):
    if not KEPT_REPORT:
        return
    terminalreporter.section("kept-set comparisons (near-threshold blocks, flips)")
    for name, blocks, near, flips in KEPT_REPORT:
        terminalreporter.write_line("%-70s blocks %8d  near %4d  flips %4d" % (name, blocks, near, flips))
