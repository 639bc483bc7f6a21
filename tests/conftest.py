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
def has_gpu():
    import torch
    return torch.cuda.is_available()


# Metrics a test reports beside its pass/fail criterion (for example the
# elementwise relative error of an output), printed at the end of the run.
_REPORTED = {}


@pytest.fixture
def report_metric():
    def record(name, value):
        _REPORTED.setdefault(name, []).append(float(value))
    return record


def pytest_terminal_summary(terminalreporter):
    if not _REPORTED:
        return
    terminalreporter.section("reported metrics (max over the cases that report them)")
    for name, values in sorted(_REPORTED.items()):
        terminalreporter.write_line("%s: max %.3e over %d cases" % (name, max(values), len(values)))

