import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: full-size workload, minutes of CPU or GPU time")


@pytest.fixture(scope="session")
def golden_dir():
    return os.path.join(ROOT, "tests", "golden")


def pytest_terminal_summary(terminalreporter):
    """Counts of mask pairs in the parity band, per GPU mask test."""
    try:
        import amb_report
    except ImportError:
        return
    if amb_report.NOTES:
        terminalreporter.write_sep("-", "measured errors")
        for line in amb_report.NOTES:
            terminalreporter.write_line(line)
    if not amb_report.COUNTS:
        return
    tot_f = sum(c[1] for c in amb_report.COUNTS)
    tot_p = sum(c[2] for c in amb_report.COUNTS)
    terminalreporter.write_sep("-", "mask pairs in the ambiguity band (excused from bit-exactness)")
    for label, f, n in amb_report.COUNTS:
        terminalreporter.write_line("%-60s %6d of %9d" % (label, f, n))
    terminalreporter.write_line("%-60s %6d of %9d" % ("total", tot_f, tot_p))
