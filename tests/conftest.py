import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: large workload (seconds to a minute)")


@pytest.fixture(scope="session")
def golden_dir():
    return os.path.join(ROOT, "tests", "golden")


def _tally():
    mod = sys.modules.get("parity_util")
    return None if mod is None else mod


def pytest_terminal_summary(terminalreporter):
    """Log the run-wide parity tally: decisions compared with the oracle, the
    low-margin ones, and the exempted differences among them."""
    pu = _tally()
    if pu is None or not pu.TALLY["decisions"]:
        return
    t = pu.TALLY
    terminalreporter.write_sep("-", "verify parity tally")
    terminalreporter.write_line("decisions compared: %d; low-margin (< 1e-6): %d; exempted differences: %d "
                                "(budget %d = floor(1e-5 x decisions))"
                                % (t["decisions"], len(t["low_margin"]), len(t["exempted"]),
                                   int(1e-5 * t["decisions"])))
    if not pu.exemption_budget_ok():
        terminalreporter.write_line("FAILED: more exempted differences than the run-wide budget allows")
    for e in t["low_margin"]:
        terminalreporter.write_line("  low-margin: request %d, %s at position %d, margin %.3g, GPU equal: %s" % e)


def pytest_sessionfinish(session, exitstatus):
    """The exempted differences of the whole run must stay within 1e-5 of its decisions."""
    pu = _tally()
    if pu is not None and pu.TALLY["decisions"] and not pu.exemption_budget_ok():
        session.exitstatus = pytest.ExitCode.TESTS_FAILED
