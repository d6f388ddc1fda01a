import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)
TESTS = os.path.dirname(os.path.abspath(__file__))
if TESTS not in sys.path:
    sys.path.insert(0, TESTS)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long-running CPU test")


@pytest.fixture(scope="session")
def orc():
    import oracle
    return oracle


def pytest_terminal_summary(terminalreporter):
    """The largest errors the parity comparisons observed, by what was compared."""
    helpers = sys.modules.get("gpu_helpers")
    if helpers is None:
        return
    if getattr(helpers, "NOTES", None):
        terminalreporter.section("figures reported by the tests")
        for line in helpers.NOTES:
            terminalreporter.write_line(line)
    if not getattr(helpers, "OBSERVED", None):
        return
    rows = sorted(helpers.OBSERVED, key=lambda r: -r[1])
    terminalreporter.section("observed parity errors (largest relative L2 first)")
    for what, rel, mx in rows[:40]:
        terminalreporter.write_line(f"rel-L2 {rel:.2e}  max-abs/RMS {mx:.2e}  {what}")
    terminalreporter.write_line(f"{len(rows)} comparisons")
