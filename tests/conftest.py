import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

# per-matrix parity figures collected by the full-size tests, printed in the
# run's summary (they pass silently otherwise)
_REPORT: list[str] = []


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: full-size workload checks")


def pytest_sessionfinish(session, exitstatus):
    """Under a bounds-checked build of the library (NVFP4HS_LIB pointing at
    libnvfp4hs_checked.so), a run with any failed check fails."""
    import os
    if not os.environ.get("NVFP4HS_LIB"):
        return
    import block_scale_search_b200 as nv
    if nv._lib is None or not nv.lib().nvfp4_debug_checks_compiled():
        return
    count, first = nv.nvfp4_debug_checks()
    _REPORT.append(f"bounds checks: {count} failed (first record {first:#x})")
    if count:
        session.exitstatus = 1


def pytest_terminal_summary(terminalreporter):
    if _REPORT:
        terminalreporter.section("parity per matrix")
        for line in _REPORT:
            terminalreporter.write_line(line)


@pytest.fixture(scope="session")
def parity_report():
    return _REPORT.append


@pytest.fixture(scope="session")
def orc():
    import oracle
    oracle.build()
    return oracle
