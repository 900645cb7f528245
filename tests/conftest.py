import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long-running (full-size workloads)")


# Parity margins of the full-size checks: each test that asks for `margins` appends
# (name, out error, final_state error, bar); the table is printed at the end of the run,
# also under -q, so that a run's log shows how far each case sits from its bar.
@pytest.fixture(scope="session")
def margins(request):
    log = getattr(request.config, "_dn_margins", None)
    if log is None:
        log = []
        request.config._dn_margins = log
    return log


def pytest_terminal_summary(terminalreporter, exitstatus, config):
    log = getattr(config, "_dn_margins", None)
    if not log:
        return
    terminalreporter.write_sep("-", "parity margins: max|x - x_ref| / max|x_ref| (bar)")
    for name, eo, es, bar in log:
        es_s = f"{es:.3e}" if es is not None else "-"
        terminalreporter.write_line(f"{name:<40s} out {eo:.3e}  final_state {es_s}  (bar {bar:g})")
