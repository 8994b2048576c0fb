import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) and the built CUDA library")


def pytest_terminal_summary(terminalreporter):
    """Worst error and worst excess over the bound of every parity check, per test."""
    try:
        from tests.gpu_util import WORST
    except ImportError:
        return
    if not WORST:
        return
    tr = terminalreporter
    tr.section("parity margins (worst error; worst excess over the bound, <= 0 passes)")
    for test in sorted(WORST):
        for check, (err, excess) in sorted(WORST[test].items()):
            tr.write_line(f"{test} | {check} | err {err:.3e} | excess {excess:+.3e}")
