import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) GPU and the built CUDA library")
    config.addinivalue_line("markers", "slow: long-running CPU test")


def pytest_terminal_summary(terminalreporter):
    """Print the observed output errors of every parity comparison."""
    try:
        from tests import parity
    except ImportError:
        return
    if not parity.RECORDS:
        return
    tr = terminalreporter
    tr.write_sep("-", "attention output vs the oracle: observed errors")
    tr.write_line(f"{'case':<58} {'dtype':<5} {'max-abs':>10} {'bound':>7} {'rel-L2':>10} {'bound':>7} {'rms(want)':>10}")
    for r in parity.RECORDS:
        tr.write_line(f"{r['case'][:58]:<58} {r['dtype']:<5} {r['max_abs']:>10.3g} {r['max_abs_bound']:>7.0e} "
                      f"{r['rel_l2']:>10.3g} {r['rel_l2_bound']:>7.0e} {r['want_rms']:>10.3g}")
