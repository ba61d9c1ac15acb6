import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)
GOLDEN = os.path.join(ROOT, "tests", "golden")


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long-running CPU test")


@pytest.fixture(scope="session")
def golden_dir():
    return GOLDEN


def pytest_terminal_summary(terminalreporter, exitstatus, config):
    """Print the boundary-window mismatch counts of the code parity checks."""
    tq_testlib = sys.modules.get("tq_testlib")
    if tq_testlib is None:
        return
    rep = tq_testlib.MISMATCH_REPORT
    if not rep:
        return
    tr = terminalreporter
    tr.section("code/sign mismatches inside the 1e-5 boundary window")
    tr.write_line(f"{'test':70s} {'coords':>11s} {'code mism':>9s} {'sign mism':>9s} "
                  f"{'code win':>8s} {'sign win':>8s} {'fraction':>10s}")
    tot = dict(coords=0, code_mism=0, sign_mism=0, code_window=0, sign_window=0)
    for r in rep:
        tr.write_line(f"{r['test'][-70:]:70s} {r['coords']:11d} {r['code_mism']:9d} {r['sign_mism']:9d} "
                      f"{r['code_window']:8d} {r['sign_window']:8d} {r['fraction']:10.2e}")
        for k in tot:
            tot[k] += r[k]
    frac = (tot["code_mism"] + tot["sign_mism"]) / max(1, tot["coords"])
    tr.write_line(f"{'total':70s} {tot['coords']:11d} {tot['code_mism']:9d} {tot['sign_mism']:9d} "
                  f"{tot['code_window']:8d} {tot['sign_window']:8d} {frac:10.2e}  (cap 1e-4)")
