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
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) and the built CUDA library")
    config.addinivalue_line("markers", "slow: full-size case (minutes)")


def pytest_terminal_summary(terminalreporter, exitstatus, config):
    """Decision flips forgiven as near-ties by the GPU parity tests."""
    try:
        from parity_helpers import CRIT_LOG, FLIP_LOG, NEAR_TIE
    except ImportError:
        return
    if not FLIP_LOG and not CRIT_LOG:
        return
    tr = terminalreporter
    tr.section("skip-decision flips (GPU vs oracle)")
    if CRIT_LOG:
        tr.write_line(f"critical values: largest |GPU - fp64| {max(e['worst'] for e in CRIT_LOG):.3e} "
                      f"over {sum(e['compared'] for e in CRIT_LOG)} tiles")
    if not FLIP_LOG:
        return
    total = sum(e["compared"] for e in FLIP_LOG)
    flips = sum(e["flips"] for e in FLIP_LOG)
    worst = max(e["worst"] for e in FLIP_LOG)
    for e in FLIP_LOG:
        if e["flips"]:
            tr.write_line(f"{e['test']}: {e['flips']} of {e['compared']} decisions flipped, "
                          f"largest |margin| {e['worst']:.3e}")
    tr.write_line(f"total: {flips} flips in {total} compared decisions over {len(FLIP_LOG)} "
                  f"checks; largest |margin| {worst:.3e} (gate NEAR_TIE = {NEAR_TIE:g})")
