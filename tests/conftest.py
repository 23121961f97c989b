import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: full-size parity cases")


def pytest_terminal_summary(terminalreporter, exitstatus, config):
    """Near-ties across the selection cut (fp64 scores within 1e-6 relative),
    per test that compared selections with the oracle, and the largest
    |GPU - oracle| of each test that compared outputs."""
    h = sys.modules.get("gpu_harness")
    if h is None:
        return
    tr = terminalreporter
    if h.MAX_ERR:
        tr.section("largest |GPU - oracle| over outputs and log-sum-exp (bar 2e-3)")
        for label, e in sorted(h.MAX_ERR.items()):
            tr.write_line(f"{label}: {e:.2e}")
    if not h.NEAR_TIES:
        return
    tr.section("near-ties at the selection cut (fp64, 1e-6 relative)")
    tot = [0, 0, 0]
    for label, (n, with_ties, pairs) in sorted(h.NEAR_TIES.items()):
        tr.write_line(f"{label}: {n} selections compared, {with_ties} with near-ties, {pairs} pairs")
        tot = [a + b for a, b in zip(tot, (n, with_ties, pairs))]
    tr.write_line(f"total: {tot[0]} selections compared, {tot[1]} with near-ties, {tot[2]} pairs")
