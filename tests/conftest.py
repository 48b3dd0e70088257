import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line(
        "markers", "gpu: needs a CUDA device (B200, sm_100a); run with -m gpu")
    config.addinivalue_line(
        "markers", "slow: long-running CPU test")


def pytest_terminal_summary(terminalreporter):
    """Parity figures of the GPU tests (rows compared with the oracle,
    near-ties, validated swaps, worst output error), so that they show in a
    quiet run's last lines: one total, then the full-size workloads."""
    try:
        from oracle.parity import RECORDS
    except ImportError:
        return
    if not RECORDS:
        return
    tr = terminalreporter
    rows = sum(r["rows"] for r in RECORDS)
    near = sum(r["near_ties"] for r in RECORDS)
    swapped = sum(r["swapped"] for r in RECORDS)
    tr.write_sep("-", "parity against the CPU oracle")
    for tol in sorted({r["tol"] for r in RECORDS}):
        sub = [r for r in RECORDS if r["tol"] == tol]
        tr.write_line(
            f"tol {tol:g}: {len(sub)} comparisons, "
            f"{sum(r['rows'] for r in sub)} rows, worst max-abs "
            f"{max(r['max_abs_err'] for r in sub):.3g}")
    tr.write_line(f"all: {len(RECORDS)} comparisons, {rows} rows, "
                  f"{near} near-tie rows, {swapped} validly swapped sets")
    for r in RECORDS:
        if any(s in r["where"] for s in ("131k", "_1m", "8k", "32k", "tiny")):
            tr.write_line(f"{r['where'].split('::')[-1]}: rows {r['rows']}, "
                          f"near-ties {r['near_ties']}, swapped "
                          f"{r['swapped']}, max-abs {r['max_abs_err']:.3g}")
