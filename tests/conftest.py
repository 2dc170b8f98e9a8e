import json
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


def pytest_collection_modifyitems(config, items):
    try:
        import torch
        have_gpu = torch.cuda.is_available()
    except Exception:  # pragma: no cover
        have_gpu = False
    if have_gpu:
        return
    skip = pytest.mark.skip(reason="no CUDA device")
    for item in items:
        if "gpu" in item.keywords:
            item.add_marker(skip)


def pytest_terminal_summary(terminalreporter):
    """Margins of every CUDA-vs-oracle comparison of this run (worst first)."""
    try:
        from kda_check import RECORDS
    except ImportError:  # pragma: no cover
        return
    if not RECORDS:
        return
    rows = sorted(RECORDS, key=lambda r: -r[3])
    tr = terminalreporter
    tr.section("parity margins (error / bound; 1.0 = at the tolerance)")
    tr.write_line(f"{'comparison':60s} {'max_abs':>10s} {'max_rel':>10s} {'err/bound':>9s}")
    for what, ma, mr, ratio in rows[:40]:
        tr.write_line(f"{what[:60]:60s} {ma:10.3e} {mr:10.3e} {ratio:9.3f}")
    tr.write_line(f"{len(rows)} comparisons; worst error/bound {rows[0][3]:.3f} ({rows[0][0]})")
    path = os.environ.get("KDA_MARGINS_FILE")
    if path:   # every record, for the run's evidence
        with open(path, "w") as f:
            json.dump([{"what": w, "max_abs": a, "max_rel": r, "err_over_bound": q} for w, a, r, q in rows], f, indent=0)
