import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


def pytest_collection_modifyitems(config, items):
    # Tests marked gpu cannot run without a device; fail loudly only when a GPU run
    # was asked for explicitly with -m gpu.
    try:
        import torch
        has_gpu = torch.cuda.is_available()
    except Exception:  # pragma: no cover
        has_gpu = False
    if has_gpu:
        return
    skip = pytest.mark.skip(reason="no CUDA device")
    for item in items:
        if "gpu" in item.keywords:
            item.add_marker(skip)


def pytest_terminal_summary(terminalreporter, exitstatus, config):
    """Mask rows that differ from the oracle's (each one checked to be a legal cut)."""
    import mask_report
    if not mask_report.RECORDS:
        return
    tr = terminalreporter
    tr.section("mask rows against the oracle (differing rows are legal cuts)")
    tot = [0, 0, 0]
    for what, differ, marginal, rows in mask_report.RECORDS:
        tr.write_line(f"{what}: {differ} differ, {marginal} marginal, of {rows} rows")
        tot = [tot[0] + differ, tot[1] + marginal, tot[2] + rows]
    tr.write_line(f"total: {tot[0]} differ, {tot[1]} marginal, of {tot[2]} rows")
