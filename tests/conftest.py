import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line(
        "markers", "gpu: needs a B200 (sm_100a) and the built libcarve.so")


def pytest_collection_modifyitems(config, items):
    # GPU tests are skipped (not failed) on a host without CUDA.
    try:
        import torch
        have_gpu = torch.cuda.is_available()
    except Exception:
        have_gpu = False
    if have_gpu:
        return
    skip = pytest.mark.skip(reason="no CUDA device on this host")
    for item in items:
        if "gpu" in item.keywords:
            item.add_marker(skip)


def pytest_terminal_summary(terminalreporter):
    """Headroom of every parity comparison of the run: the worst tensor of
    each (max|delta| / max|ref| and its share of the tolerance)."""
    mod = sys.modules.get("_parity")
    margins = getattr(mod, "MARGINS", None) if mod else None
    if not margins:
        return
    tr = terminalreporter
    tr.write_sep("-", "parity margins (max|delta| / max|ref|, worst tensor)")
    for what, tol, errs in margins:
        if not errs:
            continue
        name, worst = max(errs.items(), key=lambda kv: kv[1])
        tr.write_line("%-48s %-8s %.2e  (%3.0f%% of %.0e)" % (
            what[:48], name, worst, 100.0 * worst / tol, tol))
