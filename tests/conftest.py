import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (sm_100a) and the built CUDA library")


def pytest_collection_modifyitems(config, items):
    try:
        import torch
        have_gpu = torch.cuda.is_available()
    except Exception:  # pragma: no cover
        have_gpu = False
    if have_gpu:
        return
    skip = pytest.mark.skip(reason="no CUDA GPU in this process")
    for it in items:
        if "gpu" in it.keywords:
            it.add_marker(skip)


def pytest_terminal_summary(terminalreporter):
    """Parity record of this session: every element whose error exceeded 1e-2
    (allowed only at |oracle| >= 4, tests/_tol.py) is counted and listed."""
    try:
        from tests import _tol
    except Exception:  # pragma: no cover
        return
    rec = _tol.RECORD
    if not rec:
        return
    tr = terminalreporter
    n_el = sum(r[1] for r in rec)
    above = [r for r in rec if r[4]]
    failed = [r for r in rec if r[5]]
    tr.write_line(f"parity: {len(rec)} oracle comparisons, {n_el} outputs, worst max abs "
                  f"{max(r[2] for r in rec):.3e}, worst mean abs {max(r[3] for r in rec):.3e}; "
                  f"{sum(r[4] for r in above)} output(s) above 1e-2 in {len(above)} comparison(s)"
                  + (f"; {len(failed)} comparison(s) FAILED" if failed else ""))
    for what, n, mx, mean, a, bad in above + [r for r in failed if not r[4]]:
        tr.write_line(f"  {'FAILED ' if bad else ''}{what}: {a} of {n} above 1e-2, max {mx:.3e}, mean {mean:.3e}")
