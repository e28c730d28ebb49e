import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)
HERE = os.path.dirname(os.path.abspath(__file__))
if HERE not in sys.path:
    sys.path.insert(0, HERE)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (B200, sm_100a) and the built library")


def pytest_collection_modifyitems(config, items):
    try:
        import torch
        have_gpu = torch.cuda.is_available()
    except Exception:  # pragma: no cover
        have_gpu = False
    if have_gpu:
        return
    skip = pytest.mark.skip(reason="no CUDA GPU in this environment")
    for item in items:
        if "gpu" in item.keywords:
            item.add_marker(skip)


def pytest_terminal_summary(terminalreporter, exitstatus, config):
    """The parity figures of every 16-bit comparison run in this session: the
    largest per-row rms error ratio and ulp error per output type, with the
    test that produced each."""
    try:
        from pagedutil import DIAGNOSTICS
    except Exception:  # pragma: no cover
        return
    rows = [d for d in DIAGNOSTICS if "rms_row_max" in d]
    if not rows:
        return
    terminalreporter.section("16-bit parity figures (max over checks)")
    for dt in sorted({d["dtype"] for d in rows}):
        mine = [d for d in rows if d["dtype"] == dt]
        r = max(mine, key=lambda d: d["rms_row_max"])
        u = max(mine, key=lambda d: d["ulp_max"])
        terminalreporter.write_line(
            f"{dt}: {len(mine)} checks; per-row rms ratio max {r['rms_row_max']:.3e} ({r['test']}); "
            f"ulp max {u['ulp_max']:.2f} ({u['test']})")
