import os
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long-running GPU parity case")


def pytest_collection_modifyitems(config, items):
    try:
        import torch
        have_gpu = torch.cuda.is_available()
    except Exception:  # pragma: no cover
        have_gpu = False
    if have_gpu:
        return
    skip = pytest.mark.skip(reason="no CUDA device in this process")
    for item in items:
        if "gpu" in item.keywords:
            item.add_marker(skip)


def pytest_terminal_summary(terminalreporter):
    """The measured code-mismatch rates of the GPU decode comparisons in this run (one line per
    test label): worst and mean over steps of the share of integer codes one step off."""
    try:
        from tests.helpers import RATES
    except Exception:  # pragma: no cover
        return
    rows = [r for r in RATES if r.get("label")]
    if not rows:
        return
    tr = terminalreporter
    tr.write_sep("-", "decode code-mismatch rates (share of integer codes one step off)")
    by = {}
    for r in rows:
        by.setdefault(r["label"], []).append(r)
    for label, rs in by.items():
        gs = [r["at_gpu_scales"] for r in rs if r["at_gpu_scales"] is not None]
        tr.write_line(
            f"{label}: steps {len(rs)}, codes {sum(r['n_codes'] for r in rs)}; at the GPU's scales max "
            f"{max(gs) if gs else float('nan'):.2e}; vs the reference codes max {max(r['raw'] for r in rs):.2e} "
            f"mean {np.mean([r['raw'] for r in rs]):.2e}; vs the oracle's own codes max "
            f"{max(r['raw_own'] for r in rs):.2e}; scales differing: r {np.mean([r['r_mismatch'] for r in rs]):.2e}, "
            f"c {np.mean([r['c_mismatch'] for r in rs]):.2e}")
