import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200)")


def pytest_collection_modifyitems(config, items):
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


def pytest_terminal_summary(terminalreporter):
    """Error statistics of the cancelling-sum parity checks of this session
    (attention output and gradients): max |error|, max and median error in
    bf16 ulps of the oracle value, elements that needed the term allowance,
    the largest per-head relative L2 error, and each check's worst margin
    (1.0 = at its bound).  With LH_PARITY_STATS=path they are also written
    there as JSON."""
    try:
        from tests.helpers import STATS
    except Exception:  # pragma: no cover
        return
    if not STATS:
        return
    tr = terminalreporter
    tr.section("parity error statistics (cancelling sums)")
    tr.write_line(f"{'check':46s} {'elems':>8s} {'max|err|':>9s} {'max ulp':>8s} {'med ulp':>7s} "
                  f"{'n_term':>7s} {'headL2':>8s} {'m_elem':>6s} {'m_row':>6s} {'m_head':>6s}")
    for s in STATS:
        tr.write_line(f"{s['what'][:46]:46s} {s['elements']:8d} {s['max_abs_err']:9.2e} "
                      f"{s['max_bf16_ulp_err']:8.1f} {s['median_bf16_ulp_err']:7.2f} "
                      f"{s['n_term_allowance']:7d} {s['head_rel_l2']:8.2e} {s['elem_margin']:6.3f} "
                      f"{s['row_margin']:6.3f} {s['head_margin']:6.3f}")
    path = os.environ.get("LH_PARITY_STATS")
    if path:
        import json
        with open(path, "w") as f:
            json.dump(STATS, f, indent=1)
