import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a) and the built library")


def pytest_collection_modifyitems(config, items):
    # GPU tests are skipped (not failed) on a host without a CUDA device only when
    # the caller did not ask for them explicitly with -m gpu.
    try:
        import torch
        has_gpu = torch.cuda.is_available()
    except Exception:  # pragma: no cover
        has_gpu = False
    if has_gpu:
        return
    marker = config.getoption("-m") or ""
    if "gpu" in marker and "not gpu" not in marker:
        return
    skip = pytest.mark.skip(reason="no CUDA device")
    for item in items:
        if "gpu" in item.keywords:
            item.add_marker(skip)


def pytest_terminal_summary(terminalreporter):
    """One line per parity configuration: tiles compared with the oracle, near-tie swaps
    (kept sets that differ from the oracle's only between candidates whose oracle group
    scores are within 1e-3; those tiles are re-scored with the library's selection) and
    the output error.  Printed for -q runs too."""
    mod = sys.modules.get("parity_helpers")
    if mod is None or not getattr(mod, "REPORT", None):
        return
    rows = {}
    for label, st in mod.REPORT:
        if st.tiles == 0:
            continue
        r = rows.setdefault(label, [0, 0, 0.0, 0.0, 0])
        r[0] += st.tiles
        r[1] += st.near_ties
        r[2] = max(r[2], st.max_abs)
        r[3] += st.sum_abs
        r[4] += st.count
    if not rows:
        return
    tw = terminalreporter
    tw.write_sep("-", "parity vs oracle: tiles, near-tie swaps, max/mean |diff|")
    tot_t = tot_n = 0
    for label, (t, n, mx, sm, c) in rows.items():
        tot_t += t
        tot_n += n
        tw.write_line(f"{label}: tiles={t} near_ties={n} max_abs={mx:.2e} mean_abs={sm / max(c, 1):.2e}")
    tw.write_line(f"parity total: {len(rows)} configurations, {tot_t} tiles, {tot_n} near-tie swaps")
