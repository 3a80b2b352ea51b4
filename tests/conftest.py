import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) and the CUDA library")
    config.addinivalue_line("markers", "slow: long CPU test")


def pytest_collection_modifyitems(config, items):
    try:
        import torch
        has_gpu = torch.cuda.is_available()
    except Exception:  # pragma: no cover
        has_gpu = False
    if has_gpu:
        return
    skip = pytest.mark.skip(reason="no CUDA device")
    for it in items:
        if "gpu" in it.keywords:
            it.add_marker(skip)


def pytest_terminal_summary(terminalreporter):
    """Report the rows the GPU parity tests left out as near a discontinuity
    (their largest fraction against the expected one)."""
    mod = sys.modules.get("parity_util")
    FLAG_LOG = getattr(mod, "FLAG_LOG", None)
    if not FLAG_LOG:
        return
    worst = max(FLAG_LOG, key=lambda r: r[1])
    tot_rows = sum(r[3] for r in FLAG_LOG)
    tot_flag = sum(r[1] * r[3] for r in FLAG_LOG)
    terminalreporter.write_line(
        f"parity: {len(FLAG_LOG)} comparisons, flagged rows {tot_flag / tot_rows:.4%} of "
        f"{tot_rows}; largest {worst[1]:.4%} (expected {worst[2]:.4%}) in {worst[0]}")
