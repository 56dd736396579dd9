import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (B200, sm_100a) and the built library")
    config.addinivalue_line("markers", "slow: longer CPU test")


def pytest_collection_modifyitems(config, items):
    # GPU tests are skipped (not failed) when no GPU is present, so that the
    # CPU suite can run everywhere; on a GPU machine they must run.
    try:
        import torch
        has_gpu = torch.cuda.is_available()
    except Exception:  # pragma: no cover
        has_gpu = False
    if has_gpu:
        return
    skip = pytest.mark.skip(reason="no CUDA GPU in this environment")
    for item in items:
        if "gpu" in item.keywords:
            item.add_marker(skip)


def pytest_terminal_summary(terminalreporter, exitstatus, config):
    """Measured parity errors of this session (one line per comparison)."""
    from tests._report import RESULTS
    if not RESULTS:
        return
    tr = terminalreporter
    tr.write_sep("-", f"parity errors ({len(RESULTS)} comparisons)")
    worst = max(r[1] / r[3] for r in RESULTS)
    tr.write_line(f"largest max_abs / bound: {worst:.3f}")
    for what, ma, rl, ba, br in RESULTS:
        tr.write_line(f"{what:<60s} max_abs {ma:.3e} (<= {ba:.1e})  rel_l2 {rl:.3e} (<= {br:.1e})")
