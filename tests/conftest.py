import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (sm_100a) and the built CUDA library")
    config.addinivalue_line("markers", "slow: full-size workload checks")


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


def pytest_terminal_summary(terminalreporter, exitstatus, config):
    """Log of the index-set comparisons: how many sets were compared and how many
    differed from the oracle's inside the near-tie band (norms within 1e-5
    relative of the k-th largest)."""
    try:
        from parity import NEAR_TIE_LOG
    except Exception:  # pragma: no cover
        return
    if not NEAR_TIE_LOG:
        return
    sets = len(NEAR_TIE_LOG)
    differing = [(w, k, t) for w, k, t in NEAR_TIE_LOG if t]
    total = sum(t for _, _, t in differing)
    terminalreporter.write_line(f"index sets compared with the oracle: {sets}; sets with near-tie differences: "
                                f"{len(differing)}; indices swapped inside the band: {total}")
    for w, k, t in differing[:20]:
        terminalreporter.write_line(f"  {w}: {t} of k={k}")
