import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) GPU and the built CUDA library")
    config.addinivalue_line("markers", "slow: takes more than a few seconds")


def pytest_collection_modifyitems(config, items):
    # GPU tests cannot run without a GPU; skip them loudly instead of failing on
    # a CPU-only machine when the user did not deselect them.
    try:
        import torch
        has_gpu = torch.cuda.is_available()
    except Exception:  # pragma: no cover
        has_gpu = False
    if has_gpu:
        return
    skip = pytest.mark.skip(reason="no CUDA device on this machine")
    for item in items:
        if "gpu" in item.keywords:
            item.add_marker(skip)


def pytest_terminal_summary(terminalreporter):
    """After a GPU run: how close the checked outputs came to the parity bound."""
    gu = sys.modules.get("gpu_util")
    log = getattr(gu, "PARITY_LOG", None) if gu else None
    if not log:
        return
    worst = max(log, key=lambda r: r[1])
    terminalreporter.write_sep("-", "parity against the oracle")
    terminalreporter.write_line(
        f"{len(log)} checks, {sum(r[3] for r in log)} elements compared; worst max err/tol "
        f"{worst[1]:.3f} ({worst[0]}); largest fraction of elements above half the tolerance "
        f"{max(r[2] for r in log):.4f}")
