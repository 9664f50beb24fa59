import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: full-size case")


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


def pytest_terminal_summary(terminalreporter, exitstatus, config):
    """How often the GPU budget tests needed the ambiguous-cut rule."""
    mod = sys.modules.get("tests.gpu_helpers")
    if mod is None:
        return
    t = mod.AMBIG_TALLY
    if t["units"]:
        terminalreporter.write_line(
            f"budget checks: {t['units']} units, {t['ambiguous_accepts']} accepted through the "
            f"ambiguous-cut rule (widest window {t['max_window']:.3g})")
