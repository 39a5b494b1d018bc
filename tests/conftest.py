"""Shared pytest configuration: the `gpu` marker and import paths."""
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


def pytest_collection_modifyitems(config, items):
    try:
        import torch
        has_gpu = torch.cuda.is_available()
    except Exception:  # pragma: no cover
        has_gpu = False
    if has_gpu:
        return
    skip = pytest.mark.skip(reason="no CUDA device in this process")
    for item in items:
        if "gpu" in item.keywords:
            item.add_marker(skip)


def pytest_terminal_summary(terminalreporter):
    """The gradient tests' effective bars: for each compared tensor, the observed max and
    mean error, the bar applied, and which of the fixed bar and the rounding model's
    (1.5 x its own error) set it."""
    try:
        from parity import GRAD_LOG
    except ImportError:  # pragma: no cover
        return
    if not GRAD_LOG:
        return
    tr = terminalreporter
    tr.section("gradient bars (observed / applied; 'model' = set by the rounding model)")
    for s in GRAD_LOG:
        src_max = "model" if s["max_bar"] > s["fixed_max_bar"] else "fixed"
        src_mean = "model" if s["mean_bar"] > s["fixed_mean_bar"] else "fixed"
        tr.write_line(f"max {s['max_abs']:.3e} / {s['max_bar']:.3e} ({src_max}, "
                      f"{s['max_abs'] / s['max_bar']:.2f})   mean {s['mean_abs']:.3e} / "
                      f"{s['mean_bar']:.3e} ({src_mean}, {s['mean_abs'] / s['mean_bar']:.2f})")
