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
        have_gpu = torch.cuda.is_available()
    except Exception:  # pragma: no cover
        have_gpu = False
    if have_gpu:
        return
    skip = pytest.mark.skip(reason="no CUDA device")
    for item in items:
        if "gpu" in item.keywords:
            item.add_marker(skip)


def pytest_terminal_summary(terminalreporter):
    """Report how much of the band rule's slack the GPU tests actually used."""
    helpers = sys.modules.get("tests.helpers")
    if helpers is None or not helpers.BAND_STATS["codes"]:
        return
    s = helpers.BAND_STATS
    terminalreporter.write_line(
        f"band rule: {s['codes']} codes compared, {s['flips']} flipped by one at a tie "
        f"(largest distance of a flip from the tie {s['max_flip_tie_distance']:.2e}, allowed 2e-3); "
        f"largest relative int8 scale deviation {s['max_scale_rel']:.2e} (allowed 1e-4); "
        f"largest int4 fp16 scale difference {s['max_scale_fp16_ulps']:.0f} fp16 ulp (allowed 1)")
