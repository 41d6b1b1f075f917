import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long-running oracle statistics")


def pytest_collection_modifyitems(config, items):
    # A GPU test on a machine without CUDA is a skip, never a silent pass.
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
    # Worst ratios of the GPU results against the literal tolerances.
    try:
        from tests import parity
    except Exception:  # pragma: no cover
        return
    L = parity.LITERAL
    if L["checks"]:
        terminalreporter.write_line(
            "literal-bound ratios (worst over all checks): score err / (1e-4 |s|) where |s| >= typical scale "
            f"{L['score_rel']:.3g}; over all scores {L['score_rel_all']:.3g}; fp32 outputs max |err| / 2e-3 "
            f"{L['out_abs_f32']:.3g}; bf16 outputs max |err| / (2e-3 + half spacing) {L['out_bf16_vs_rounding']:.3g}")
