import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (sm_100a) and the built library")
    config.addinivalue_line("markers", "slow: full-size workloads (minutes of input generation)")


def pytest_collection_modifyitems(config, items):
    """GPU tests are skipped in a process that has no CUDA device (the CPU container)."""
    import torch

    if torch.cuda.is_available():
        return
    skip = pytest.mark.skip(reason="no CUDA device in this process")
    for item in items:
        if "gpu" in item.keywords:
            item.add_marker(skip)


def pytest_terminal_summary(terminalreporter):
    """How the GPU parity tests used the top-k tie band (rows checked, swaps, widening)."""
    helpers = sys.modules.get("gpu_helpers")
    if helpers is None or not helpers.BAND_STATS["rows"]:
        return
    st = helpers.BAND_STATS
    terminalreporter.write_line(
        f"tie band: {st['rows']} selections checked, {st['floor_binding']} where the fp32 floor exceeded "
        f"1e-4 |s_n|, {st['swapped']} (row, layer) outputs compared with a set that differs inside the band, "
        f"largest tolerance widening {st['max_widening']:.3g}")
