import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) and the built CUDA library")


def pytest_terminal_summary(terminalreporter):
    # the worst attention errors per GPU test, against max-abs 2e-2, rel-L2 5e-3
    try:
        from gpu_common import MARGINS
    except Exception:
        return
    if not MARGINS:
        return
    terminalreporter.write_line("attention margins (worst max-abs, rel-L2 per test):")
    for node, (mx, rl) in sorted(MARGINS.items()):
        terminalreporter.write_line(f"  {mx:.4f} {rl:.5f}  {node}")


def pytest_collection_modifyitems(config, items):
    # GPU tests fail loudly (not skip) when a GPU exists but the library is missing;
    # without any CUDA device they are skipped so that the CPU suite stays green.
    try:
        import torch
        have_gpu = torch.cuda.is_available()
    except Exception:
        have_gpu = False
    if have_gpu:
        return
    skip = pytest.mark.skip(reason="no CUDA device in this process")
    for item in items:
        if "gpu" in item.keywords:
            item.add_marker(skip)
