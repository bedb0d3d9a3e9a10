import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) and the built CUDA library")
    config.addinivalue_line("markers", "slow: long CPU work (full-size oracle)")
    # The boundary tests load libmls.so; build it in-tree when it is missing
    # (nvcc cross-compiles without a GPU).
    try:
        from lm_head_loss_junction_b200 import build
        if not os.path.exists(build.LIB):
            build.build(force=True)
    except Exception as exc:  # the tests that need the library then fail with its error
        sys.stderr.write(f"libmls.so could not be built: {exc}\n")


def pytest_collection_modifyitems(config, items):
    try:
        import torch
        have_gpu = torch.cuda.is_available()
    except Exception:
        have_gpu = False
    if have_gpu:
        return
    skip = pytest.mark.skip(reason="no CUDA device")
    for it in items:
        if "gpu" in it.keywords:
            it.add_marker(skip)
