import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) and the built CUDA library")
    config.addinivalue_line("markers", "slow: long CPU work (full-size oracle)")
    # The boundary and GPU tests load libmls.so; build it in-tree when it is
    # missing or was built from other sources than the ones in the tree (a
    # content hash, so a copied tree keeps its library; nvcc cross-compiles
    # without a GPU).
    try:
        from lm_head_loss_junction_b200 import build
        build.build()
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
