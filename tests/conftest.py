import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (sm_100a) and the built libkvc")
    config.addinivalue_line("markers", "slow: full-size workload check")


def pytest_sessionstart(session):
    """A fresh checkout has no libkvc.so (it is not versioned): build it once when nvcc is
    here, so the ABI tests and the GPU tests find it."""
    from long_context_kv_obs_b200 import build
    if os.path.exists(build.LIB):
        return
    try:
        build.nvcc()
    except RuntimeError:
        return                  # no toolchain: tests needing the library say so themselves
    build.build()


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
