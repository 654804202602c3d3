import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) and the built CUDA library")
    config.addinivalue_line("markers", "slow: large-size case (minutes)")
    # a fresh checkout has no libflide.so: build it (nvcc cross-compiles for
    # sm_100a without a GPU) so the ABI and host-logic tests can load it
    from tree_forked_decision_b200 import build as flide_build
    if not os.path.exists(flide_build.LIB):
        try:
            flide_build._nvcc()
        except RuntimeError:
            return  # no toolchain: the tests that need the library report it
        flide_build.build()


def pytest_collection_modifyitems(config, items):
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
