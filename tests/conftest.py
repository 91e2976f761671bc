import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) and the built libxkv.so")
    config.addinivalue_line("markers", "slow: CPU test that takes more than ~20 s")


def pytest_collection_modifyitems(config, items):
    # GPU tests cannot run without a device; skip them instead of erroring so a
    # plain `pytest` on a CPU machine stays green.
    try:
        import torch
        have_gpu = torch.cuda.is_available()
    except Exception:  # pragma: no cover
        have_gpu = False
    if have_gpu:
        return
    skip = pytest.mark.skip(reason="no CUDA device")
    for it in items:
        if "gpu" in it.keywords:
            it.add_marker(skip)


def build_xkv():
    """Build libxkv.so (if stale) without importing the package, then import it."""
    import importlib.util
    path = os.path.join(ROOT, "cross_layer_rank_b200", "build.py")
    spec = importlib.util.spec_from_file_location("_xkv_build", path)
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    mod.build()
    import cross_layer_rank_b200
    return cross_layer_rank_b200


@pytest.fixture(scope="session")
def xkv():
    return build_xkv()
