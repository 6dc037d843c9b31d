import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def build_library() -> str:
    """Build libmoedec.so in-tree if it is missing or older than its sources (nvcc cross-compiles
    for sm_100a without a GPU); returns its path.  The build script is loaded by path because
    importing the package loads the library."""
    import importlib.util
    spec = importlib.util.spec_from_file_location("moedec_build", os.path.join(ROOT, "moe_decode_layer_moedec_b200",
                                                                                "build.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod.build()


def pytest_configure(config):
    build_library()
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: CPU test that takes tens of seconds")


def cuda_available() -> bool:
    try:
        import torch
        return torch.cuda.is_available()
    except Exception:
        return False


def pytest_collection_modifyitems(config, items):
    if cuda_available():
        return
    skip = pytest.mark.skip(reason="no CUDA device")
    for item in items:
        if "gpu" in item.keywords:
            item.add_marker(skip)
