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


def pytest_terminal_summary(terminalreporter, exitstatus, config):
    """Worst float error per (config, tap) of the parity tests that ran, against the bounds."""
    try:
        from tests.harness import MARGINS, TOL_MAX_REL, TOL_REL_L2
    except Exception:
        return
    if not MARGINS:
        return
    tr = terminalreporter
    tr.section("parity margins (worst over the tests that ran)")
    tr.write_line(f"{'config':44s} {'tap':6s} {'rel L2':>10s} {'of bound':>9s} {'max rel':>10s} {'of bound':>9s}")
    for (cfg, tap), (r, m) in sorted(MARGINS.items()):
        tr.write_line(f"{cfg:44s} {tap:6s} {r:10.3e} {r / TOL_REL_L2:9.3f} {m:10.3e} {m / TOL_MAX_REL:9.3f}")
    path = os.environ.get("MOEDEC_PARITY_REPORT")
    if path:
        import json
        with open(path, "w") as f:
            json.dump([{"config": c, "tap": t, "rel_l2": r, "max_rel": m} for (c, t), (r, m) in sorted(MARGINS.items())],
                      f, indent=1)
