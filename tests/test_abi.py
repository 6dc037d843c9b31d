"""The C-ABI library builds for sm_100a, loads without a GPU and exports every declared symbol."""
import ctypes
import os
import re

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared(header):
    text = open(os.path.join(ROOT, "include", header)).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return re.findall(r"MOEDEC_API\s+[\w\s\*]+?\b(moedec_\w+)\s*\(", text)


def test_library_exports_every_declared_symbol():
    from tests.conftest import build_library
    so = build_library()
    lib = ctypes.CDLL(so)
    names = _declared("moedec.h")
    assert {"moedec_create", "moedec_step", "moedec_destroy"} <= set(names)
    for n in names:
        assert hasattr(lib, n), f"{n} declared in include/moedec.h but not exported"


def test_status_strings_and_argument_checks_without_gpu():
    import moe_decode_layer_moedec_b200 as m
    assert m.lib.moedec_status_string(0) == b"MOEDEC_OK"
    assert m.lib.moedec_status_string(-2) == b"MOEDEC_ERR_UNSUPPORTED"
    # NULL arguments are rejected before any CUDA call
    h = ctypes.c_void_p()
    assert m.lib.moedec_create(None, None, ctypes.byref(h)) == -1
    assert m.lib.moedec_step(None, None, 1, None, None) == -1
    assert m.lib.moedec_destroy(None) == 0
    cfg = m._Config(m.ABI_VERSION + 1, 512, 256, 64, 4, 256, 256, 1, 1, 0)
    w = m._Weights()
    assert m.lib.moedec_create(ctypes.byref(cfg), ctypes.byref(w), ctypes.byref(h)) == -1
    cfg = m._Config(m.ABI_VERSION, 500, 256, 64, 4, 256, 256, 1, 1, 0)  # H not a multiple of 128
    assert m.lib.moedec_create(ctypes.byref(cfg), ctypes.byref(w), ctypes.byref(h)) == -2


def test_product_package_does_not_reach_the_oracle():
    pkg = os.path.join(ROOT, "moe_decode_layer_moedec_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h", ".cpp")):
                src = open(os.path.join(dirpath, f)).read()
                assert "oracle" not in re.sub(r"#.*|//.*", "", src), f"{f} mentions the oracle"
