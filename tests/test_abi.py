"""The C-ABI library loads without a GPU and exports every entry point of include/sn.h."""
import ctypes
import re
from pathlib import Path

from schnet_gnn_molecular_cell_b200 import binding, build

ROOT = Path(__file__).resolve().parents[1]


def declared_symbols():
    text = (ROOT / "include" / "sn.h").read_text()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(sn_[a-z_0-9]+)\s*\(", text)))


def test_library_builds_and_exports_every_declared_symbol():
    build.build()
    lib = ctypes.CDLL(str(build.LIB))
    names = declared_symbols()
    assert len(names) >= 10
    for n in names:
        assert hasattr(lib, n), f"{n} declared in sn.h but not exported"
    assert sorted(binding.EXPORTS) == names


def test_binding_loads_and_reports_version():
    assert binding.version().startswith("snflash")


def test_create_rejects_bad_arguments_without_touching_the_gpu():
    L = binding.load()
    h = ctypes.c_void_p()
    cfg = binding.Config(128, 50, 3, 20, 12.0, 10.0, 0)
    # NULL weights and a wrong blob size are rejected before any CUDA call
    assert L.sn_create(ctypes.byref(cfg), None, 10, None, ctypes.byref(h)) == binding.Status.INVALID_ARG
    import numpy as np
    w = np.zeros(10, np.float32)
    assert L.sn_create(ctypes.byref(cfg), w.ctypes.data, 10, None, ctypes.byref(h)) == binding.Status.INVALID_ARG
    bad = binding.Config(96, 50, 3, 20, 12.0, 10.0, 0)     # F = 96 is not built
    assert L.sn_create(ctypes.byref(bad), w.ctypes.data, 10, None, ctypes.byref(h)) == binding.Status.UNSUPPORTED
    assert h.value is None


def test_every_status_of_the_header_has_a_binding_member():
    # the binding turns every status the library can return into a Status member: an
    # enumerator missing on the Python side would raise ValueError instead of SNError
    text = (ROOT / "include" / "sn.h").read_text()
    block = text[text.index("typedef enum {"):text.index("} sn_status;")]
    block = re.sub(r"/\*.*?\*/", "", block, flags=re.S)
    pairs = re.findall(r"\b(SN_(?:OK|ERR_[A-Z_]+))\s*=\s*(\d+)", block)
    assert len(pairs) >= 9
    for name, value in pairs:
        short = name[len("SN_ERR_"):] if name.startswith("SN_ERR_") else "OK"
        assert binding.Status[short] == int(value), name
        assert isinstance(binding.SNError(int(value), "x").status, binding.Status)
