"""The C-ABI library loads and exports every entry point the header declares; host-side
argument validation works without a GPU (no compute call is made here)."""
import ctypes
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "pi_sparse_ffn.h")


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return re.findall(r"^\s*(?:const\s+)?[A-Za-z_][A-Za-z0-9_]*\s*\*?\s*(pi_[a-z0-9_]+)\s*\(", src, flags=re.M)


@pytest.fixture(scope="module")
def lib():
    # the build script is loaded by path: importing the package loads libpi.so, which
    # fails when an older library lacks a symbol the binding binds
    import importlib.util
    spec = importlib.util.spec_from_file_location(
        "_pi_build_for_tests", os.path.join(ROOT, "activation_sparse_decode_bitmask_b200", "_build.py"))
    _build = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(_build)
    path = _build.build()
    return ctypes.CDLL(path), path


def test_header_declares_the_boundary():
    names = set(declared_functions())
    for n in ("pi_load_layer", "pi_reorder_hot_prefix", "pi_predict", "pi_compact_active",
              "pi_sparse_ffn", "pi_decode_stack", "pi_free_layer", "pi_status_str"):
        assert n in names


def test_every_declared_symbol_is_exported(lib):
    cdll, path = lib
    names = declared_functions()
    assert len(names) >= 18
    out = subprocess.run(["nm", "-D", "--defined-only", path], capture_output=True, text=True, check=True).stdout
    exported = set(re.findall(r"\bT\s+(pi_[a-z0-9_]+)", out))
    for n in names:
        assert n in exported, n
        assert hasattr(cdll, n)
    # and the binding wraps every one of them
    import activation_sparse_decode_bitmask_b200 as pi
    assert sorted(pi.EXPORTS) == sorted(names)


def test_host_validation_without_gpu(lib):
    import activation_sparse_decode_bitmask_b200 as pi
    L = pi.lib()
    assert L.pi_abi_version() == 10000
    assert L.pi_status_str(0) == b"ok"
    assert L.pi_status_str(5) == b"a device-side wait timed out"
    assert pi.kernel_launches() == 0       # nothing has launched in this CPU-only process
    # argument errors are returned before any CUDA call
    h = ctypes.c_void_p()
    assert L.pi_workspace_create(0, 1024, 64, 1, 1, ctypes.byref(h)) == 1
    assert L.pi_workspace_create(512, 1000, 64, 1, 1, ctypes.byref(h)) == 1     # d_ff % 32
    assert L.pi_workspace_create(512, 1024, 64, 33, 1, ctypes.byref(h)) == 1    # batch > 32
    desc = pi.make_desc(512, 2048, 64, "relu", "f16", "f32", "f16")             # mixed family
    w = pi.LayerWeights()
    assert L.pi_load_layer(ctypes.byref(desc), ctypes.byref(w), None, ctypes.byref(h)) == 2
    desc = pi.make_desc(500, 2048, 64, "relu", "f16", "f16", "f16")             # d % 64
    assert L.pi_load_layer(ctypes.byref(desc), ctypes.byref(w), None, ctypes.byref(h)) == 1
    desc = pi.make_desc(512, 2048, 1024, "relu", "f16", "f16", "f16")           # rank > d
    assert L.pi_load_layer(ctypes.byref(desc), ctypes.byref(w), None, ctypes.byref(h)) == 1
    desc = pi.make_desc(768, 2048, 64, "reglu", "q4_0", "f16", "f16")           # Q4_0 needs d % 256
    assert L.pi_load_layer(ctypes.byref(desc), ctypes.byref(w), None, ctypes.byref(h)) == 1
    desc = pi.make_desc(512, 2048, 64, "relu", "f16", "f16", "f16")             # null weights
    assert L.pi_load_layer(ctypes.byref(desc), ctypes.byref(w), None, ctypes.byref(h)) == 1
    assert L.pi_compact_active(None, 1, 64, None, None, None) == 1
    assert L.pi_decode_stack(None, 1, None, 1, None, None, None) == 1
    assert L.pi_layer_get_desc(None, None) == 1
