"""Host-side checks of the C-ABI library (no GPU needed): it loads, exports
every entry point include/fnl.h declares, and reports errors without a device."""
import ctypes
import os
import re
import subprocess

import pytest

from transformer_layer_residual_b200 import fnl

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_symbols():
    with open(os.path.join(ROOT, "include", "fnl.h")) as f:
        text = f.read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(fnl_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = declared_symbols()
    for n in ("fnl_create", "fnl_add_norm_qkv", "fnl_add_norm_swiglu", "fnl_add_bias_norm_gelu",
              "fnl_destroy"):
        assert n in names
    assert set(names) == set(fnl.EXPORTED)


def test_library_exports_every_declared_symbol():
    L = fnl.lib()
    for n in declared_symbols():
        assert hasattr(L, n), n
    out = subprocess.run(["nm", "-D", "--defined-only", fnl.lib_path()], capture_output=True, text=True).stdout
    exported = set(re.findall(r" T (fnl_\w+)", out))
    assert set(declared_symbols()) <= exported


def test_debug_build_exports_the_same_symbols():
    """libfnl_debug.so (output stores bounds-checked) is a drop-in for libfnl.so."""
    path = os.path.join(os.path.dirname(fnl.lib_path()), "libfnl_debug.so")
    if not os.path.exists(path):
        pytest.skip("debug build not built")
    out = subprocess.run(["nm", "-D", "--defined-only", path], capture_output=True, text=True).stdout
    assert set(declared_symbols()) <= set(re.findall(r" T (fnl_\w+)", out))


def test_library_is_sm100a_only_and_self_contained():
    out = subprocess.run(["ldd", fnl.lib_path()], capture_output=True, text=True).stdout
    assert "libcudart" not in out          # runtime linked statically
    assert "libtorch" not in out and "libc10" not in out


def test_status_strings():
    L = fnl.lib()
    for code, name in fnl.STATUS_NAMES.items():
        assert L.fnl_status_string(code).decode() == name
    assert L.fnl_status_string(99).decode() == "FNL_ERR_UNKNOWN"


def test_null_handle_paths():
    L = fnl.lib()
    assert L.fnl_destroy(None) == 0
    assert L.fnl_last_error(None).decode() == ""
    assert L.fnl_check(None, None) == 1
    assert L.fnl_create(None, 0, None) == 1
    # an entry point called with a NULL handle is rejected before touching the GPU
    args = [None] * 21
    args[7] = 0
    args[8] = ctypes.c_float(1e-5)
    for i in (11, 12, 13, 14, 15):
        args[i] = 1
    assert L.fnl_add_norm_qkv(*args) == 1


def test_create_without_a_usable_device_fails_cleanly():
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is visible")
    h = ctypes.c_void_p()
    st = fnl.lib().fnl_create(ctypes.byref(h), 0, None)
    assert st in (4, 5) and not h.value


def _header_enum_values():
    with open(os.path.join(ROOT, "include", "fnl.h")) as f:
        text = re.sub(r"/\*.*?\*/", "", f.read(), flags=re.S)
    return {k: int(v) for k, v in re.findall(r"\b(FNL_[A-Z_]+)\s*=\s*(\d+)", text)}


def test_binding_codes_match_the_header():
    """The binding's names for paths, norms, precisions and status codes are
    the header's enum values (a mismatch would silently pick another kernel)."""
    e = _header_enum_values()
    paths = {"auto": "FNL_PATH_AUTO", "tile": "FNL_PATH_TILE", "splitk": "FNL_PATH_SPLITK",
             "wide": "FNL_PATH_TILE_WIDE", "cluster": "FNL_PATH_SPLITK_CLUSTER", "pair": "FNL_PATH_TILE_PAIR",
             "pair_sk": "FNL_PATH_TILE_PAIR_SPLIT"}
    assert {k: e[v] for k, v in paths.items()} == fnl.PATHS
    assert {"layernorm": e["FNL_NORM_LAYERNORM"], "rmsnorm": e["FNL_NORM_RMSNORM"]} == fnl.NORMS
    precisions = {"default": "FNL_PRECISION_DEFAULT", "split": "FNL_PRECISION_SPLIT",
                  "single": "FNL_PRECISION_SINGLE"}
    assert {k: e[v] for k, v in precisions.items()} == fnl.PRECISIONS
    assert {e[n]: n for n in fnl.STATUS_NAMES.values()} == fnl.STATUS_NAMES
