"""The C-ABI library loads and exports every symbol include/moe_mx.h declares (CPU only).

No compute call is made here: only host-side argument validation, which runs
before any CUDA work, and the pure host helpers.
"""
import ctypes
import os
import re

import pytest

from block_scaled_moe_softmax_b200 import build as build_mod
from block_scaled_moe_softmax_b200 import moe_mx

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "moe_mx.h")


def _declared_symbols():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(moe_mx_[a-z_]+)\s*\(", text)))


@pytest.fixture(scope="module")
def lib():
    build_mod.build()
    return moe_mx.load_library()


def test_every_declared_symbol_is_exported(lib):
    syms = _declared_symbols()
    assert "moe_mx_forward" in syms and "moe_mx_create" in syms and "moe_mx_destroy" in syms
    for s in syms:
        assert hasattr(lib, s), f"{s} declared in moe_mx.h but not exported"
    assert sorted(moe_mx.SIGNATURES) == syms, "the Python binding must cover exactly the declared entry points"


def test_only_declared_symbols_are_exported(lib):
    # -fvisibility=hidden: nothing else leaks from the shared object
    out = os.popen(f"nm -D --defined-only {moe_mx.LIB_PATH}").read()
    exported = sorted(set(re.findall(r"\b(moe_mx_[a-z_]+)\b", out)))
    assert exported == _declared_symbols()


def test_library_is_built_for_sm100a_only(lib):
    # every translation unit and the link are compiled for sm_100a alone (no PTX for other
    # targets), so the GPU tests' launches only succeed on an sm_100 device
    flags = build_mod.FLAGS
    gencodes = [flags[i + 1] for i, f in enumerate(flags) if f == "-gencode"]
    assert gencodes == ["arch=compute_100a,code=sm_100a"]


def test_host_validation_without_gpu(lib):
    # argument errors are reported before any CUDA call
    assert lib.moe_mx_forward(None, None, None, 1, None, None, None, None, 1, 0, None, None) == moe_mx.MOE_MX_ERR_INVALID_ARG
    assert b"handle" in lib.moe_mx_last_error()
    assert lib.moe_mx_quantize(None, 4, 48, 0, None, None, None) == moe_mx.MOE_MX_ERR_INVALID_ARG
    assert lib.moe_mx_quantize(None, 4, 64, 7, None, None, None) == moe_mx.MOE_MX_ERR_INVALID_ARG
    h = ctypes.c_void_p()
    assert lib.moe_mx_create(ctypes.byref(h), 200, 128, 8, 16, 2, 0) == moe_mx.MOE_MX_ERR_UNSUPPORTED
    assert lib.moe_mx_create(ctypes.byref(h), 256, 100, 8, 16, 2, 0) == moe_mx.MOE_MX_ERR_UNSUPPORTED
    assert lib.moe_mx_create(ctypes.byref(h), 256, 128, 8, 16, 33, 0) == moe_mx.MOE_MX_ERR_INVALID_ARG
    assert lib.moe_mx_create(ctypes.byref(h), 256, 128, 2000, 16, 2, 0) == moe_mx.MOE_MX_ERR_UNSUPPORTED
    assert lib.moe_mx_create(None, 256, 128, 8, 16, 2, 0) == moe_mx.MOE_MX_ERR_INVALID_ARG
    ce = lib.moe_mx_create_ex
    assert ce(ctypes.byref(h), 256, 128, 1000, 30, 16, 2, 0) == moe_mx.MOE_MX_ERR_UNSUPPORTED  # E + S > 1024
    assert ce(ctypes.byref(h), 256, 128, 8, 4, 16, 30, 0) == moe_mx.MOE_MX_ERR_UNSUPPORTED     # top_k + S > 32
    assert ce(ctypes.byref(h), 256, 128, 8, -1, 16, 2, 0) == moe_mx.MOE_MX_ERR_UNSUPPORTED
    fr = lib.moe_mx_forward_routed
    assert fr(None, None, None, None, 1, 1, 0, None, None, None, None, 0, None, 0, None) == moe_mx.MOE_MX_ERR_INVALID_ARG
    assert fr(None, None, None, None, 1, 1, 0, None, None, None, None, 0, None, 5, None) == moe_mx.MOE_MX_ERR_INVALID_ARG
    assert b"out_dtype" in lib.moe_mx_last_error()
    assert lib.moe_mx_block_rows() == 128
    assert lib.moe_mx_destroy(None) == moe_mx.MOE_MX_OK
    assert lib.moe_mx_debug_watchdog(None, 10, None) == moe_mx.MOE_MX_ERR_INVALID_ARG


def test_binding_fails_loudly_when_library_missing(tmp_path):
    with pytest.raises(RuntimeError, match="no fallback"):
        moe_mx._lib_saved = moe_mx._lib
        try:
            moe_mx._lib = None
            moe_mx.load_library(str(tmp_path / "libmoe_mx.so"))
        finally:
            moe_mx._lib = moe_mx._lib_saved
