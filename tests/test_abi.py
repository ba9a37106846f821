"""The C ABI library without a GPU: it loads, exports exactly the entry points the
header declares, and validates shapes before touching a device."""
import ctypes
import os
import re
import subprocess

import pytest

import sparse_moe_rmsnorm_b200 as moe
from sparse_moe_rmsnorm_b200 import build as moe_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "moe_b200.h")


def declared_symbols():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"MOE_API\s+(?:const\s+)?\w+\s*\*?\s*(moe_\w+)\s*\(", text)))


@pytest.fixture(scope="module")
def lib():
    moe_build.build()
    return moe.lib()


def test_header_declares_the_boundary():
    syms = declared_symbols()
    for s in ["moe_init", "moe_forward", "moe_destroy", "moe_route", "moe_group", "moe_expert_up",
              "moe_expert_down", "moe_finalize", "moe_sync_status", "moe_strerror", "moe_forward_noalloc"]:
        assert s in syms


def test_library_exports_exactly_the_declared_symbols(lib):
    out = subprocess.run(["nm", "-D", "--defined-only", moe.library_path()], capture_output=True, text=True,
                         check=True).stdout
    exported = sorted(set(m for m in re.findall(r" T (moe_\w+)", out)))
    assert exported == declared_symbols()
    for s in declared_symbols():
        assert hasattr(lib, s)


def test_strings_and_shape_validation_without_gpu(lib):
    assert moe.moe_version().startswith("moe_b200")
    assert moe.moe_strerror(moe.MOE_ERR_TIMEOUT) == "device-side wait timed out"
    bad = [moe.MoEShape(0, 128, 128, 8, 4, 1e-5), moe.MoEShape(16, 100, 128, 8, 4, 1e-5),
           moe.MoEShape(16, 128, 96, 8, 4, 1e-5), moe.MoEShape(16, 128, 128, 0, 1, 1e-5),
           moe.MoEShape(16, 128, 128, 4, 5, 1e-5), moe.MoEShape(16, 128, 128, 300, 4, 1e-5),
           moe.MoEShape(16, 128, 128, 8, 9, 1e-5), moe.MoEShape(16, 128, 128, 8, 4, -1.0)]
    for s in bad:
        h = ctypes.c_void_p()
        assert lib.moe_init(ctypes.byref(s), ctypes.byref(h)) == moe.MOE_ERR_ARG
    assert lib.moe_init(None, None) == moe.MOE_ERR_ARG
    # no-alloc entry: argument checks come before any device work
    assert lib.moe_forward_noalloc(65, 128, 128, 8, 4, 1e-5, *([None] * 12)) == moe.MOE_ERR_ARG
    assert lib.moe_forward_noalloc(16, 100, 128, 8, 4, 1e-5, *([None] * 12)) == moe.MOE_ERR_ARG
    assert lib.moe_forward_noalloc(0, 128, 128, 8, 4, 1e-5, *([None] * 12)) == moe.MOE_OK
    # null context
    assert lib.moe_sync_status(None, None) == moe.MOE_ERR_ARG
    assert lib.moe_forward(None, 1, *([None] * 10), 4, *([None] * 4)) == moe.MOE_ERR_ARG


def test_stage_calls_reject_null_context(lib):
    assert lib.moe_group(None, 4, 4, None) == moe.MOE_ERR_ARG
    assert lib.moe_expert_up(None, 4, 4, None, None, None, None) == moe.MOE_ERR_ARG
    assert lib.moe_copy_workspace(None, 0, None, 0, None) == moe.MOE_ERR_ARG
