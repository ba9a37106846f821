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
              "moe_expert_down", "moe_expert_ffn", "moe_finalize", "moe_sync_status", "moe_strerror",
              "moe_forward_noalloc"]:
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
    assert lib.moe_expert_up(None, 4, 4, None, None, None, None, None) == moe.MOE_ERR_ARG
    assert lib.moe_expert_ffn(None, 4, 4, *([None] * 7)) == moe.MOE_ERR_ARG
    assert lib.moe_copy_workspace(None, 0, None, 0, None) == moe.MOE_ERR_ARG


# (T, d, F, E, k) of the benchmark workloads; decode-sized batches use stacked
# 16-row token blocks with per-item scale factors, the others 192-row blocks
PLAN_CASES = {
    "tiny": (16, 128, 128, 8, 4, "decode"),
    "decode20b": (32, 2880, 2880, 32, 4, "decode"),
    "decode120b": (64, 2880, 2880, 128, 4, "decode"),
    "prefill20b": (8192, 2880, 2880, 32, 4, "large"),
    "stack20b": (2048, 2880, 2880, 32, 4, "large"),
    "single token": (1, 2880, 2880, 32, 4, "decode"),
}


@pytest.mark.parametrize("name", sorted(PLAN_CASES))
@pytest.mark.parametrize("mode", [0, 1])
def test_gemm_launch_plan_fits_the_sm(lib, name, mode):
    """The host planner's choices, without a GPU: within 227 KB of shared memory and 512 TMEM columns,
    a persistent grid of at most one CTA per SM, the K stages and weight-row blocks of the shape."""
    T, d, F, E, k, kind = PLAN_CASES[name]
    pl = moe.moe_debug_plan(mode, T, k, d, F, E, T * k, 148)
    K = d if mode == 0 else F
    assert pl["smem"] <= 227 * 1024 and pl["tmem_cols"] <= 512
    assert 2 <= pl["n_stages"] <= 12 and 1 <= pl["grid"] <= 148
    assert pl["k_stages"] == -(-K // 128) and pl["k_full_stages"] == K // 128
    assert pl["row_blocks"] == (F // 64 if mode == 0 else -(-d // 128))
    if kind == "decode":
        assert (pl["nb_rows"], pl["stacked"], pl["sf_item"]) == (16, 1, 1)
    else:
        assert (pl["nb_rows"], pl["stacked"], pl["sf_item"]) == (192, 0, 0)
        assert pl["n_stages"] == 3            # 16 KB of codes + 48 KB of two-term tokens per stage


def test_gemm_launch_plan_rejects_bad_arguments(lib):
    out = (ctypes.c_int * 10)()
    assert lib.moe_debug_plan(2, 32, 4, 2880, 2880, 32, 128, 148, out) == moe.MOE_ERR_ARG     # mode
    assert lib.moe_debug_plan(0, 32, 4, 2880, 2880, 32, 127, 148, out) == moe.MOE_ERR_ARG     # P_max < T k
    assert lib.moe_debug_plan(0, 32, 4, 100, 2880, 32, 128, 148, out) == moe.MOE_ERR_ARG      # d
    assert lib.moe_debug_plan(0, 32, 9, 2880, 2880, 32, 288, 148, out) == moe.MOE_ERR_ARG     # top_k
    assert lib.moe_debug_plan(0, 32, 4, 2880, 2880, 32, 128, 148, None) == moe.MOE_ERR_ARG
