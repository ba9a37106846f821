"""The allocation-free entry point against the regular one.

Some callers cannot allocate device memory (a CUDA graph being captured in a
mode that forbids allocation, a framework whose allocator owns all device
memory, a plugin host that forbids it).  moe_forward_noalloc serves them from a
fixed scratch array inside the library.  This file is collected last so that a
run stopping at its first failure has run every other test already; it passes
alone in a fresh process and after the other tests.
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

import sparse_moe_rmsnorm_b200 as moe
from moe_inputs import CONFIGS, custom_layer, make_config_inputs
from _parity import MAX_REL, MEAN_REL

pytestmark = pytest.mark.gpu


def _bf16(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.uint16).view(np.int16)).view(torch.bfloat16).cuda()


def _close(a, b):
    a = a.float().cpu().numpy().astype(np.float64)
    b = b.float().cpu().numpy().astype(np.float64)
    diff = np.abs(a - b)
    return diff.max() <= MAX_REL * np.abs(b).max() and diff.sum() <= MEAN_REL * np.abs(b).sum()


@pytest.mark.parametrize("name", ["tiny", "decode20b"])
def test_noalloc_matches_regular_entry_point_twice(name):
    cfg = CONFIGS[name]
    inp = make_config_inputs(cfg)
    w = moe.MoEWeights.from_numpy(inp)
    x = _bf16(inp["x"])
    ctx = moe.MoE(cfg.T, cfg.d, cfg.F, cfg.E, cfg.k, cfg.eps)
    y_ref = ctx.forward(x, w)
    torch.cuda.synchronize()
    assert ctx.sync_status() == moe.MOE_OK
    ctx.close()
    for _ in range(2):
        y = torch.full_like(x, float("nan"))
        moe.moe_forward_noalloc(cfg.T, cfg.d, cfg.F, cfg.E, cfg.k, cfg.eps, x, w.router_w, w.router_b,
                                w.w13_codes, w.w13_scales, w.b13, w.w2_codes, w.w2_scales, w.b2, w.norm_scale, y)
        torch.cuda.synchronize()
        assert _close(y, y_ref)


def test_noalloc_rejects_batches_beyond_its_scratch():
    inp = custom_layer(T=65, d=128, F=128, E=8, k=4, seed=1)
    w = moe.MoEWeights.from_numpy(inp)
    x = _bf16(inp["x"])
    y = torch.empty_like(x)
    with pytest.raises(moe.MoEError) as e:
        moe.moe_forward_noalloc(65, 128, 128, 8, 4, 1e-5, x, w.router_w, w.router_b, w.w13_codes, w.w13_scales,
                                w.b13, w.w2_codes, w.w2_scales, w.b2, w.norm_scale, y)
    assert e.value.code == moe.MOE_ERR_ARG
