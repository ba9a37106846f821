"""bench.py's roofline arithmetic on the CPU, against figures fixed independently of it.

The per-expert bytes and per-pair FLOPs follow from the MXFP4 format and the block's shapes:
an expert of the 2880-wide layer holds 3·2880·2880 weights (gate, linear and down rows) at
4 bits plus one E8M0 byte per 32, and bf16 biases for its 2·2880 + 2880 outputs; a routed
(token, expert) pair costs two multiply-adds per weight.  These are written out here from the
shapes, not from bench.py's own expressions.
"""
import os
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402

D = F = 2880
WEIGHTS_PER_EXPERT = 3 * D * F                       # 24,883,200
CODE_AND_SCALE_BYTES = WEIGHTS_PER_EXPERT // 2 + WEIGHTS_PER_EXPERT // 32
BIAS_BYTES = 2 * (2 * F + D)
FLOPS_PER_PAIR = 2 * WEIGHTS_PER_EXPERT


def test_scope_figures_written_out():
    # the totals of the hot-path scope table, from the format alone
    assert WEIGHTS_PER_EXPERT == 24_883_200
    assert CODE_AND_SCALE_BYTES == 13_219_200
    assert CODE_AND_SCALE_BYTES + BIAS_BYTES == 13_236_480
    assert FLOPS_PER_PAIR == 49_766_400


@pytest.mark.parametrize("name", ["decode20b", "decode120b", "prefill20b"])
def test_algorithmic_counts_from_the_routing(name):
    cfg = bench.CONFIGS[name]
    pairs = cfg.T * cfg.k
    # a routing that leaves the last quarter of the experts untouched
    counts = np.zeros(cfg.E, np.int64)
    live = cfg.E - cfg.E // 4
    counts[:live] = pairs // live
    counts[0] += pairs - counts.sum()
    c = bench.algorithmic_counts(cfg, counts)
    assert c["touched"] == live
    assert c["w13_expert"] + c["w2_expert"] == CODE_AND_SCALE_BYTES + BIAS_BYTES
    assert c["flops_up"] + c["flops_down"] == pairs * FLOPS_PER_PAIR
    assert c["flops_up"] == 2 * c["flops_down"]                     # 2F gate/linear rows against d down rows
    # layer: touched experts, the router (bf16 rows, fp32 bias), the RMSNorm scale, x in and y out
    router = cfg.E * cfg.d * 2 + cfg.E * 4
    assert c["layer_bytes"] == live * (CODE_AND_SCALE_BYTES + BIAS_BYTES) + router + cfg.d * 2 + 2 * cfg.T * cfg.d * 2
    assert c["layer_flops"] == 2 * cfg.T * cfg.d * cfg.E + pairs * FLOPS_PER_PAIR
    # the one-launch FFN's bytes: both GEMMs' weights, xn in, h out and back in, weighted fp32 rows out
    assert c["bytes_ffn"] == (live * (CODE_AND_SCALE_BYTES + BIAS_BYTES) + cfg.T * cfg.d * 2
                              + 2 * pairs * cfg.F * 2 + pairs * cfg.d * 4)


def test_untouched_experts_cost_nothing():
    cfg = bench.CONFIGS["decode20b"]
    counts = np.zeros(cfg.E, np.int64)
    counts[3] = cfg.T * cfg.k
    c = bench.algorithmic_counts(cfg, counts)
    assert c["touched"] == 1
    assert c["bytes_up"] - c["w13_expert"] == cfg.T * cfg.d * 2 + cfg.T * cfg.k * cfg.F * 2


@pytest.mark.parametrize("name,launches", [
    ("tiny", 3),          # route + group, both GEMMs, combine
    ("decode20b", 3),
    ("decode120b", 3),
    ("stack20b", 7),      # route, group, encoder (8192 pairs), pass plan, gate/up, down, combine
    ("prefill20b", 7),
])
def test_launches_per_layer_of_the_workloads(name, launches):
    cfg = bench.CONFIGS[name]
    assert bench.kernels_per_layer(cfg.T, cfg.k, cfg.d, cfg.F) == launches


def test_launches_per_layer_at_the_size_boundaries():
    assert bench.kernels_per_layer(64, 4, 2880, 2880) == 3       # largest decode-sized batch
    assert bench.kernels_per_layer(64, 4, 2880, 1440) == 4       # d != F: the two GEMMs apart
    assert bench.kernels_per_layer(64, 4, 4096, 4096) == 5       # d > 3072: route and group apart
    assert bench.kernels_per_layer(65, 4, 2880, 2880) == 6       # the pass plan joins
    assert bench.kernels_per_layer(512, 4, 2880, 2880) == 6      # 2048 pairs: encoder fused in the grouping
    assert bench.kernels_per_layer(513, 4, 2880, 2880) == 7
