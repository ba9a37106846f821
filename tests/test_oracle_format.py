"""Pins of the oracle's MXFP4 decode and of the format's size arithmetic.

The decode is checked against the OCP MX closed form of E2M1 (sign bit, two
exponent bits with bias 1, one mantissa bit, subnormal when the exponent bits
are zero) times the E8M0 scale 2^(s-127) -- written here from the spec, not
from the oracle's table -- on all 16 codes x 256 scale bytes.  The storage
arithmetic is checked against the checkpoint sizes the gpt-oss write-ups print.
"""
import json
import math
import os

import numpy as np
import pytest

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "pages_figures.json")


def ocp_e2m1(code: int) -> float:
    sign = -1.0 if (code >> 3) & 1 else 1.0
    exp = (code >> 1) & 3
    man = code & 1
    if exp == 0:
        mag = man * 0.5                       # subnormal: 0.m x 2^(1-bias), bias 1
    else:
        mag = 2.0 ** (exp - 1) * (1.0 + man / 2.0)
    return sign * mag


def test_decode_table_exhaustive():
    for s in range(256):
        for c in range(16):
            got = oracle.mxfp4_value(c, s)
            if s == 255:
                assert math.isnan(got), (c, s)
                continue
            want = ocp_e2m1(c) * math.ldexp(1.0, s - 127)
            assert got == want, (c, s, got, want)
            assert math.copysign(1.0, got) == math.copysign(1.0, want), (c, s)


def test_decode_magnitudes_and_negative_zero():
    mags = sorted({abs(oracle.mxfp4_value(c, 127)) for c in range(16)})
    assert mags == [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]
    negz = oracle.mxfp4_value(8, 127)
    assert negz == 0.0 and math.copysign(1.0, negz) == -1.0
    for c in range(8):
        assert oracle.mxfp4_value(c | 8, 127) == -oracle.mxfp4_value(c, 127)


def test_decode_bf16_exact_range():
    """Every decoded value is exactly a bf16 number for scale bytes 1..252."""
    for s in range(1, 253):
        for c in range(16):
            v = np.float64(oracle.mxfp4_value(c, s))
            f = np.float32(v)
            assert np.float64(f) == v
            bits = f.view(np.uint32)
            assert bits & 0xFFFF == 0, (c, s)


def test_decode_matrix_nibble_order_and_block_axis():
    rng = np.random.default_rng(1)
    R, K = 5, 96
    codes = rng.integers(0, 256, size=(R, K // 2), dtype=np.uint8)
    scales = rng.integers(100, 150, size=(R, K // 32), dtype=np.uint8)
    want = np.empty((R, K))
    for r in range(R):
        for m in range(K // 2):
            lo, hi = int(codes[r, m]) & 15, int(codes[r, m]) >> 4
            want[r, 2 * m] = ocp_e2m1(lo) * 2.0 ** (int(scales[r, (2 * m) // 32]) - 127)
            want[r, 2 * m + 1] = ocp_e2m1(hi) * 2.0 ** (int(scales[r, (2 * m + 1) // 32]) - 127)
    got = oracle.decode_matrix(codes, scales)
    assert np.array_equal(got, want)


def _golden():
    with open(GOLDEN) as f:
        return {k: v["value"] for k, v in json.load(f).items() if not k.startswith("_")}


def test_bits_per_weight_matches_pages():
    g = _golden()
    bits = oracle.mxfp4_bytes(1, 32) * 8 / 32
    assert bits == g["bits_per_weight"]


@pytest.mark.parametrize("model", ["20b", "120b"])
def test_checkpoint_size_matches_pages(model):
    g = _golden()
    d, F = g["d_model"], g["d_ff"]
    E, L = g["experts"][model], g["layers"][model]
    per_expert = oracle.mxfp4_bytes(2 * F, d) + oracle.mxfp4_bytes(d, F)
    assert per_expert == 13_219_200
    moe_params = L * E * 3 * d * F
    share = moe_params / g["params_total"][model]
    assert share > g["moe_share_min"]
    other_params = g["params_total"][model] - moe_params       # stored at 16 bits
    est_gib = (L * E * per_expert + 2 * other_params) / 2 ** 30
    assert abs(est_gib - g["checkpoint_gib"][model]) / g["checkpoint_gib"][model] < g["checkpoint_rel_tol"]
    # the routed experts of one token are a part of the active parameters
    assert L * g["top_k"] * 3 * d * F < g["params_active"][model]
