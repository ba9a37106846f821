"""Pins of the oracle's whole block.

* E = 1, top-1: the block reduces to a dense FFN with routing weight exactly 1,
  evaluated here with numpy matrix products in float64.
* Dense brute force: every expert evaluated for every token with numpy
  (einsum over the fully decoded weights), then combined through the one-hot
  routing mask times the softmax weights.  The sparse oracle must agree to
  ~1e-10 relative.
* Planted mistakes: copies of the oracle source with one plausible mistake each
  (a dropped bias, swapped nibbles, swapped gate/linear rows, ...) are built and
  must fail at least one of the pins.

The numpy side decodes MXFP4 with the OCP closed form from test_oracle_format
and shares nothing with the C oracle.
"""
import os
import shutil
import tempfile

import numpy as np
import pytest

import oracle
from moe_inputs import bf16_bits_to_f32, custom_layer
from test_oracle_format import ocp_e2m1

_LUT = np.array([ocp_e2m1(c) for c in range(16)])


def np_decode(codes, scales):
    codes = codes.astype(np.int64)
    vals = np.empty(codes.shape[:-1] + (codes.shape[-1] * 2,))
    vals[..., 0::2] = _LUT[codes & 15]
    vals[..., 1::2] = _LUT[codes >> 4]
    sc = np.where(scales == 255, np.nan, np.ldexp(1.0, scales.astype(np.int64) - 127))
    return vals * np.repeat(sc, 32, axis=-1)


def np_swiglu(gate, lin):
    g = np.minimum(gate, 7.0)
    u = np.clip(lin, -7.0, 7.0)
    return g / (1.0 + np.exp(-1.702 * g)) * (u + 1.0)


def dense_block(inp, k, eps):
    x = bf16_bits_to_f32(inp["x"]).astype(np.float64)
    T, d = x.shape
    E = inp["router_w"].shape[0]
    F = inp["w13_codes"].shape[1] // 2
    s = bf16_bits_to_f32(inp["norm_scale"]).astype(np.float64)
    xn = x / np.sqrt((x * x).mean(axis=1, keepdims=True) + eps) * s
    logits = (xn @ bf16_bits_to_f32(inp["router_w"]).astype(np.float64).T
              + inp["router_b"].astype(np.float64)).astype(np.float32)
    W13 = np_decode(inp["w13_codes"], inp["w13_scales"])             # [E, 2F, d]
    W2 = np_decode(inp["w2_codes"], inp["w2_scales"])                # [E, d, F]
    b13 = bf16_bits_to_f32(inp["b13"]).astype(np.float64)
    b2 = bf16_bits_to_f32(inp["b2"]).astype(np.float64)
    Z = np.einsum("td,efd->tef", xn, W13) + b13[None]
    H = np_swiglu(Z[..., :F], Z[..., F:])
    O = np.einsum("tef,edf->ted", H, W2) + b2[None]
    M = np.zeros((T, E))
    for t in range(T):
        order = sorted(range(E), key=lambda e: (-float(logits[t, e]), e))[:k]
        l = logits[t, order].astype(np.float64)
        w = np.exp(l - l.max())
        M[t, order] = w / w.sum()
    y = x + np.einsum("te,ted->td", M, O)
    return y, M, logits


SHAPES = [(dict(T=16, d=128, F=128, E=8), 4), (dict(T=7, d=64, F=96, E=5), 2),
          (dict(T=9, d=96, F=64, E=6), 6), (dict(T=5, d=64, F=64, E=3), 1)]


@pytest.mark.parametrize("shape,k", SHAPES)
def test_dense_brute_force(shape, k):
    inp = custom_layer(**shape, k=k, seed=11, scale_lo=118, scale_hi=124)
    got = oracle.moe_forward(inp, k, 1e-5)
    y, M, logits = dense_block(inp, k, 1e-5)
    assert np.array_equal(got["logits"], logits) or np.max(np.abs(got["logits"] - logits)) < 1e-6
    for t in range(shape["T"]):
        assert set(got["idx"][t]) == set(np.nonzero(M[t])[0])
        assert np.allclose(got["w"][t], M[t, got["idx"][t]], rtol=1e-12)
    assert np.max(np.abs(got["y"] - y)) <= 1e-10 * np.max(np.abs(y))


def test_single_expert_top1_is_dense_ffn():
    inp = custom_layer(T=6, d=64, F=64, E=1, k=1, seed=3)
    got = oracle.moe_forward(inp, 1, 1e-5)
    assert np.all(got["idx"] == 0) and np.all(got["w"] == 1.0)
    x = bf16_bits_to_f32(inp["x"]).astype(np.float64)
    s = bf16_bits_to_f32(inp["norm_scale"]).astype(np.float64)
    xn = x / np.sqrt((x * x).mean(axis=1, keepdims=True) + 1e-5) * s
    W13 = np_decode(inp["w13_codes"][0], inp["w13_scales"][0])
    W2 = np_decode(inp["w2_codes"][0], inp["w2_scales"][0])
    z = xn @ W13.T + bf16_bits_to_f32(inp["b13"][0]).astype(np.float64)
    h = np_swiglu(z[:, :64], z[:, 64:])
    y = x + h @ W2.T + bf16_bits_to_f32(inp["b2"][0]).astype(np.float64)
    assert np.max(np.abs(got["y"] - y)) <= 1e-12 * np.max(np.abs(y))


def test_expert_function_matches_block():
    inp = custom_layer(T=3, d=64, F=64, E=4, k=2, seed=5)
    got = oracle.moe_forward(inp, 2, 1e-5)
    xn = oracle.rmsnorm(inp["x"], inp["norm_scale"], 1e-5)
    x = bf16_bits_to_f32(inp["x"]).astype(np.float64)
    for t in range(3):
        y = x[t].copy()
        for i in range(2):
            _, o = oracle.expert(inp, int(got["idx"][t, i]), xn[t])
            y += got["w"][t, i] * o
        assert np.allclose(y, got["y"][t], rtol=0, atol=1e-12 * np.abs(y).max())


def test_empty_batch_and_bad_shape():
    inp = custom_layer(T=0, d=64, F=64, E=4, k=2, seed=1)
    got = oracle.moe_forward(inp, 2, 1e-5)
    assert got["y"].shape == (0, 64)
    with pytest.raises(ValueError):
        oracle.moe_forward(inp, 5, 1e-5)      # k > E


# --------------------------------------------------------- planted mistakes

MUTATIONS = {
    "dropped_b2": ("o[r] = mx_row_dot(w2_codes, w2_scales, F, r, h) + bf16_value(b2[r]);",
                   "o[r] = mx_row_dot(w2_codes, w2_scales, F, r, h);"),
    "nibbles_swapped": ("int code = (j & 1) ? (byte >> 4) : (byte & 15);",
                        "int code = (j & 1) ? (byte & 15) : (byte >> 4);"),
    "gate_linear_swapped": ("double gate = mx_row_dot(w13_codes, w13_scales, d, j, xn_t)",
                            "double gate = mx_row_dot(w13_codes, w13_scales, d, F + j, xn_t)"),
    "ties_to_higher_index": ("if (best < 0 || logit[e] > logit[best]) best = e;",
                             "if (best < 0 || logit[e] >= logit[best]) best = e;"),
    "sigmoid_sign": ("return g * (1.0 / (1.0 + exp(-1.702 * g))) * (u + 1.0);",
                     "return g * (1.0 / (1.0 + exp(1.702 * g))) * (u + 1.0);"),
    "no_plus_one": ("return g * (1.0 / (1.0 + exp(-1.702 * g))) * (u + 1.0);",
                    "return g * (1.0 / (1.0 + exp(-1.702 * g))) * u;"),
    "gate_clamped_below": ("double g = fmin(gate, 7.0);", "double g = fmax(fmin(gate, 7.0), -7.0);"),
    "no_residual": ("for (int j = 0; j < d; ++j) yt[j] = bf16_value(x[(size_t)t * d + j]);",
                    "for (int j = 0; j < d; ++j) yt[j] = 0.0;"),
    "scale_block_index": ("scales[(size_t)r * (size_t)(K / 32) + (size_t)(j / 32)]",
                          "scales[(size_t)r * (size_t)(K / 32) + (size_t)((j / 16) % (K / 32))]"),
    "no_eps": ("double inv_rms = 1.0 / sqrt(ss / d + eps);", "double inv_rms = 1.0 / sqrt(ss / d);"),
    "router_on_raw_x": ("router_token(d, E, xn, router_w, router_b, logit);",
                        "for (int j = 0; j < d; ++j) xn[j] = bf16_value(x[(size_t)t * d + j]);\n"
                        "        router_token(d, E, xn, router_w, router_b, logit);\n"
                        "        oracle_rmsnorm(1, d, eps, x + (size_t)t * d, norm_scale, xn);"),
    "softmax_over_all": ("for (int i = 0; i < k; ++i) w[i] /= sum;",
                         "for (int e = 0; e < E; ++e) if (1) { int c = 0; for (int i = 0; i < k; ++i) c |= idx[i] == e;"
                         " if (!c) sum += exp((double)logit[e] - lmax); }\n    for (int i = 0; i < k; ++i) w[i] /= sum;"),
    "alpha_wrong": ("exp(-1.702 * g)", "exp(-1.5 * g)"),
}


def _all_pins_pass(lib) -> bool:
    """The pins above, run against one build of the oracle; False on the first miss."""
    try:
        # decode table
        for s in (100, 120, 127, 140):
            for c in range(16):
                if oracle.mxfp4_value(c, s, lib=lib) != ocp_e2m1(c) * 2.0 ** (s - 127):
                    return False
        # SwiGLU special cases and symmetry
        if oracle.swiglu(7.0, 0.0, lib=lib) != oracle.swiglu(9.0, 0.0, lib=lib):
            return False
        if oracle.swiglu(-10.0, 0.0, lib=lib) == oracle.swiglu(-7.0, 0.0, lib=lib):
            return False
        g = np.log(3.0) / 1.702
        if abs(oracle.swiglu(g, 0.0, lib=lib) / g - 0.75) > 1e-14 or oracle.swiglu(1.0, -1.0, lib=lib) != 0.0:
            return False
        # top-k ties
        idx, _ = oracle.topk_softmax(np.array([[1.0, 3.0, 3.0, 0.0, 3.0, 2.0]], np.float32), 4, lib=lib)
        if list(idx[0]) != [1, 2, 4, 5]:
            return False
        # dense brute force
        for shape, k in ((dict(T=8, d=64, F=64, E=6), 3), (dict(T=6, d=64, F=96, E=4), 2)):
            inp = custom_layer(**shape, k=k, seed=7, scale_lo=118, scale_hi=124)
            got = oracle.moe_forward(inp, k, 1e-5, lib=lib)
            y, _, _ = dense_block(inp, k, 1e-5)
            if not np.max(np.abs(got["y"] - y)) <= 1e-10 * np.max(np.abs(y)):
                return False
    except Exception:
        return False
    return True


def test_committed_oracle_passes_mutation_battery():
    assert _all_pins_pass(oracle._load())


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_planted_mistake_is_caught(name):
    before, after = MUTATIONS[name]
    src = open(os.path.join(os.path.dirname(oracle.__file__), "moe_oracle.c")).read()
    assert src.count(before) >= 1, name
    tmp = tempfile.mkdtemp(prefix="oracle_mut_")
    try:
        path = os.path.join(tmp, "m.c")
        with open(path, "w") as f:
            f.write(src.replace(before, after))
        lib = oracle.load_variant(oracle.compile_source(path, os.path.join(tmp, "libm_%s.so" % name)))
        assert not _all_pins_pass(lib), "planted mistake %r passed every pin" % name
    finally:
        shutil.rmtree(tmp, ignore_errors=True)
