"""Pins of the oracle's per-step functions: RMSNorm, router, top-k, softmax, SwiGLU."""
import math

import numpy as np
import pytest

import oracle
from moe_inputs import bf16_bits_to_f32, f32_to_bf16_bits


# ------------------------------------------------------------------ RMSNorm

@pytest.mark.parametrize("c", [0.5, 1.0, -3.0, 1e-3, 0.0])
def test_rmsnorm_constant_row_closed_form(c):
    d, eps = 64, 1e-5
    x = f32_to_bf16_bits(np.full((1, d), c, dtype=np.float32))
    one = f32_to_bf16_bits(np.ones(d, dtype=np.float32))
    xn = oracle.rmsnorm(x, one, eps)
    cb = float(bf16_bits_to_f32(x)[0, 0])
    want = cb / math.sqrt(cb * cb + eps)
    assert np.allclose(xn, want, rtol=1e-15, atol=0)


def test_rmsnorm_scale_is_elementwise_and_unit_mean_square():
    rng = np.random.default_rng(2)
    d, eps = 256, 1e-5
    x = f32_to_bf16_bits(rng.standard_normal((3, d), dtype=np.float32) * 4)
    s = f32_to_bf16_bits(1 + 0.3 * rng.standard_normal(d, dtype=np.float32))
    one = f32_to_bf16_bits(np.ones(d, dtype=np.float32))
    xn1 = oracle.rmsnorm(x, one, eps)
    xns = oracle.rmsnorm(x, s, eps)
    assert np.allclose(xns, xn1 * bf16_bits_to_f32(s).astype(np.float64), rtol=1e-14)
    xf = bf16_bits_to_f32(x).astype(np.float64)
    ms = (xf ** 2).mean(axis=1)
    assert np.allclose((xn1 ** 2).mean(axis=1), ms / (ms + eps), rtol=1e-12)
    # no mean subtraction: a shifted row does not normalise like its centred copy
    assert not np.allclose(xn1, xn1 - xn1.mean(axis=1, keepdims=True))


def test_rmsnorm_scale_invariance():
    rng = np.random.default_rng(3)
    d = 128
    xf = rng.standard_normal((2, d)).astype(np.float32)
    x1 = f32_to_bf16_bits(xf)
    x2 = f32_to_bf16_bits(bf16_bits_to_f32(x1) * 8)        # exact power-of-two scaling
    one = f32_to_bf16_bits(np.ones(d, dtype=np.float32))
    a, b = oracle.rmsnorm(x1, one, 0.0), oracle.rmsnorm(x2, one, 0.0)
    assert np.allclose(a, b, rtol=1e-14)


# ------------------------------------------------------------------- router

def test_router_matches_matmul_and_onehot_rows():
    rng = np.random.default_rng(4)
    T, d, E = 5, 96, 7
    xn = rng.standard_normal((T, d))
    W = f32_to_bf16_bits(rng.standard_normal((E, d), dtype=np.float32) / np.sqrt(d))
    b = rng.standard_normal(E).astype(np.float32)
    got = oracle.router(xn, W, b)
    want = (xn @ bf16_bits_to_f32(W).astype(np.float64).T + b.astype(np.float64)).astype(np.float32)
    assert got.dtype == np.float32
    assert np.array_equal(got, want) or np.max(np.abs(got - want)) <= 2 * np.finfo(np.float32).eps * np.max(np.abs(want))
    # one-hot router rows pick a coordinate of xn
    W1 = np.zeros((E, d), dtype=np.float32)
    cols = rng.permutation(d)[:E]
    W1[np.arange(E), cols] = 1.0
    got1 = oracle.router(xn, f32_to_bf16_bits(W1), b)
    assert np.array_equal(got1, (xn[:, cols] + b.astype(np.float64)).astype(np.float32))


# --------------------------------------------------------- top-k, softmax

def _stable_topk(l, k):
    return sorted(range(len(l)), key=lambda e: (-float(l[e]), e))[:k]


@pytest.mark.parametrize("E,k", [(8, 4), (32, 4), (128, 4), (5, 1), (6, 6), (40, 8)])
def test_topk_against_full_sort(E, k):
    rng = np.random.default_rng(E * 10 + k)
    logits = rng.standard_normal((50, E)).astype(np.float32)
    logits[::7, : E // 2] = logits[::7, E // 2: 2 * (E // 2)]            # plant exact ties
    logits[3, :] = 0.25                                                  # all equal
    idx, _ = oracle.topk_softmax(logits, k)
    for t in range(logits.shape[0]):
        assert list(idx[t]) == _stable_topk(logits[t], k), t
    assert list(idx[3]) == list(range(k))


def test_topk_ties_go_to_lower_index():
    logits = np.array([[1.0, 3.0, 3.0, 0.0, 3.0, 2.0]], dtype=np.float32)
    idx, _ = oracle.topk_softmax(logits, 4)
    assert list(idx[0]) == [1, 2, 4, 5]


def test_softmax_over_chosen_logits():
    rng = np.random.default_rng(5)
    T, E, k = 40, 32, 4
    logits = (rng.standard_normal((T, E)) * 3).astype(np.float32)
    idx, w = oracle.topk_softmax(logits, k)
    assert np.allclose(w.sum(axis=1), 1.0, atol=1e-15)
    assert np.all(np.diff(w, axis=1) <= 0)          # weights follow the logit order
    # identical to the full softmax renormalised over the chosen experts
    L = logits.astype(np.float64)
    full = np.exp(L - L.max(axis=1, keepdims=True))
    full /= full.sum(axis=1, keepdims=True)
    sel = np.take_along_axis(full, idx.astype(np.int64), axis=1)
    assert np.allclose(w, sel / sel.sum(axis=1, keepdims=True), rtol=1e-13)
    _, w1 = oracle.topk_softmax(logits, 1)
    assert np.all(w1 == 1.0)


# ------------------------------------------------------------------- SwiGLU

def test_swiglu_special_cases():
    sw = oracle.swiglu
    for u in (-3.0, 0.0, 2.5):
        assert sw(0.0, u) == 0.0                        # g = 0
    for g in (-2.0, 0.5, 6.0):
        assert sw(g, -1.0) == 0.0                       # u + 1 = 0
    for u in (-8.0, 0.3, 9.0):
        assert sw(7.0, u) == sw(8.0, u) == sw(1e6, u)   # gate clamped above at 7
    for g in (-1.0, 3.0):
        assert sw(g, 7.0) == sw(g, 50.0)                      # linear clamped at +7
        assert sw(g, -7.0) == sw(g, -1e9)                     # and at -7
    # no lower clamp on the gate: large negative gates decay to 0 from below
    assert sw(-10.0, 0.0) < 0 and sw(-50.0, 0.0) < 0 and abs(sw(-50.0, 0.0)) < 1e-30
    assert sw(-10.0, 0.0) != sw(-7.0, 0.0)
    # at g = 7 the sigmoid is within 1e-5 of one: h ~= 7 (u + 1)
    assert 7.0 * (1 - 1e-5) < sw(7.0, 0.0) < 7.0


def test_swiglu_sigmoid_symmetry():
    # sigma(a) + sigma(-a) = 1  =>  h(g,u)/g + h(-g,u)/(-g) = u + 1 for |g| <= 7
    for g in (0.1, 0.7, 2.0, 5.5, 7.0):
        for u in (-0.5, 0.0, 3.0):
            s = oracle.swiglu(g, u) / g + oracle.swiglu(-g, u) / (-g)
            assert abs(s - (u + 1)) < 1e-14
    # alpha = 1.702: h(g, 0) / g = sigma(1.702 g); check at g = ln(3)/1.702, sigma = 3/4
    g = math.log(3.0) / 1.702
    assert abs(oracle.swiglu(g, 0.0) / g - 0.75) < 1e-14
