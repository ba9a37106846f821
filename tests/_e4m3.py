"""The E4M3 terms of activations the block-scaled GEMMs read, in plain numpy.

This is the definition the device encoders (the permute kernel for the normalised tokens, the
gate/up epilogue for h) implement, written out for tests: per block of 32 consecutive elements
of a row, with v the fp32 values,
  s   = x - 8 + [m > 1.75], where max|v| = m * 2^x, 1 <= m < 2, clamped to [-126, 126]
        (the E8M0 exponent that brings the block maximum to at most 448 = 1.75 * 2^8);
  hi  = e4m3(v * 2^-s),   lo = e4m3((v - hi * 2^s) * 2^-s_lo),   s_lo = max(s - 4, -126),
  lo2 = e4m3((v - hi * 2^s - lo * 2^s_lo) * 2^-s),
with e4m3() the round-to-nearest-even conversion to OCP E4M3 (bias 7, 3 mantissa bits,
subnormals below 2^-6, largest finite 448), saturating to +-448.  Two terms represent v as
hi * 2^s + lo * 2^s_lo, three add lo2 * 2^s (lo2 shares hi's scale); the scale bytes are
s + 127 and s_lo + 127.
"""
from __future__ import annotations

import numpy as np


def e4m3_decode(b: np.ndarray) -> np.ndarray:
    """E4M3 bytes to float64 (0x7F / 0xFF, the NaN codes, decode to NaN)."""
    b = np.asarray(b, dtype=np.uint8).astype(np.int64)
    sign = np.where(b & 0x80, -1.0, 1.0)
    e = (b >> 3) & 0xF
    m = b & 7
    v = np.where(e == 0, m / 8.0 * 2.0 ** -6, (1 + m / 8.0) * np.exp2(e - 7.0))
    v = np.where((b & 0x7F) == 0x7F, np.nan, v)
    return sign * v


def e4m3_encode(x: np.ndarray) -> np.ndarray:
    """Round-to-nearest-even to E4M3 bytes, saturating at +-448 (x finite, float64 exact)."""
    x = np.asarray(x, dtype=np.float64)
    a = np.abs(x)
    # the quantum of the binade holding a: 2^(e-3) for normals (e >= -6), 2^-9 below
    e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    e = np.maximum(e, -6.0)
    q = np.exp2(e - 3.0)
    r = a / q
    n = np.floor(r)
    frac = r - n
    n = n + ((frac > 0.5) | ((frac == 0.5) & (np.mod(n, 2) == 1)))
    mag = np.minimum(n * q, 448.0)
    # magnitude -> code by search over the 127 non-negative finite codes
    table = e4m3_decode(np.arange(0x7F, dtype=np.uint8))
    code = np.searchsorted(table, mag).astype(np.uint8)
    assert np.all(table[code] == mag)
    return np.where((x < 0) & (mag > 0), code | 0x80, code).astype(np.uint8)


def block_exponent(amax: np.ndarray) -> np.ndarray:
    a = np.asarray(amax, dtype=np.float32)
    bits = a.view(np.uint32).astype(np.int64)
    x = ((bits >> 23) & 0xFF) - 127
    s = x - 8 + ((bits & 0x7FFFFF) > 0x600000)
    return np.clip(s, -126, 126)


def encode_two_term(v: np.ndarray):
    """v: float32 [rows, K] (K a multiple of 32) -> (hi u8, lo u8, s_hi u8, s_lo u8 [rows, K/32])."""
    v = np.asarray(v, dtype=np.float32)
    rows, K = v.shape
    blk = v.reshape(rows, K // 32, 32).astype(np.float64)
    s = block_exponent(np.abs(v.reshape(rows, K // 32, 32)).max(axis=2))
    s_lo = np.maximum(s - 4, -126)
    hi = e4m3_encode(blk * np.exp2(-s)[..., None])
    res = blk - e4m3_decode(hi) * np.exp2(s)[..., None]
    lo = e4m3_encode(res * np.exp2(-s_lo)[..., None])
    return (hi.reshape(rows, K), lo.reshape(rows, K), (s + 127).astype(np.uint8), (s_lo + 127).astype(np.uint8))


def encode_three_term(v: np.ndarray):
    """v: float32 [rows, K] -> (hi u8, lo u8, lo2 u8, s_hi u8, s_lo u8 [rows, K/32])."""
    v = np.asarray(v, dtype=np.float32)
    rows, K = v.shape
    hi, lo, s_hi, s_lo = encode_two_term(v)
    blk = v.reshape(rows, K // 32, 32).astype(np.float64)
    s = s_hi.astype(np.float64) - 127
    sl = s_lo.astype(np.float64) - 127
    res = (blk - e4m3_decode(hi.reshape(rows, K // 32, 32)) * np.exp2(s)[..., None]
           - e4m3_decode(lo.reshape(rows, K // 32, 32)) * np.exp2(sl)[..., None])
    lo2 = e4m3_encode(res * np.exp2(-s)[..., None])
    return hi, lo, lo2.reshape(rows, K), s_hi, s_lo


def decode_terms(planes, s_hi, s_lo) -> np.ndarray:
    """Sum of the first len(planes) terms (hi, lo[, lo2]) -> float64 [rows, K]."""
    rows, K = planes[0].shape
    scale = (s_hi, s_lo, s_hi)
    out = np.zeros((rows, K // 32, 32))
    for q, sc in zip(planes, scale):
        out += e4m3_decode(q).reshape(rows, K // 32, 32) * np.exp2(sc.astype(np.float64) - 127)[..., None]
    return out.reshape(rows, K)


def decode_two_term(hi, lo, s_hi, s_lo) -> np.ndarray:
    rows, K = hi.shape
    a = e4m3_decode(hi).reshape(rows, K // 32, 32) * np.exp2(s_hi.astype(np.float64) - 127)[..., None]
    b = e4m3_decode(lo).reshape(rows, K // 32, 32) * np.exp2(s_lo.astype(np.float64) - 127)[..., None]
    return (a + b).reshape(rows, K)


def scale_bytes_from_words(words: np.ndarray, plane: int, rows, n_blocks: int) -> np.ndarray:
    """words: int32 [G, 2, P_max] scale words -> u8 [len(rows), n_blocks] for one plane."""
    w = np.asarray(words).view(np.uint32)[:, plane, :]            # [G, P_max]
    by = w.view(np.uint8).reshape(w.shape[0], w.shape[1], 4)      # little endian: byte i = block 4g+i
    by = by.transpose(1, 0, 2).reshape(w.shape[1], -1)            # [P_max, 4G]
    return by[np.asarray(rows)][:, :n_blocks]
