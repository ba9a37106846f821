"""CPU oracle for the gpt-oss MoE feed-forward block -- TEST INFRASTRUCTURE.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s cpu_baseline /
``--impl reference`` leg may import this package.  The CUDA product path never
imports, links or executes it, and the two share no code: the arithmetic lives
in ``moe_oracle.c`` (plain fp64 loops, one token at a time, each step citing the
passage of the gpt-oss write-ups it follows); this module only compiles it with
gcc and marshals numpy arrays.

Every function here is pinned by the ``-m "not gpu"`` tests in
``tests/test_oracle_*.py`` (decode table against the OCP E2M1/E8M0 closed form,
top-k against a full stable sort, softmax identities, SwiGLU special cases,
E=1/top-1 against a dense numpy FFN, and dense brute force over all experts).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading
from typing import Dict, Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "moe_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_libs = {}


def compile_source(src_path: str, lib_path: str) -> str:
    """gcc -O2 -fopenmp, no FP contraction, into a shared library."""
    tmp = lib_path + ".tmp.%d" % os.getpid()
    cmd = ["gcc", "-O2", "-fopenmp", "-ffp-contract=off", "-fno-fast-math", "-shared", "-fPIC",
           "-o", tmp, src_path, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, lib_path)
    return lib_path


def build(force: bool = False) -> str:
    """Compile moe_oracle.c into liboracle.so when it is missing or stale."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        compile_source(_SRC, _LIB)
    return _LIB


def _declare(lib):
    P = ctypes.c_void_p
    lib.oracle_mxfp4_value.restype = ctypes.c_double
    lib.oracle_mxfp4_value.argtypes = [ctypes.c_int, ctypes.c_int]
    lib.oracle_mxfp4_bytes.restype = ctypes.c_longlong
    lib.oracle_mxfp4_bytes.argtypes = [ctypes.c_longlong, ctypes.c_longlong]
    lib.oracle_mxfp4_decode_matrix.restype = None
    lib.oracle_mxfp4_decode_matrix.argtypes = [ctypes.c_int, ctypes.c_int, P, P, P]
    lib.oracle_rmsnorm.restype = None
    lib.oracle_rmsnorm.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_double, P, P, P]
    lib.oracle_router.restype = None
    lib.oracle_router.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int, P, P, P, P]
    lib.oracle_topk_softmax.restype = None
    lib.oracle_topk_softmax.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int, P, P, P]
    lib.oracle_swiglu.restype = ctypes.c_double
    lib.oracle_swiglu.argtypes = [ctypes.c_double, ctypes.c_double]
    lib.oracle_expert.restype = None
    lib.oracle_expert.argtypes = [ctypes.c_int, ctypes.c_int, P, P, P, P, P, P, P, P, P]
    lib.oracle_moe_forward.restype = ctypes.c_int
    lib.oracle_moe_forward.argtypes = [ctypes.c_int] * 5 + [ctypes.c_double] + [P] * 14 + [ctypes.c_int]
    lib.oracle_max_threads.restype = ctypes.c_int
    lib.oracle_max_threads.argtypes = []
    return lib


def _load(path: Optional[str] = None):
    """The oracle library (default: the committed source's build)."""
    with _lock:
        key = path or "default"
        if key not in _libs:
            _libs[key] = _declare(ctypes.CDLL(path or build()))
        return _libs[key]


def _p(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def max_threads() -> int:
    return int(_load().oracle_max_threads())


def mxfp4_value(code: int, scale: int, lib=None) -> float:
    """Value of one E2M1 code under an E8M0 scale byte (NaN for 255)."""
    return float((lib or _load()).oracle_mxfp4_value(int(code), int(scale)))


def mxfp4_bytes(rows: int, K: int) -> int:
    """Storage bytes of a rows x K MXFP4 matrix (codes + scales)."""
    return int(_load().oracle_mxfp4_bytes(int(rows), int(K)))


def decode_matrix(codes: np.ndarray, scales: np.ndarray, lib=None) -> np.ndarray:
    """Dense fp64 decode of an MXFP4 matrix: codes uint8 [R, K/2], scales uint8 [R, K/32]."""
    codes = _c(codes, np.uint8)
    scales = _c(scales, np.uint8)
    R, K = codes.shape[0], codes.shape[1] * 2
    assert scales.shape == (R, K // 32)
    out = np.empty((R, K), dtype=np.float64)
    (lib or _load()).oracle_mxfp4_decode_matrix(R, K, _p(codes), _p(scales), _p(out))
    return out


def rmsnorm(x_bits: np.ndarray, scale_bits: np.ndarray, eps: float, lib=None) -> np.ndarray:
    x_bits = _c(x_bits, np.uint16)
    scale_bits = _c(scale_bits, np.uint16)
    T, d = x_bits.shape
    out = np.empty((T, d), dtype=np.float64)
    (lib or _load()).oracle_rmsnorm(T, d, float(eps), _p(x_bits), _p(scale_bits), _p(out))
    return out


def router(xn: np.ndarray, w_bits: np.ndarray, b: np.ndarray, lib=None) -> np.ndarray:
    xn = _c(xn, np.float64)
    w_bits = _c(w_bits, np.uint16)
    b = _c(b, np.float32)
    T, d = xn.shape
    E = w_bits.shape[0]
    out = np.empty((T, E), dtype=np.float32)
    (lib or _load()).oracle_router(T, d, E, _p(xn), _p(w_bits), _p(b), _p(out))
    return out


def topk_softmax(logits: np.ndarray, k: int, lib=None):
    logits = _c(logits, np.float32)
    T, E = logits.shape
    idx = np.empty((T, k), dtype=np.int32)
    w = np.empty((T, k), dtype=np.float64)
    (lib or _load()).oracle_topk_softmax(T, E, int(k), _p(logits), _p(idx), _p(w))
    return idx, w


def swiglu(gate: float, lin: float, lib=None) -> float:
    return float((lib or _load()).oracle_swiglu(float(gate), float(lin)))


def expert(inp: Dict[str, np.ndarray], e: int, xn_t: np.ndarray, lib=None):
    """One expert on one normalised token: returns (h [F], o [d]) in fp64."""
    w13c = _c(inp["w13_codes"][e], np.uint8)
    w13s = _c(inp["w13_scales"][e], np.uint8)
    b13 = _c(inp["b13"][e], np.uint16)
    w2c = _c(inp["w2_codes"][e], np.uint8)
    w2s = _c(inp["w2_scales"][e], np.uint8)
    b2 = _c(inp["b2"][e], np.uint16)
    d = w2c.shape[0]
    F = w13c.shape[0] // 2
    xn_t = _c(xn_t, np.float64)
    h = np.empty(F, dtype=np.float64)
    o = np.empty(d, dtype=np.float64)
    (lib or _load()).oracle_expert(d, F, _p(xn_t), _p(w13c), _p(w13s), _p(b13), _p(w2c), _p(w2s), _p(b2), _p(h), _p(o))
    return h, o


def moe_forward(inp: Dict[str, np.ndarray], k: int, eps: float, x: Optional[np.ndarray] = None,
                threads: int = 0, lib=None) -> Dict[str, np.ndarray]:
    """The whole block on the rows of ``x`` (default ``inp['x']``).

    Returns ``y`` [T, d] fp64, ``idx`` [T, k] int32, ``w`` [T, k] fp64 and the fp32
    router ``logits`` [T, E].
    """
    x = _c(inp["x"] if x is None else x, np.uint16)
    T, d = x.shape
    E = inp["router_w"].shape[0]
    F = inp["w13_codes"].shape[1] // 2
    arrs = [_c(inp["norm_scale"], np.uint16), _c(inp["router_w"], np.uint16), _c(inp["router_b"], np.float32),
            _c(inp["w13_codes"], np.uint8), _c(inp["w13_scales"], np.uint8), _c(inp["b13"], np.uint16),
            _c(inp["w2_codes"], np.uint8), _c(inp["w2_scales"], np.uint8), _c(inp["b2"], np.uint16)]
    y = np.empty((T, d), dtype=np.float64)
    idx = np.empty((T, k), dtype=np.int32)
    w = np.empty((T, k), dtype=np.float64)
    logits = np.empty((T, E), dtype=np.float32)
    rc = (lib or _load()).oracle_moe_forward(T, d, F, E, int(k), float(eps), _p(x), *[_p(a) for a in arrs],
                                             _p(y), _p(idx), _p(w), _p(logits), int(threads))
    if rc != 0:
        raise ValueError("oracle_moe_forward rejected the shape (T=%d d=%d F=%d E=%d k=%d)" % (T, d, F, E, k))
    return {"y": y, "idx": idx, "w": w, "logits": logits}


def load_variant(lib_path: str):
    """A separately built copy of the oracle (the pin tests use this to show that
    a mistake planted in a copy of the source makes a pin fail)."""
    return _load(lib_path)
