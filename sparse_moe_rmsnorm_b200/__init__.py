"""B200 (sm_100a) gpt-oss MoE feed-forward block.

RMSNorm -> linear router (fp32 logits) -> top-k with softmax over the chosen
experts -> MXFP4 gated-SwiGLU experts -> weighted combine -> residual, all in
hand-written CUDA kernels behind the C ABI declared in ``include/moe_b200.h``
(``libmoe_b200.so``, built in-tree by ``python -m sparse_moe_rmsnorm_b200.build``).

This module only marshals arguments: it passes tensor data pointers and the
current CUDA stream to the library.  PyTorch provides device memory and
streams.  There is no fallback: every call raises when the library or a
B200 is missing.
"""
from __future__ import annotations

import ctypes
import dataclasses
import os
from typing import Dict, Optional

__all__ = [
    "MOE_OK", "MOE_ERR_ARG", "MOE_ERR_CUDA", "MOE_ERR_TIMEOUT", "MOE_ERR_UNSUPPORTED", "MOE_ERR_NOMEM",
    "MoEError", "MoEShape", "MoEWeights", "MoE", "lib", "library_path",
    "moe_init", "moe_destroy", "moe_forward", "moe_route", "moe_group", "moe_expert_up", "moe_expert_down",
    "moe_expert_ffn", "moe_finalize", "moe_copy_workspace", "moe_sync_status", "moe_set_wait_limit_ns",
    "moe_selftest_wait_timeout", "moe_debug_decode", "moe_debug_plan", "moe_strerror", "moe_version", "WS",
    "moe_forward_noalloc", "MOE_NOALLOC_MAX_TOKENS",
]

MOE_NOALLOC_MAX_TOKENS = 64

MOE_OK, MOE_ERR_ARG, MOE_ERR_CUDA, MOE_ERR_TIMEOUT, MOE_ERR_UNSUPPORTED, MOE_ERR_NOMEM = 0, -1, -2, -3, -4, -5

# workspace buffer ids of moe_copy_workspace
WS = dict(xn=0, topk_idx=2, topk_w=3, counts=4, offsets=5, row_token=6, row_w=7, h=8, out_rows=9, tiles=10,
          pair_row=11, xperm=12, xsf=13, hsf=14)

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "libmoe_b200.so")
_lib = None


def library_path() -> str:
    return _LIB_PATH


class MoEError(RuntimeError):
    def __init__(self, code: int, what: str = ""):
        self.code = code
        super().__init__("%s%s (code %d)" % (what + ": " if what else "", moe_strerror(code), code))


class MoEShape(ctypes.Structure):
    _fields_ = [("T_max", ctypes.c_int), ("d_model", ctypes.c_int), ("d_ff", ctypes.c_int),
                ("n_experts", ctypes.c_int), ("top_k", ctypes.c_int), ("eps", ctypes.c_float)]


_SIGS = {
    "moe_init": (ctypes.c_int, [ctypes.POINTER(MoEShape), ctypes.POINTER(ctypes.c_void_p)]),
    "moe_destroy": (ctypes.c_int, [ctypes.c_void_p]),
    "moe_forward": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_int] + [ctypes.c_void_p] * 10 + [ctypes.c_int]
                    + [ctypes.c_void_p] * 4),
    "moe_route": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_int] + [ctypes.c_void_p] * 4 + [ctypes.c_int, ctypes.c_void_p]),
    "moe_group": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_int, ctypes.c_int, ctypes.c_void_p]),
    "moe_expert_up": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_int, ctypes.c_int] + [ctypes.c_void_p] * 5),
    "moe_expert_down": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_int, ctypes.c_int] + [ctypes.c_void_p] * 4),
    "moe_expert_ffn": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_int, ctypes.c_int] + [ctypes.c_void_p] * 7),
    "moe_finalize": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_int, ctypes.c_int] + [ctypes.c_void_p] * 5),
    "moe_copy_workspace": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p, ctypes.c_size_t,
                                          ctypes.c_void_p]),
    "moe_sync_status": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_void_p]),
    "moe_set_wait_limit_ns": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_ulonglong]),
    "moe_selftest_wait_timeout": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_void_p]),
    "moe_debug_decode": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int, ctypes.c_int,
                                        ctypes.c_void_p, ctypes.c_void_p]),
    "moe_forward_noalloc": (ctypes.c_int, [ctypes.c_int] * 5 + [ctypes.c_float] + [ctypes.c_void_p] * 12),
    "moe_debug_plan": (ctypes.c_int, [ctypes.c_int] * 8 + [ctypes.c_void_p]),
    "moe_strerror": (ctypes.c_char_p, [ctypes.c_int]),
    "moe_version": (ctypes.c_char_p, []),
}


def lib():
    """The loaded CUDA library (raises when it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(_LIB_PATH):
            raise RuntimeError("libmoe_b200.so is not built; run `python -m sparse_moe_rmsnorm_b200.build` "
                               "(there is no CPU fallback)")
        L = ctypes.CDLL(_LIB_PATH)
        for name, (res, args) in _SIGS.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def _ptr(t) -> Optional[int]:
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(rc: int, what: str) -> int:
    if rc != MOE_OK:
        raise MoEError(rc, what)
    return rc


# ------------------------------------------------------- C-ABI-named wrappers

def moe_strerror(code: int) -> str:
    return lib().moe_strerror(int(code)).decode()


def moe_version() -> str:
    return lib().moe_version().decode()


def moe_init(shape: MoEShape) -> int:
    h = ctypes.c_void_p()
    _check(lib().moe_init(ctypes.byref(shape), ctypes.byref(h)), "moe_init")
    return h.value


def moe_destroy(ctx: int) -> None:
    lib().moe_destroy(ctx)


def moe_forward(ctx, T, x, router_w, router_b, w13_codes, w13_scales, b13, w2_codes, w2_scales, b2, norm_scale,
                top_k, y, topk_idx_out=None, topk_w_out=None, stream=None) -> None:
    _check(lib().moe_forward(ctx, int(T), _ptr(x), _ptr(router_w), _ptr(router_b), _ptr(w13_codes),
                             _ptr(w13_scales), _ptr(b13), _ptr(w2_codes), _ptr(w2_scales), _ptr(b2),
                             _ptr(norm_scale), int(top_k), _ptr(y), _ptr(topk_idx_out), _ptr(topk_w_out),
                             _stream(stream)), "moe_forward")


def moe_route(ctx, T, x, norm_scale, router_w, router_b, top_k, stream=None) -> None:
    _check(lib().moe_route(ctx, int(T), _ptr(x), _ptr(norm_scale), _ptr(router_w), _ptr(router_b), int(top_k),
                           _stream(stream)), "moe_route")


def moe_group(ctx, T, top_k, stream=None) -> None:
    _check(lib().moe_group(ctx, int(T), int(top_k), _stream(stream)), "moe_group")


def moe_expert_up(ctx, T, top_k, w13_codes, w13_scales, b13, w2_scales, stream=None) -> None:
    _check(lib().moe_expert_up(ctx, int(T), int(top_k), _ptr(w13_codes), _ptr(w13_scales), _ptr(b13),
                               _ptr(w2_scales), _stream(stream)), "moe_expert_up")


def moe_expert_down(ctx, T, top_k, w2_codes, w2_scales, b2, stream=None) -> None:
    _check(lib().moe_expert_down(ctx, int(T), int(top_k), _ptr(w2_codes), _ptr(w2_scales), _ptr(b2),
                                 _stream(stream)), "moe_expert_down")


def moe_expert_ffn(ctx, T, top_k, w13_codes, w13_scales, b13, w2_codes, w2_scales, b2, stream=None) -> bool:
    """Both expert GEMMs in one launch; False (nothing launched) where the batch or shape does
    not allow it, and the caller runs moe_expert_up and moe_expert_down."""
    rc = lib().moe_expert_ffn(ctx, int(T), int(top_k), _ptr(w13_codes), _ptr(w13_scales), _ptr(b13),
                              _ptr(w2_codes), _ptr(w2_scales), _ptr(b2), _stream(stream))
    if rc == MOE_ERR_UNSUPPORTED:
        return False
    _check(rc, "moe_expert_ffn")
    return True


def moe_finalize(ctx, T, top_k, x, y, topk_idx_out=None, topk_w_out=None, stream=None) -> None:
    _check(lib().moe_finalize(ctx, int(T), int(top_k), _ptr(x), _ptr(y), _ptr(topk_idx_out), _ptr(topk_w_out),
                              _stream(stream)), "moe_finalize")


def moe_forward_noalloc(T, d_model, d_ff, n_experts, top_k, eps, x, router_w, router_b, w13_codes, w13_scales, b13,
                        w2_codes, w2_scales, b2, norm_scale, y, stream=None) -> None:
    """The whole block with no device allocation (library-owned fixed scratch; see the C header)."""
    _check(lib().moe_forward_noalloc(int(T), int(d_model), int(d_ff), int(n_experts), int(top_k), float(eps),
                                     _ptr(x), _ptr(router_w), _ptr(router_b), _ptr(w13_codes), _ptr(w13_scales),
                                     _ptr(b13), _ptr(w2_codes), _ptr(w2_scales), _ptr(b2), _ptr(norm_scale), _ptr(y),
                                     _stream(stream)), "moe_forward_noalloc")


def moe_copy_workspace(ctx, which, dst, nbytes, stream=None) -> None:
    _check(lib().moe_copy_workspace(ctx, int(which), _ptr(dst), int(nbytes), _stream(stream)),
           "moe_copy_workspace")


def moe_sync_status(ctx, stream=None) -> int:
    return int(lib().moe_sync_status(ctx, _stream(stream)))


def moe_set_wait_limit_ns(ctx, ns: int) -> None:
    _check(lib().moe_set_wait_limit_ns(ctx, int(ns)), "moe_set_wait_limit_ns")


def moe_selftest_wait_timeout(ctx, stream=None) -> None:
    _check(lib().moe_selftest_wait_timeout(ctx, _stream(stream)), "moe_selftest_wait_timeout")


def moe_debug_decode(codes, scales, R, K, out, stream=None) -> None:
    _check(lib().moe_debug_decode(_ptr(codes), _ptr(scales), int(R), int(K), _ptr(out), _stream(stream)),
           "moe_debug_decode")


PLAN_FIELDS = ("nb_rows", "stacked", "n_stages", "sf_item", "grid", "smem", "tmem_cols", "k_full_stages",
               "k_stages", "row_blocks")


def moe_debug_plan(mode: int, T: int, top_k: int, d_model: int, d_ff: int, n_experts: int, P_max: int,
                   num_sms: int) -> Dict[str, int]:
    """The grouped-GEMM launch plan of one stage (mode 0 gate/up, 1 down), computed on the host."""
    out = (ctypes.c_int * len(PLAN_FIELDS))()
    _check(lib().moe_debug_plan(int(mode), int(T), int(top_k), int(d_model), int(d_ff), int(n_experts), int(P_max),
                                int(num_sms), out), "moe_debug_plan")
    return dict(zip(PLAN_FIELDS, list(out)))


# ------------------------------------------------------------- torch layer

@dataclasses.dataclass
class MoEWeights:
    """One layer's parameters as device tensors in the boundary layout."""
    router_w: "torch.Tensor"      # bf16 [E, d]
    router_b: "torch.Tensor"      # fp32 [E]
    w13_codes: "torch.Tensor"     # uint8 [E, 2F, d/2]
    w13_scales: "torch.Tensor"    # uint8 [E, 2F, d/32]
    b13: "torch.Tensor"           # bf16 [E, 2F]
    w2_codes: "torch.Tensor"      # uint8 [E, d, F/2]
    w2_scales: "torch.Tensor"     # uint8 [E, d, F/32]
    b2: "torch.Tensor"            # bf16 [E, d]
    norm_scale: "torch.Tensor"    # bf16 [d]

    @classmethod
    def from_numpy(cls, arrs: Dict[str, "object"], device="cuda") -> "MoEWeights":
        """From the numpy layout of ``moe_inputs`` (bf16 as uint16 bit patterns)."""
        import numpy as np
        import torch

        def bf16(a):
            return torch.from_numpy(np.ascontiguousarray(a, dtype=np.uint16).view(np.int16)).view(
                torch.bfloat16).to(device)

        def u8(a):
            return torch.from_numpy(np.ascontiguousarray(a, dtype=np.uint8)).to(device)

        return cls(router_w=bf16(arrs["router_w"]),
                   router_b=torch.from_numpy(np.ascontiguousarray(arrs["router_b"], dtype=np.float32)).to(device),
                   w13_codes=u8(arrs["w13_codes"]), w13_scales=u8(arrs["w13_scales"]), b13=bf16(arrs["b13"]),
                   w2_codes=u8(arrs["w2_codes"]), w2_scales=u8(arrs["w2_scales"]), b2=bf16(arrs["b2"]),
                   norm_scale=bf16(arrs["norm_scale"]))

    @property
    def n_experts(self) -> int:
        return int(self.router_w.shape[0])

    @property
    def d_model(self) -> int:
        return int(self.router_w.shape[1])

    @property
    def d_ff(self) -> int:
        return int(self.w13_codes.shape[1] // 2)

    def nbytes_expert(self) -> int:
        """Bytes of one expert's codes, scales and biases."""
        E = self.n_experts
        return sum(int(t.numel() * t.element_size()) // E
                   for t in (self.w13_codes, self.w13_scales, self.b13, self.w2_codes, self.w2_scales, self.b2))


class MoE:
    """A context of the library: workspace for up to ``T_max`` tokens of one shape."""

    def __init__(self, T_max: int, d_model: int, d_ff: int, n_experts: int, top_k: int = 4, eps: float = 1e-5,
                 device=None):
        import torch
        if device is not None:
            torch.cuda.set_device(device)
        self.shape = MoEShape(int(T_max), int(d_model), int(d_ff), int(n_experts), int(top_k), float(eps))
        self.ctx = moe_init(self.shape)
        self.top_k = int(top_k)

    def close(self) -> None:
        if getattr(self, "ctx", None):
            moe_destroy(self.ctx)
            self.ctx = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def forward(self, x, w: MoEWeights, top_k: Optional[int] = None, y=None, routing: bool = False,
                stream=None):
        """y = block(x) for bf16 x [T, d] on the device; optionally also (topk_idx, topk_w)."""
        import torch
        k = self.top_k if top_k is None else int(top_k)
        T = int(x.shape[0])
        if y is None:
            y = torch.empty_like(x)
        idx = wts = None
        if routing:
            idx = torch.empty((T, k), dtype=torch.int32, device=x.device)
            wts = torch.empty((T, k), dtype=torch.float32, device=x.device)
        moe_forward(self.ctx, T, x, w.router_w, w.router_b, w.w13_codes, w.w13_scales, w.b13, w.w2_codes,
                    w.w2_scales, w.b2, w.norm_scale, k, y, idx, wts, stream)
        return (y, idx, wts) if routing else y

    def forward_host(self, x_host, w: MoEWeights, y_host, x_dev, y_dev, top_k: Optional[int] = None,
                     stream=None):
        """End-to-end call from pinned host memory: copy x in, run the block, copy y out, all
        three in order on `stream` (default: the current stream)."""
        import torch
        s = torch.cuda.current_stream() if stream is None else stream
        if isinstance(s, int):
            s = torch.cuda.ExternalStream(s)
        with torch.cuda.stream(s):
            x_dev.copy_(x_host, non_blocking=True)
            self.forward(x_dev, w, top_k=top_k, y=y_dev, stream=s)
            y_host.copy_(y_dev, non_blocking=True)
        return y_host

    def workspace(self, name: str, T: int, top_k: Optional[int] = None, stream=None):
        """A device copy of one workspace buffer for the first T tokens.

        The E4M3 operands (``xperm``, ``h``: hi, lo and lo2 planes) and their scale
        words (``xsf``, ``hsf``: hi's, also lo2's, and lo's) are returned whole, sized
        by T_max: ``xperm`` u8 [3, T_max*k, Kd], ``xsf`` int32 [Kd/128, 2, T_max*k]
        (Kd = d_model rounded up to 128; ``h`` / ``hsf`` likewise with d_ff)."""
        import torch
        k = self.top_k if top_k is None else int(top_k)
        s = self.shape
        P = T * k
        P_max = s.T_max * s.top_k
        Kd = (s.d_model + 127) // 128 * 128
        Kf = (s.d_ff + 127) // 128 * 128
        spec = {
            "xn": ((T, s.d_model), torch.float32),
            "topk_idx": ((T, k), torch.int32), "topk_w": ((T, k), torch.float32),
            "counts": ((s.n_experts,), torch.int32), "offsets": ((s.n_experts + 1,), torch.int32),
            "row_token": ((P,), torch.int32), "row_w": ((P,), torch.float32),
            "out_rows": ((P, s.d_model), torch.float32),
            "tiles": ((s.n_experts + 1,), torch.int32), "pair_row": ((P,), torch.int32),
            "xperm": ((3, P_max, Kd), torch.uint8), "xsf": ((Kd // 128, 2, P_max), torch.int32),
            "h": ((3, P_max, Kf), torch.uint8), "hsf": ((Kf // 128, 2, P_max), torch.int32),
        }[name]
        out = torch.empty(spec[0], dtype=spec[1], device="cuda")
        moe_copy_workspace(self.ctx, WS[name], out, out.numel() * out.element_size(), stream)
        return out

    def sync_status(self, stream=None) -> int:
        return moe_sync_status(self.ctx, stream)
