"""Fused Mixture-of-Experts layer for one NVIDIA B200 (sm_100a).

Python binding of the C ABI in ``include/moe.h`` (``libmoe_b200.so``): argument
marshalling only.  Every step of the layer runs in the library's CUDA
kernels; there is no Python, PyTorch or CPU fallback.  If the library is not
built, importing the binding's entry points raises.

Tensors are torch CUDA tensors (device memory and streams are torch's);
bf16 tensors are ``torch.bfloat16``, E4M3 tensors ``torch.uint8`` codes.
"""
from __future__ import annotations

import ctypes as C
import os

import torch

BF16, E4M3 = 0, 1
SOFTMAX, SIGMOID = 0, 1
AUTO, SWAP_AB, NORMAL = 0, 1, 2

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libmoe_b200.so")

STATUS = {0: "MOE_OK", -1: "MOE_ERR_INVALID_ARG", -2: "MOE_ERR_UNSUPPORTED",
          -3: "MOE_ERR_WORKSPACE_TOO_SMALL", -4: "MOE_ERR_CUDA", -5: "MOE_ERR_DEVICE_CHECK",
          -6: "MOE_ERR_TIMEOUT"}

EXPORTS = ["moe_max_rows", "moe_workspace_size", "moe_route_topk", "moe_align_permute", "moe_gather",
           "moe_grouped_gemm_swiglu", "moe_grouped_gemm_down", "moe_combine", "moe_fused_forward",
           "moe_get_device_status", "moe_reset_device_status", "moe_status_string",
           "moe_last_launch_count", "moe_align_permute_noalloc", "moe_router_topk",
           "moe_fused_forward_router", "moe_selftest_wait_timeout", "moe_selftest_pair_abort",
           "moe_inv_rope_quant_per_head"]


class MoeError(RuntimeError):
    def __init__(self, code: int, what: str):
        self.code = code
        super().__init__(f"{what}: {STATUS.get(code, code)} ({status_string(code)})")


class Shape(C.Structure):
    """Mirror of moe_shape_t."""
    _fields_ = [("T", C.c_int32), ("H", C.c_int32), ("I", C.c_int32), ("E", C.c_int32),
                ("k", C.c_int32), ("n_shared", C.c_int32), ("gate", C.c_int32), ("renorm", C.c_int32),
                ("routed_scale", C.c_float), ("wdtype", C.c_int32), ("adtype", C.c_int32),
                ("pad", C.c_int32), ("variant", C.c_int32)]

    @classmethod
    def of(cls, wl, pad: int = 16, variant: int = AUTO, T: int | None = None) -> "Shape":
        return cls(T=wl.T if T is None else T, H=wl.H, I=wl.I, E=wl.E, k=wl.k, n_shared=wl.n_shared,
                   gate=wl.gate, renorm=int(wl.renorm), routed_scale=wl.routed_scale,
                   wdtype=wl.wdtype, adtype=wl.adtype, pad=pad, variant=variant)


class RopeShape(C.Structure):
    """Mirror of moe_rope_shape_t."""
    _fields_ = [("num_tokens", C.c_int32), ("n_heads", C.c_int32), ("head_dim", C.c_int32),
                ("rot_dim", C.c_int32), ("max_pos", C.c_int32), ("interleaved", C.c_int32)]

    @classmethod
    def of(cls, rw, T: int | None = None) -> "RopeShape":
        return cls(num_tokens=rw.T if T is None else T, n_heads=rw.n_heads, head_dim=rw.head_dim,
                   rot_dim=rw.rot_dim, max_pos=rw.max_pos, interleaved=int(rw.interleaved))


_lib = None


def lib() -> C.CDLL:
    """The loaded library; raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"libmoe_b200.so not built ({LIB_PATH}); run "
                               "`python -m mixture_experts_layer_22_b200.build`")
        L = C.CDLL(LIB_PATH)
        P, S = C.c_void_p, C.POINTER(Shape)
        sig = {
            "moe_max_rows": [S, C.POINTER(C.c_int64)],
            "moe_workspace_size": [S, C.POINTER(C.c_size_t)],
            "moe_route_topk": [S, P, P, P, P],
            "moe_align_permute": [S, P, P, P, P, P, P, C.c_size_t, P],
            "moe_gather": [S, P, P, P, C.c_float, P, P],
            "moe_grouped_gemm_swiglu": [S, P, P, P, C.c_float, C.c_float, P, P, P, C.c_size_t, P],
            "moe_grouped_gemm_down": [S, P, P, P, C.c_float, P, P, P, C.c_size_t, P],
            "moe_combine": [S, P, P, P, P, P, P],
            "moe_fused_forward": [S, P, P, P, P, P, P, C.c_float, C.c_float, P, P, C.c_size_t, P],
            "moe_get_device_status": [P, C.POINTER(C.c_int32), P],
            "moe_reset_device_status": [P, P],
            "moe_status_string": [C.c_int],
            "moe_last_launch_count": [],
            "moe_align_permute_noalloc": [S, P, P, P, P, P, P, P],
            "moe_router_topk": [S, P, P, P, P, P, P, C.c_size_t, P],
            "moe_fused_forward_router": [S, P, P, P, P, P, P, C.c_float, C.c_float, P, P, C.c_size_t, P],
            "moe_selftest_wait_timeout": [P, P, P],
            "moe_selftest_pair_abort": [S, P, P, P, P, P, C.c_size_t, P],
            "moe_inv_rope_quant_per_head": [C.POINTER(RopeShape), P, P, P, P, P, P, P],
        }
        for name, args in sig.items():
            fn = getattr(L, name)
            fn.argtypes = args
            fn.restype = C.c_char_p if name == "moe_status_string" else C.c_int
        _lib = L
    return _lib


def status_string(code: int) -> str:
    try:
        return lib().moe_status_string(code).decode()
    except RuntimeError:
        return "library not loaded"


def _ptr(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    if not t.is_cuda:
        raise ValueError("device tensor expected")
    if not t.is_contiguous():
        raise ValueError("contiguous tensor expected")
    return t.data_ptr()


def _stream(stream):
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return stream if isinstance(stream, int) else stream.cuda_stream


def _check(code: int, what: str):
    if code != 0:
        raise MoeError(code, what)


def max_rows(shape: Shape) -> int:
    v = C.c_int64()
    _check(lib().moe_max_rows(C.byref(shape), C.byref(v)), "moe_max_rows")
    return v.value


def workspace_size(shape: Shape) -> int:
    v = C.c_size_t()
    _check(lib().moe_workspace_size(C.byref(shape), C.byref(v)), "moe_workspace_size")
    return v.value


def workspace(shape: Shape, device="cuda") -> torch.Tensor:
    return torch.empty(workspace_size(shape), dtype=torch.uint8, device=device)


def last_launch_count() -> int:
    return lib().moe_last_launch_count()


def route_topk(shape, logits, ids, w, stream=None):
    _check(lib().moe_route_topk(C.byref(shape), _ptr(logits), _ptr(ids), _ptr(w), _stream(stream)),
           "moe_route_topk")


def router_topk(shape, x, wg, logits, ids, w, ws, stream=None):
    """Router logits x . wg^T (fixed summation order) and top-k in one launch."""
    _check(lib().moe_router_topk(C.byref(shape), _ptr(x), _ptr(wg), _ptr(logits), _ptr(ids), _ptr(w),
                                 _ptr(ws), ws.numel(), _stream(stream)), "moe_router_topk")


def align_permute(shape, ids, counts, offsets, sorted_rows, inv, ws, stream=None):
    _check(lib().moe_align_permute(C.byref(shape), _ptr(ids), _ptr(counts), _ptr(offsets),
                                   _ptr(sorted_rows), _ptr(inv), _ptr(ws), ws.numel(), _stream(stream)),
           "moe_align_permute")


def align_permute_noalloc(shape, ids, counts, offsets, sorted_rows, inv, status=None, stream=None):
    """moe_align_permute without a workspace: for callers that cannot allocate
    one (the library keeps the scratch in a fixed device array; calls that
    overlap on the GPU race)."""
    _check(lib().moe_align_permute_noalloc(C.byref(shape), _ptr(ids), _ptr(counts), _ptr(offsets),
                                           _ptr(sorted_rows), _ptr(inv), _ptr(status), _stream(stream)),
           "moe_align_permute_noalloc")


def gather(shape, x, sorted_rows, offsets, a1, xp, stream=None):
    _check(lib().moe_gather(C.byref(shape), _ptr(x), _ptr(sorted_rows), _ptr(offsets), a1, _ptr(xp),
                            _stream(stream)), "moe_gather")


def grouped_gemm_swiglu(shape, xp, w13, w13_scale, a1, a2, offsets, h, ws, stream=None):
    _check(lib().moe_grouped_gemm_swiglu(C.byref(shape), _ptr(xp), _ptr(w13), _ptr(w13_scale), a1, a2,
                                         _ptr(offsets), _ptr(h), _ptr(ws), ws.numel(), _stream(stream)),
           "moe_grouped_gemm_swiglu")


def grouped_gemm_down(shape, h, w2, w2_scale, a2, offsets, y, ws, stream=None):
    _check(lib().moe_grouped_gemm_down(C.byref(shape), _ptr(h), _ptr(w2), _ptr(w2_scale), a2,
                                       _ptr(offsets), _ptr(y), _ptr(ws), ws.numel(), _stream(stream)),
           "moe_grouped_gemm_down")


def combine(shape, y, w, inv, offsets, out, stream=None):
    _check(lib().moe_combine(C.byref(shape), _ptr(y), _ptr(w), _ptr(inv), _ptr(offsets), _ptr(out),
                             _stream(stream)), "moe_combine")


def fused_forward(shape, x, logits, w13, w13_scale, w2, w2_scale, a1, a2, out, ws, stream=None):
    _check(lib().moe_fused_forward(C.byref(shape), _ptr(x), _ptr(logits), _ptr(w13), _ptr(w13_scale),
                                   _ptr(w2), _ptr(w2_scale), a1, a2, _ptr(out), _ptr(ws), ws.numel(),
                                   _stream(stream)), "moe_fused_forward")


def fused_forward_router(shape, x, wg, w13, w13_scale, w2, w2_scale, a1, a2, out, ws, stream=None):
    _check(lib().moe_fused_forward_router(C.byref(shape), _ptr(x), _ptr(wg), _ptr(w13), _ptr(w13_scale),
                                          _ptr(w2), _ptr(w2_scale), a1, a2, _ptr(out), _ptr(ws), ws.numel(),
                                          _stream(stream)), "moe_fused_forward_router")


def inv_rope_quant(shape, x, positions, cos_sin, q, scales, status=None, stream=None):
    """Inverse rotary embedding + per-head E4M3 quantisation (one launch)."""
    _check(lib().moe_inv_rope_quant_per_head(C.byref(shape), _ptr(x), _ptr(positions), _ptr(cos_sin), _ptr(q),
                                             _ptr(scales), _ptr(status), _stream(stream)),
           "moe_inv_rope_quant_per_head")


def selftest_wait_timeout(ws, gave_up, stream=None):
    """Launch the failure-path self-test (about 2 s on the GPU): its bounded
    waits run out and it reports MOE_ERR_TIMEOUT in ws's status word."""
    _check(lib().moe_selftest_wait_timeout(_ptr(ws), _ptr(gave_up), _stream(stream)), "moe_selftest_wait_timeout")


def selftest_pair_abort(shape, h, w2, offsets, y, ws, stream=None):
    """The down projection with the second CTA of every CTA pair stalled
    (about 2 s on the GPU): the pairs' waits run out, they take their abort
    tear-down and MOE_ERR_TIMEOUT goes to ws's status word."""
    _check(lib().moe_selftest_pair_abort(C.byref(shape), _ptr(h), _ptr(w2), _ptr(offsets), _ptr(y), _ptr(ws),
                                         ws.numel(), _stream(stream)), "moe_selftest_pair_abort")


def device_status(ws, stream=None) -> int:
    v = C.c_int32()
    _check(lib().moe_get_device_status(_ptr(ws), C.byref(v), _stream(stream)), "moe_get_device_status")
    return v.value


def reset_device_status(ws, stream=None):
    _check(lib().moe_reset_device_status(_ptr(ws), _stream(stream)), "moe_reset_device_status")


class MoELayer:
    """One fused-MoE layer with its weights resident on the GPU.

    ``forward(x, logits)`` runs the whole layer (one moe_fused_forward call)
    and returns out [T, H] bf16.  The workspace is sized for ``max_T`` tokens
    and reused; any T <= max_T runs without re-allocation or recompilation."""

    def __init__(self, *, H, I, E, k, w13, w2, w13_scale=None, w2_scale=None, n_shared=0,
                 gate=SOFTMAX, renorm=True, routed_scale=1.0, wdtype=BF16, adtype=BF16, a1=1.0,
                 a2=1.0, pad=16, variant=AUTO, max_T=256):
        self.base = Shape(T=max_T, H=H, I=I, E=E, k=k, n_shared=n_shared, gate=gate, renorm=int(renorm),
                          routed_scale=routed_scale, wdtype=wdtype, adtype=adtype, pad=pad, variant=variant)
        self.w13, self.w2, self.w13_scale, self.w2_scale = w13, w2, w13_scale, w2_scale
        self.a1, self.a2 = a1, a2
        self.max_T = max_T
        self.ws = workspace(self.base, device=w13.device)

    def shape(self, T: int) -> Shape:
        s = Shape.from_buffer_copy(self.base)
        s.T = T
        return s

    def forward(self, x, logits, out=None, stream=None):
        T = x.shape[0]
        if T > self.max_T:
            raise ValueError(f"T={T} exceeds max_T={self.max_T}")
        s = self.shape(T)
        if self.ws.numel() < workspace_size(s):
            self.ws = workspace(s, device=x.device)
        if out is None:
            out = torch.empty((T, s.H), dtype=torch.bfloat16, device=x.device)
        fused_forward(s, x, logits, self.w13, self.w13_scale, self.w2, self.w2_scale, self.a1, self.a2,
                      out, self.ws, stream)
        return out
