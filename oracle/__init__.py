"""CPU oracle for the fused Mixture-of-Experts layer -- TEST INFRASTRUCTURE.

Only the test-suite, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product path (the CUDA library and
its Python binding) never touches it, and it never touches them.

This module is argument marshalling around ``moe_oracle.c``: a plain per-token,
double-precision implementation of the layer written from its definition (see
the header of that file for the passages it follows).  Arrays are numpy;
bf16 tensors travel as their uint16 bit patterns, E4M3 tensors as uint8 codes.
"""
from __future__ import annotations

import ctypes as C
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "moe_oracle.c")
_LIB = os.path.join(_HERE, "libmoe_oracle.so")

BF16, E4M3 = 0, 1
SOFTMAX, SIGMOID = 0, 1

_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (-O2, OpenMP, no fast-math, no contraction of
    a * b + c into a fused multiply-add)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fno-fast-math", "-ffp-contract=off", "-shared", "-fPIC",
                               "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = C.CDLL(build())
            P = C.c_void_p
            i, l, d, f = C.c_int, C.c_long, C.c_double, C.c_float
            lib.orc_bf16_decode.restype = d
            lib.orc_bf16_decode.argtypes = [C.c_uint16]
            lib.orc_e4m3_decode.restype = d
            lib.orc_e4m3_decode.argtypes = [C.c_uint8]
            lib.orc_e4m3_encode.restype = C.c_uint8
            lib.orc_e4m3_encode.argtypes = [d]
            lib.orc_bf16_encode.restype = C.c_uint16
            lib.orc_bf16_encode.argtypes = [d]
            lib.orc_quant_e4m3_f32.restype = None
            lib.orc_quant_e4m3_f32.argtypes = [P, f, P, l]
            lib.orc_router_logits.restype = None
            lib.orc_router_logits.argtypes = [i, i, i, P, P, P]
            lib.orc_route.restype = None
            lib.orc_route.argtypes = [i, i, i, i, i, d, P, P, P]
            lib.orc_align.restype = l
            lib.orc_align.argtypes = [i, i, i, i, i, P, P, P, P, P]
            lib.orc_expert_swiglu.restype = None
            lib.orc_expert_swiglu.argtypes = [i, i, i, P, P, i, d, P, i, P, P]
            lib.orc_expert_down.restype = None
            lib.orc_expert_down.argtypes = [i, i, i, P, P, i, d, P, i, P, P]
            lib.orc_combine.restype = None
            lib.orc_combine.argtypes = [i, i, i, i, i, P, P, P, P, P]
            lib.orc_forward.restype = None
            lib.orc_forward.argtypes = [i, i, i, i, i, i, i, i, d, i, i, P, P, P, P, P, P,
                                        d, d, P, l, P]
            lib.orc_hidden_amax.restype = d
            lib.orc_hidden_amax.argtypes = [i, i, i, i, i, i, i, d, i, i, P, P, P, P, d, P, l]
            lib.orc_inv_rope_quant.restype = None
            lib.orc_inv_rope_quant.argtypes = [i, i, i, i, i, P, P, P, i, P, P]
            lib.orc_num_threads.restype = i
            lib.orc_num_threads.argtypes = []
            _lib = lib
    return _lib


def _p(a: np.ndarray | None):
    if a is None:
        return None
    assert a.flags["C_CONTIGUOUS"], "oracle arrays must be C-contiguous"
    return a.ctypes.data_as(C.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def num_threads() -> int:
    return _load().orc_num_threads()


# ---------------------------------------------------------------- formats
def e4m3_decode(codes) -> np.ndarray:
    lib = _load()
    codes = np.asarray(codes, dtype=np.uint8)
    return np.array([lib.orc_e4m3_decode(int(c)) for c in codes.ravel()]).reshape(codes.shape)


def e4m3_encode(values) -> np.ndarray:
    lib = _load()
    v = np.asarray(values, dtype=np.float64)
    return np.array([lib.orc_e4m3_encode(float(x)) for x in v.ravel()], dtype=np.uint8).reshape(v.shape)


def bf16_decode(bits) -> np.ndarray:
    b = np.asarray(bits, dtype=np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def bf16_encode(values) -> np.ndarray:
    lib = _load()
    v = np.asarray(values, dtype=np.float64)
    return np.array([lib.orc_bf16_encode(float(x)) for x in v.ravel()], dtype=np.uint16).reshape(v.shape)


def quant_e4m3_f32(values, scale: float) -> np.ndarray:
    """E4M3 codes of fp32(values / scale) (quotient formed in fp32)."""
    v = _c(values, np.float32)
    out = np.empty(v.shape, dtype=np.uint8)
    _load().orc_quant_e4m3_f32(_p(v), C.c_float(scale), _p(out), v.size)
    return out


# ---------------------------------------------------------------- routing
def router_logits(x_bits, wg_bits) -> np.ndarray:
    """Router logits [T, E] fp32 from x [T, H] and Wg [E, H] (bf16 bits), in
    the fixed summation order the C function documents."""
    xb = _c(x_bits, np.uint16)
    wb = _c(wg_bits, np.uint16)
    T, H = xb.shape
    E = wb.shape[0]
    if wb.shape[1] != H or H % 8:
        raise ValueError("x [T,H] and Wg [E,H] with H a multiple of 8 expected")
    out = np.empty((T, E), dtype=np.float32)
    _load().orc_router_logits(T, E, H, _p(xb), _p(wb), _p(out))
    return out


def route(logits, k: int, gate: int = SOFTMAX, renorm: bool = True, routed_scale: float = 1.0):
    lg = _c(logits, np.float32)
    T, E = lg.shape
    ids = np.empty((T, k), dtype=np.int32)
    w = np.empty((T, k), dtype=np.float64)
    _load().orc_route(T, E, k, gate, int(renorm), routed_scale, _p(lg), _p(ids), _p(w))
    return ids, w


def max_rows(T: int, k: int, E: int, n_shared: int, pad: int) -> int:
    return T * k + n_shared * T + (E + n_shared) * (pad - 1)


def align(ids, E: int, n_shared: int = 0, pad: int = 16):
    ids = _c(ids, np.int32)
    T, k = ids.shape
    Et = E + n_shared
    counts = np.empty(Et, dtype=np.int32)
    offsets = np.empty(Et + 1, dtype=np.int32)
    rows = np.empty(max_rows(T, k, E, n_shared, pad), dtype=np.int32)
    inv = np.empty(T * k, dtype=np.int32)
    total = _load().orc_align(T, k, E, n_shared, pad, _p(ids), _p(counts), _p(offsets), _p(rows), _p(inv))
    return counts, offsets, rows[:total].copy(), inv


def gather(x_bits, sorted_rows, k: int, T: int, n_shared: int = 0):
    """xp[s] = x[token of row code s] (bf16 bits), zero rows for pad slots."""
    x_bits = np.asarray(x_bits)
    R = T * k
    xp = np.zeros((len(sorted_rows), x_bits.shape[1]), dtype=x_bits.dtype)
    for s, f in enumerate(sorted_rows):
        if f < 0:
            continue
        t = f // k if f < R else (f - R) % T
        xp[s] = x_bits[t]
    return xp


# ---------------------------------------------------------------- expert math
def expert_swiglu(xp, offsets, w13, wdtype: int, w13_scale=None, adtype: int = BF16, a1: float = 1.0):
    xp = np.ascontiguousarray(xp)
    offsets = _c(offsets, np.int32)
    w13 = np.ascontiguousarray(w13)
    Et = offsets.size - 1
    H = xp.shape[1]
    I = w13.shape[1] // 2
    h = np.zeros((xp.shape[0], I), dtype=np.float64)
    sc = None if w13_scale is None else _c(w13_scale, np.float32)
    _load().orc_expert_swiglu(H, I, Et, _p(offsets), _p(xp), adtype, a1, _p(w13), wdtype, _p(sc), _p(h))
    return h


def expert_down(h, offsets, w2, wdtype: int, w2_scale=None, adtype: int = BF16, a2: float = 1.0):
    h = np.ascontiguousarray(h)
    offsets = _c(offsets, np.int32)
    w2 = np.ascontiguousarray(w2)
    Et = offsets.size - 1
    I = h.shape[1]
    H = w2.shape[1]
    y = np.zeros((h.shape[0], H), dtype=np.float64)
    sc = None if w2_scale is None else _c(w2_scale, np.float32)
    _load().orc_expert_down(H, I, Et, _p(offsets), _p(h), adtype, a2, _p(w2), wdtype, _p(sc), _p(y))
    return y


def combine(y, w, inv, offsets, E: int, n_shared: int = 0):
    y = _c(y, np.float64)
    w = _c(w, np.float64)
    inv = _c(inv, np.int32)
    offsets = _c(offsets, np.int32)
    T, k = w.shape
    H = y.shape[1]
    out = np.empty((T, H), dtype=np.float64)
    _load().orc_combine(T, H, k, E, n_shared, _p(offsets), _p(y), _p(w), _p(inv), _p(out))
    return out


# ---------------------------------------------------------------- the layer
def forward(x_bits, logits, w13, w2, *, E: int, k: int, n_shared: int = 0, gate: int = SOFTMAX,
            renorm: bool = True, routed_scale: float = 1.0, wdtype: int = BF16, adtype: int = BF16,
            w13_scale=None, w2_scale=None, a1: float = 1.0, a2: float = 1.0, tokens=None):
    """Per-token dense definition; returns double [len(tokens), H]."""
    x_bits = _c(x_bits, np.uint16)
    lg = _c(logits, np.float32)
    T, H = x_bits.shape
    I = w13.shape[1] // 2
    w13 = np.ascontiguousarray(w13)
    w2 = np.ascontiguousarray(w2)
    toks = _c(np.arange(T) if tokens is None else tokens, np.int32)
    out = np.empty((toks.size, H), dtype=np.float64)
    s13 = None if w13_scale is None else _c(w13_scale, np.float32)
    s2 = None if w2_scale is None else _c(w2_scale, np.float32)
    _load().orc_forward(T, H, I, E, k, n_shared, gate, int(renorm), routed_scale, wdtype, adtype,
                        _p(x_bits), _p(lg), _p(w13), _p(s13), _p(w2), _p(s2), a1, a2,
                        _p(toks), toks.size, _p(out))
    return out


def hidden_amax(x_bits, logits, w13, *, E: int, k: int, n_shared: int = 0, gate: int = SOFTMAX,
                renorm: bool = True, routed_scale: float = 1.0, wdtype: int = BF16, adtype: int = BF16,
                w13_scale=None, a1: float = 1.0, tokens=None) -> float:
    x_bits = _c(x_bits, np.uint16)
    lg = _c(logits, np.float32)
    T, H = x_bits.shape
    I = w13.shape[1] // 2
    w13 = np.ascontiguousarray(w13)
    toks = _c(np.arange(T) if tokens is None else tokens, np.int32)
    s13 = None if w13_scale is None else _c(w13_scale, np.float32)
    return _load().orc_hidden_amax(H, I, E, k, n_shared, gate, int(renorm), routed_scale, wdtype,
                                   adtype, _p(x_bits), _p(lg), _p(w13), _p(s13), a1, _p(toks),
                                   toks.size)


# ---------------------------------------------------------------- attention side
def inv_rope_quant(x_bits, positions, cos_sin, rot_dim: int, interleaved: bool = False):
    """Inverse rotary embedding then per-head E4M3 quantisation.
    x_bits [T, n_heads, head_dim] bf16 bits, positions [T] int32, cos_sin
    [max_pos, rot_dim] fp32; returns (codes [T, n_heads, head_dim] uint8,
    scales [T, n_heads] fp32)."""
    xb = _c(x_bits, np.uint16)
    T, nh, hd = xb.shape
    pos = _c(positions, np.int32)
    cs = _c(cos_sin, np.float32)
    if cs.shape[1] != rot_dim or rot_dim % 2 or rot_dim > hd or pos.shape != (T,):
        raise ValueError("cos_sin [max_pos, rot_dim], even rot_dim <= head_dim, positions [T] expected")
    q = np.empty((T, nh, hd), dtype=np.uint8)
    sc = np.empty((T, nh), dtype=np.float32)
    _load().orc_inv_rope_quant(T, nh, hd, rot_dim, int(interleaved), _p(xb), _p(pos), _p(cs), cs.shape[0],
                               _p(q), _p(sc))
    return q, sc
