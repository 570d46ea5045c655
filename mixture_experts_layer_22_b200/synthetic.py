"""Seeded synthetic inputs for the fused-MoE layer.

This module is the one piece shared by the CUDA path's tests/benchmark and the
CPU oracle: it draws the inputs and nothing else.  It holds none of the layer's
arithmetic (no routing, permutation, GEMM, activation or combine).  Weights
that are stored in FP8 are prepared here the way a checkpoint would be (one
fp32 scale per expert matrix, scale = amax / 448); that is input preparation,
not a step of the layer.

Every tensor comes from its own Philox stream keyed by (seed, tensor name,
expert), so a tensor is the same bits whatever else is generated and however
many threads generate it.  Everything is produced on the host as numpy arrays:
bf16 tensors as uint16 bit patterns, FP8 E4M3 tensors as uint8 codes.

Workloads (the layer shapes the library is measured and checked on):
  tiny                 T=16  H=256  I=512   E=8   top-2 softmax, bf16
  mixtral_decode       T=64 (1, 8) H=4096 I=14336 E=8 top-2 softmax, bf16
  mixtral_prefill_fp8  T=4096 H=4096 I=14336 E=8 top-2 softmax, E4M3 weights and
                       activations, static per-tensor scales
  dsv3_decode_fp8w     T=1/8/32/128 H=7168 I=2048 E=256 top-8 sigmoid x2.5
                       (renormalised) + 1 shared expert, E4M3 weights, bf16 acts
  dsv3_decode_fp8      the same layer (same weights and tokens) with E4M3
                       activations too: static per-tensor scales calibrated
                       on the 128 seeded tokens
  qwen2_skewed_prefill T=8192 H=2048 I=1408 E=60 top-4 softmax, bf16, router
                       logits N(0,1) + Zipf(1.2) expert bias
Attention side (the inverse-rotary + per-head E4M3 step): rope_mixtral (32
heads x 128, neox pairs, base 1e6) and rope_dsv3 (128 heads x 64, interleaved
pairs, base 1e4), T tokens at uniform random positions.
Distributions: x ~ N(0,1); router weight W_g ~ N(0, 0.02^2) in bf16 and
logits = fp32(x . W_g^T) computed in double; expert weights ~ N(0, 1/fan_in)
(standard deviation 1/sqrt(fan_in), fan_in = H for W1/W3 and I for W2).
"""
from __future__ import annotations

import dataclasses
import os
import zlib
from concurrent.futures import ThreadPoolExecutor

import numpy as np
import torch

BF16, E4M3 = 0, 1
SOFTMAX, SIGMOID = 0, 1
E4M3_MAX = 448.0


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    T: int
    H: int
    I: int
    E: int
    k: int
    n_shared: int = 0
    gate: int = SOFTMAX
    renorm: bool = True
    routed_scale: float = 1.0
    wdtype: int = BF16
    adtype: int = BF16
    logits: str = "router"          # "router" (x . W_g) or "zipf" (N(0,1) + bias)
    zipf_s: float = 1.2
    seed: int = 0
    calib_T: int = 0                # E4M3 activations: a1 from the first calib_T tokens
                                    # (0: from this batch's own T tokens)

    @property
    def E_tot(self) -> int:
        return self.E + self.n_shared

    def with_T(self, T: int) -> "Workload":
        return dataclasses.replace(self, T=T)


WORKLOADS = {
    "tiny": Workload("tiny", T=16, H=256, I=512, E=8, k=2),
    "mixtral_decode": Workload("mixtral_decode", T=64, H=4096, I=14336, E=8, k=2),
    "mixtral_prefill_fp8": Workload("mixtral_prefill_fp8", T=4096, H=4096, I=14336, E=8, k=2,
                                    wdtype=E4M3, adtype=E4M3),
    "dsv3_decode_fp8w": Workload("dsv3_decode_fp8w", T=128, H=7168, I=2048, E=256, k=8,
                                 n_shared=1, gate=SIGMOID, routed_scale=2.5, wdtype=E4M3),
    "dsv3_decode_fp8": Workload("dsv3_decode_fp8", T=128, H=7168, I=2048, E=256, k=8,
                                n_shared=1, gate=SIGMOID, routed_scale=2.5, wdtype=E4M3, adtype=E4M3,
                                calib_T=128),
    "qwen2_skewed_prefill": Workload("qwen2_skewed_prefill", T=8192, H=2048, I=1408, E=60, k=4,
                                     logits="zipf"),
}


def _rng(seed: int, name: str, index: int = 0) -> np.random.Generator:
    return np.random.Generator(np.random.Philox(key=[seed, (zlib.crc32(name.encode()) << 20) + index]))


def _normal(seed: int, name: str, index: int, shape, std: float) -> np.ndarray:
    g = _rng(seed, name, index)
    return g.standard_normal(size=shape, dtype=np.float32) * np.float32(std)


def to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round fp32 to bf16 (nearest-even, torch's cast) and return the bits."""
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16).view(
        torch.int16).numpy().view(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def to_e4m3_codes(a: np.ndarray) -> np.ndarray:
    """fp32 values already inside [-448, 448] -> E4M3 codes (torch's cast)."""
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).clamp_(-E4M3_MAX, E4M3_MAX)
    return t.to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def _threads() -> int:
    return max(1, min(32, os.cpu_count() or 1))


def _expert_matrix(seed, name, e, rows, cols, std, wdtype):
    w = _normal(seed, name, e, (rows, cols), std)
    if wdtype == BF16:
        return to_bf16_bits(w), np.float32(1.0)
    scale = np.float32(np.abs(w).max() / np.float32(E4M3_MAX))
    return to_e4m3_codes(w / scale), scale


def expert_weights(wl: Workload, which: str):
    """Stacked expert weights: W13 [E_tot, 2I, H] (I gate rows then I up rows,
    K-major) or W2 [E_tot, H, I]; plus per-expert fp32 scales (ones for bf16).
    Shared experts follow the E routed ones."""
    if which == "w13":
        rows, cols, std = 2 * wl.I, wl.H, 1.0 / np.sqrt(wl.H)
    else:
        rows, cols, std = wl.H, wl.I, 1.0 / np.sqrt(wl.I)
    dt = np.uint16 if wl.wdtype == BF16 else np.uint8
    out = np.empty((wl.E_tot, rows, cols), dtype=dt)
    scales = np.empty(wl.E_tot, dtype=np.float32)

    def one(e):
        m, s = _expert_matrix(wl.seed, which, e, rows, cols, std, wl.wdtype)
        out[e] = m
        scales[e] = s

    with ThreadPoolExecutor(_threads()) as ex:
        list(ex.map(one, range(wl.E_tot)))
    return out, scales


def tokens(wl: Workload) -> np.ndarray:
    """x [T, H] bf16 bits, N(0,1)."""
    return to_bf16_bits(_normal(wl.seed, "x", 0, (wl.T, wl.H), 1.0))


def router_weight(wl: Workload) -> np.ndarray:
    """Router (gate) weight W_g [E, H], bf16 bits, std 0.02."""
    return to_bf16_bits(_normal(wl.seed, "w_gate", 0, (wl.E, wl.H), 0.02))


def router_logits(wl: Workload, x_bits: np.ndarray) -> np.ndarray:
    """Router logits [T, E] fp32 (an input of the layer): x . W_g^T summed in
    double by numpy, or for the Zipf workload N(0,1) noise plus a Zipf bias."""
    if wl.logits == "zipf":
        n = _normal(wl.seed, "logit_noise", 0, (wl.T, wl.E), 1.0).astype(np.float64)
        r = np.arange(1, wl.E + 1, dtype=np.float64) ** (-wl.zipf_s)
        bias = np.log(r / r.sum())
        return (n + bias[None, :]).astype(np.float32)
    wg = router_weight(wl)
    xd = bf16_bits_to_f32(x_bits).astype(np.float64)
    wd = bf16_bits_to_f32(wg).astype(np.float64)
    return (xd @ wd.T).astype(np.float32)


def activation_scale(x_bits: np.ndarray) -> float:
    """Static per-tensor activation scale amax(x)/448 (fp32)."""
    return float(np.float32(np.abs(bf16_bits_to_f32(x_bits)).max() / np.float32(E4M3_MAX)))


def make_inputs(wl: Workload, weights: bool = True) -> dict:
    """All inputs of one layer call (host numpy arrays)."""
    x = tokens(wl)
    d = {"x": x, "logits": router_logits(wl, x)}
    if weights:
        d["w13"], d["w13_scale"] = expert_weights(wl, "w13")
        d["w2"], d["w2_scale"] = expert_weights(wl, "w2")
    if wl.adtype == E4M3:
        d["a1"] = activation_scale(x if not wl.calib_T else tokens(wl.with_T(wl.calib_T)))
    else:
        d["a1"] = 1.0
    return d


# ---------------------------------------------------------------- attention side
@dataclasses.dataclass(frozen=True)
class RopeWorkload:
    """Inputs of the inverse-rotary + per-head E4M3 step: T tokens of n_heads
    vectors of head_dim, the first rot_dim of which carry the rotation."""
    name: str
    T: int
    n_heads: int
    head_dim: int
    rot_dim: int
    interleaved: bool = False
    base: float = 1.0e6
    max_pos: int = 32768
    seed: int = 0

    def with_T(self, T: int) -> "RopeWorkload":
        return dataclasses.replace(self, T=T)


ROPE_WORKLOADS = {
    # Mixtral-shaped attention (32 heads of 128, rotary base 1e6, neox pairs)
    "rope_mixtral": RopeWorkload("rope_mixtral", T=8192, n_heads=32, head_dim=128, rot_dim=128),
    # DeepSeek-V3-shaped rotary part (128 heads of 64, interleaved pairs)
    "rope_dsv3": RopeWorkload("rope_dsv3", T=8192, n_heads=128, head_dim=64, rot_dim=64, interleaved=True,
                              base=1.0e4, max_pos=163840),
}


def rope_table(rw: RopeWorkload) -> np.ndarray:
    """The model's rotary table cos_sin [max_pos, rot_dim] fp32: row p holds
    cos(p w_i) for i < rot_dim/2 then sin(p w_i), w_i = base^(-2i/rot_dim),
    evaluated in double and rounded once (a constant of the model, built at
    start-up like its weights)."""
    half = rw.rot_dim // 2
    w = rw.base ** (-2.0 * np.arange(half, dtype=np.float64) / rw.rot_dim)
    ang = np.arange(rw.max_pos, dtype=np.float64)[:, None] * w[None, :]
    return np.concatenate([np.cos(ang), np.sin(ang)], axis=1).astype(np.float32)


def rope_inputs(rw: RopeWorkload) -> dict:
    """x [T, n_heads, head_dim] bf16 bits ~ N(0, 1), positions [T] int32
    uniform in [0, max_pos), and the rotary table."""
    x = to_bf16_bits(_normal(rw.seed, "rope_x", 0, (rw.T, rw.n_heads, rw.head_dim), 1.0))
    pos = _rng(rw.seed, "rope_pos").integers(0, rw.max_pos, size=rw.T, dtype=np.int32)
    return {"x": x, "positions": pos, "cos_sin": rope_table(rw)}


def random_rows(seed: int, name: str, rows: int, cols: int, dtype: int, std: float = 1.0):
    """Stand-alone activation rows (bf16 bits or E4M3 codes) used to exercise a
    single GEMM entry point in isolation."""
    v = _normal(seed, name, 0, (rows, cols), std)
    if dtype == BF16:
        return to_bf16_bits(v)
    return to_e4m3_codes(v / np.float32(np.abs(v).max() / E4M3_MAX))


def random_f32(seed: int, name: str, shape, std: float = 1.0) -> np.ndarray:
    return _normal(seed, name, 0, shape, std)
