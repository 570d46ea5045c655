"""Shared helpers for the GPU parity tests: moving seeded inputs to the device,
running library calls and comparing with the oracle."""
from __future__ import annotations

import numpy as np
import torch

import mixture_experts_layer_22_b200 as moe
from mixture_experts_layer_22_b200 import synthetic as syn

BF16_TOL = 1e-2     # max |err| <= tol * rms(ref)
FP8_TOL = 3e-2


def dev_bf16(bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).cuda().view(torch.bfloat16)


def dev_u8(codes: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(codes)).cuda()


def dev_w(wl, a):
    return dev_bf16(a) if wl.wdtype == syn.BF16 else dev_u8(a)


def host_bf16_bits(t: torch.Tensor) -> np.ndarray:
    return t.view(torch.int16).cpu().numpy().view(np.uint16)


def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    return syn.bf16_bits_to_f32(bits).astype(np.float64)


def half_ulp(ref: np.ndarray, fmt: str = "bf16") -> np.ndarray:
    """Half a unit in the last place of each reference value in the output
    format: the error the exact answer itself picks up when stored in it
    (bf16: 8 significant bits; e4m3: 4)."""
    bits = {"bf16": 8, "e4m3": 4, "f32": 24}[fmt]
    a = np.abs(np.asarray(ref, dtype=np.float64))
    e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    return np.where(a > 0, np.exp2(e - bits), 0.0)


def rel_err(got: np.ndarray, ref: np.ndarray, fmt: str = "f32") -> float:
    """max_i (|got_i - ref_i| - half_ulp_fmt(ref_i))^+ / rms(ref).

    The layer's bound is max|err| <= tol * rms(ref); a result stored in a
    narrow format (bf16 output, E4M3 hidden vector) cannot beat the rounding
    of the exact value to that format, so each element's half-ulp of the
    reference is granted on top of the bound (for fmt="f32" it is ~0)."""
    rms = float(np.sqrt(np.mean(np.square(ref))))
    excess = np.maximum(np.abs(got - ref) - half_ulp(ref, fmt), 0.0)
    return float(np.max(excess)) / max(rms, 1e-30)


class Layer:
    """Device copies of one workload's inputs plus a fused-forward runner."""

    def __init__(self, wl, d: dict, pad: int = 16, variant: int = moe.AUTO, a2: float = 1.0):
        self.wl, self.d = wl, d
        self.shape = moe.Shape.of(wl, pad=pad, variant=variant)
        self.x = dev_bf16(d["x"])
        self.logits = torch.from_numpy(d["logits"]).cuda()
        self.w13 = dev_w(wl, d["w13"])
        self.w2 = dev_w(wl, d["w2"])
        fp8w = wl.wdtype == syn.E4M3
        self.s13 = torch.from_numpy(d["w13_scale"]).cuda() if fp8w else None
        self.s2 = torch.from_numpy(d["w2_scale"]).cuda() if fp8w else None
        self.a1 = float(d.get("a1", 1.0))
        self.a2 = a2
        self.ws = moe.workspace(self.shape)
        self.out = torch.empty((wl.T, wl.H), dtype=torch.bfloat16, device="cuda")

    def run(self):
        moe.reset_device_status(self.ws)
        moe.fused_forward(self.shape, self.x, self.logits, self.w13, self.s13, self.w2, self.s2,
                          self.a1, self.a2, self.out, self.ws)
        torch.cuda.synchronize()
        return bf16_to_f64(host_bf16_bits(self.out))

    def status(self):
        return moe.device_status(self.ws)


def oracle_forward(wl, d, tokens=None, a2: float = 1.0):
    import oracle as orc
    return orc.forward(d["x"], d["logits"], d["w13"], d["w2"], E=wl.E, k=wl.k, n_shared=wl.n_shared,
                       gate=wl.gate, renorm=wl.renorm, routed_scale=wl.routed_scale, wdtype=wl.wdtype,
                       adtype=wl.adtype, w13_scale=d["w13_scale"], w2_scale=d["w2_scale"],
                       a1=float(d.get("a1", 1.0)), a2=a2, tokens=tokens)
