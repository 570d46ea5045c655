"""The five workloads at their full sizes, in the launch configuration
bench.py times, checked against the oracle.

Decode batches (T <= 128) are checked on every token.  Prefill batches are
checked on a set of tokens chosen from the oracle's own routing and
alignment: at least one token for every 64-row block of every expert's
segment, so that every row tile the full-size launch produces is checked
(GEMM1's 128-row tiles, both 128-row halves of every 256-row CTA-pair tile of
GEMM2, and the stream-K split tiles, which are row tiles too), plus evenly
spaced tokens up to a budget the oracle finishes in seconds.  Each check
prints the raw max|err|/rms next to the figure the bound is applied to (the
raw one minus each element's half-ulp of the bf16 reference)."""
import json
import os

import numpy as np
import pytest

import oracle as orc
import mixture_experts_layer_22_b200 as moe
from mixture_experts_layer_22_b200 import synthetic as syn
from helpers import BF16_TOL, FP8_TOL, Layer, oracle_forward, rel_err

pytestmark = pytest.mark.gpu

W = syn.WORKLOADS
GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")
PAD = 16                       # the segment padding Layer and bench.py use
BLOCK = 64                     # finest row-tile granularity of any launch here

_weights = {}


def _inputs(wl):
    """make_inputs with the (large) expert weights generated once per layer
    shape and reused across token counts."""
    key = (wl.H, wl.I, wl.E, wl.n_shared, wl.wdtype, wl.seed)     # the weights' own generator key
    d = syn.make_inputs(wl, weights=key not in _weights)
    if key in _weights:
        d.update(_weights[key])
    else:
        _weights.clear()
        _weights[key] = {n: d[n] for n in ("w13", "w13_scale", "w2", "w2_scale")}
    return d


def tile_cover_tokens(wl, d, budget):
    """Tokens that touch every BLOCK-row block of every expert segment (the
    oracle's align on the oracle's routing), topped up with evenly spaced
    tokens to `budget`."""
    ids, _ = orc.route(d["logits"], wl.k, gate=wl.gate, renorm=wl.renorm, routed_scale=wl.routed_scale)
    counts, offsets, rows, _ = orc.align(ids, wl.E, wl.n_shared, PAD)
    R = wl.T * wl.k
    toks = set()
    for e in range(wl.E + wl.n_shared):
        for b in range(0, int(counts[e]), BLOCK):
            f = int(rows[offsets[e] + b])
            toks.add(f // wl.k if f < R else (f - R) % wl.T)
    need = len(toks)
    extra = max(0, budget - need)
    toks.update(np.linspace(0, wl.T - 1, extra).astype(int).tolist())
    return np.array(sorted(toks), dtype=np.int32), need


def _check(wl, tol, a2=1.0, budget=None):
    d = _inputs(wl)
    L = Layer(wl, d, a2=a2)
    got = L.run()
    assert L.status() == 0
    if budget is None or budget >= wl.T:
        toks, need = np.arange(wl.T, dtype=np.int32), wl.T
    else:
        toks, need = tile_cover_tokens(wl, d, budget)
    ref = oracle_forward(wl, d, tokens=toks, a2=a2)
    err = rel_err(got[toks], ref, "bf16")
    rms = float(np.sqrt(np.mean(np.square(ref))))
    raw = float(np.max(np.abs(got[toks] - ref))) / rms
    print(f"\n{wl.name} T={wl.T}: {len(toks)} tokens checked ({need} cover every {BLOCK}-row block); "
          f"raw max|err|/rms = {raw:.3e}, beyond half-ulp = {err:.3e}, bound {tol:.0e}")
    assert err <= tol, err
    return got


def test_full_mixtral_decode_T64():
    _check(W["mixtral_decode"], BF16_TOL)


@pytest.mark.parametrize("T", [1, 8])
def test_full_mixtral_decode_small_batches(T):
    _check(W["mixtral_decode"].with_T(T), BF16_TOL)


def test_full_qwen2_skewed_prefill_T8192():
    got = _check(W["qwen2_skewed_prefill"], BF16_TOL, budget=1024)
    assert np.isfinite(got).all()


def test_full_mixtral_prefill_fp8_T4096():
    with open(os.path.join(GOLDEN, "mixtral_prefill_fp8_hidden_scale.json")) as f:
        a2 = json.load(f)["a2"]
    _check(W["mixtral_prefill_fp8"], FP8_TOL, a2=a2, budget=160)


@pytest.mark.parametrize("T", [1, 8, 32, 128])
def test_full_dsv3_decode_fp8_weights(T):
    # E4M3 weights with bf16 activations: the oracle works on the same E4M3
    # weight values and the bf16 tokens, so the bf16 bound applies
    _check(W["dsv3_decode_fp8w"].with_T(T), BF16_TOL)


@pytest.mark.parametrize("T", [1, 8, 32, 128])
def test_full_dsv3_decode_fp8_activations(T):
    """The same layer with E4M3 activations as well (static per-tensor scales
    a1, a2 calibrated once on the 128 seeded tokens): one E4M3 plane per token
    row on the kind::f8f6f4 tensor path; the oracle quantises x and h with the
    same scales."""
    wl = W["dsv3_decode_fp8"].with_T(T)
    with open(os.path.join(GOLDEN, "dsv3_decode_fp8_hidden_scale.json")) as f:
        a2 = json.load(f)["a2"]
    _check(wl, FP8_TOL, a2=a2)
