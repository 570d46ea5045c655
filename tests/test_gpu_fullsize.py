"""The five workloads at their full sizes, in the launch configuration
bench.py times, checked against the oracle on sampled tokens (the oracle
computes each sampled token's output from the per-token definition)."""
import json
import os

import numpy as np
import pytest

import mixture_experts_layer_22_b200 as moe
from mixture_experts_layer_22_b200 import synthetic as syn
from helpers import BF16_TOL, FP8_TOL, Layer, oracle_forward, rel_err

pytestmark = pytest.mark.gpu

W = syn.WORKLOADS
GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _sample(T, n, ids=None):
    toks = set(np.linspace(0, T - 1, n).astype(int).tolist())
    return np.array(sorted(toks), dtype=np.int32)


def _check(wl, tol, a2=1.0, n_tok=8, variant=moe.AUTO):
    d = syn.make_inputs(wl)
    L = Layer(wl, d, variant=variant, a2=a2)
    got = L.run()
    assert L.status() == 0
    toks = _sample(wl.T, n_tok)
    ref = oracle_forward(wl, d, tokens=toks, a2=a2)
    err = rel_err(got[toks], ref, "bf16")
    assert err <= tol, err
    return got


def test_full_mixtral_decode_T64():
    _check(W["mixtral_decode"], BF16_TOL)


def test_full_qwen2_skewed_prefill_T8192():
    wl = W["qwen2_skewed_prefill"]
    got = _check(wl, BF16_TOL, n_tok=10)
    assert np.isfinite(got).all()


def test_full_mixtral_prefill_fp8_T4096():
    with open(os.path.join(GOLDEN, "mixtral_prefill_fp8_hidden_scale.json")) as f:
        a2 = json.load(f)["a2"]
    _check(W["mixtral_prefill_fp8"], FP8_TOL, a2=a2, n_tok=8)


@pytest.mark.parametrize("T", [1, 8, 32, 128])
def test_full_dsv3_decode_fp8_weights(T):
    _check(W["dsv3_decode_fp8w"].with_T(T), FP8_TOL, n_tok=min(T, 6))
