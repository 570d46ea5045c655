"""GPU parity: every entry point of libmoe_b200.so against the CPU oracle on the
same seeded inputs.  Routing ids, counts, offsets, the permutation and the
gathered rows are compared bit for bit; floating-point outputs within
max|err| <= 1e-2 * rms(ref) (bf16) or 3e-2 * rms(ref) (FP8)."""
import dataclasses

import numpy as np
import pytest
import torch

import mixture_experts_layer_22_b200 as moe
import oracle as orc
from mixture_experts_layer_22_b200 import synthetic as syn
from helpers import (BF16_TOL, FP8_TOL, Layer, bf16_to_f64, dev_bf16, dev_u8, dev_w, host_bf16_bits,
                     oracle_forward, rel_err)

pytestmark = pytest.mark.gpu

W = syn.WORKLOADS


def _shape(wl, **kw):
    return moe.Shape.of(wl, **kw)


# ------------------------------------------------------------------ routing
ROUTE_CASES = [W["tiny"], W["mixtral_decode"], W["qwen2_skewed_prefill"],
               dataclasses.replace(W["dsv3_decode_fp8w"], wdtype=syn.BF16),
               syn.Workload("route_odd", T=333, H=128, I=128, E=37, k=5, seed=11)]


@pytest.mark.parametrize("wl", ROUTE_CASES, ids=lambda w: w.name)
def test_route_topk_bit_exact(wl):
    x = syn.tokens(wl)
    logits = syn.router_logits(wl, x)
    s = _shape(wl)
    ids = torch.empty((wl.T, wl.k), dtype=torch.int32, device="cuda")
    w = torch.empty((wl.T, wl.k), dtype=torch.float32, device="cuda")
    moe.route_topk(s, torch.from_numpy(logits).cuda(), ids, w)
    rid, rw = orc.route(logits, wl.k, wl.gate, wl.renorm, wl.routed_scale)
    assert np.array_equal(ids.cpu().numpy(), rid)
    assert np.allclose(w.cpu().numpy(), rw, rtol=2e-6, atol=2e-7)


@pytest.mark.parametrize("gate,renorm", [(syn.SOFTMAX, False), (syn.SIGMOID, False)])
def test_route_without_renorm(gate, renorm):
    wl = syn.Workload("r", T=100, H=128, I=128, E=16, k=4, gate=gate, renorm=renorm, routed_scale=1.5, seed=3)
    logits = syn.router_logits(wl, syn.tokens(wl))
    ids = torch.empty((100, 4), dtype=torch.int32, device="cuda")
    w = torch.empty((100, 4), dtype=torch.float32, device="cuda")
    moe.route_topk(_shape(wl), torch.from_numpy(logits).cuda(), ids, w)
    rid, rw = orc.route(logits, 4, gate, renorm, 1.5)
    assert np.array_equal(ids.cpu().numpy(), rid)
    assert np.allclose(w.cpu().numpy(), rw, rtol=2e-6, atol=2e-7)


def test_route_ties_and_nan():
    rng = np.random.default_rng(0)
    logits = rng.integers(-2, 3, size=(500, 40)).astype(np.float32)
    logits[0] = 0.0
    logits[1, :] = -0.0
    logits[1, 7] = 0.0
    logits[2, 3] = np.nan
    logits[3, :] = -np.inf
    wl = syn.Workload("ties", T=500, H=128, I=128, E=40, k=6)
    ids = torch.empty((500, 6), dtype=torch.int32, device="cuda")
    w = torch.empty((500, 6), dtype=torch.float32, device="cuda")
    moe.route_topk(_shape(wl), torch.from_numpy(logits).cuda(), ids, w)
    rid, _ = orc.route(logits, 6)
    assert np.array_equal(ids.cpu().numpy(), rid)


# ------------------------------------------------------------------ align
def _ids(T, E, k, seed, skew=None):
    rng = np.random.default_rng(seed)
    if skew is None:
        return np.stack([rng.permutation(E)[:k] for _ in range(T)]).astype(np.int32)
    p = np.arange(1, E + 1, dtype=np.float64) ** -skew
    p /= p.sum()
    return np.stack([rng.choice(E, size=k, replace=False, p=p) for _ in range(T)]).astype(np.int32)


ALIGN_CASES = [(16, 8, 2, 0, 16, None), (64, 8, 2, 0, 16, None), (1, 8, 2, 0, 16, None),
               (8192, 60, 4, 0, 16, 1.2), (4096, 8, 2, 0, 128, None), (128, 256, 8, 1, 16, None),
               (1000, 37, 3, 0, 1, None), (3000, 512, 8, 1, 32, 0.8), (777, 5, 5, 0, 7, None)]


@pytest.mark.parametrize("T,E,k,ns,pad,skew", ALIGN_CASES)
def test_align_permute_bit_exact(T, E, k, ns, pad, skew):
    ids = _ids(T, E, k, T + E, skew)
    wl = syn.Workload("a", T=T, H=128, I=128, E=E, k=k, n_shared=ns)
    s = _shape(wl, pad=pad)
    mr = moe.max_rows(s)
    ws = moe.workspace(s)
    moe.reset_device_status(ws)
    counts = torch.empty(E + ns, dtype=torch.int32, device="cuda")
    offsets = torch.empty(E + ns + 1, dtype=torch.int32, device="cuda")
    rows = torch.full((mr,), -7, dtype=torch.int32, device="cuda")
    inv = torch.empty(T * k, dtype=torch.int32, device="cuda")
    moe.align_permute(s, torch.from_numpy(ids).cuda(), counts, offsets, rows, inv, ws)
    c, o, r, v = orc.align(ids, E, ns, pad)
    assert np.array_equal(counts.cpu().numpy(), c)
    assert np.array_equal(offsets.cpu().numpy(), o)
    assert np.array_equal(rows.cpu().numpy()[:o[-1]], r)
    assert np.array_equal(inv.cpu().numpy(), v)
    assert moe.device_status(ws) == 0


def test_align_one_expert_takes_all_and_empty_experts():
    T, E, k = 300, 16, 1
    ids = np.full((T, k), 5, dtype=np.int32)
    wl = syn.Workload("a", T=T, H=128, I=128, E=E, k=k)
    s = _shape(wl, pad=16)
    ws = moe.workspace(s)
    moe.reset_device_status(ws)
    counts = torch.empty(E, dtype=torch.int32, device="cuda")
    offsets = torch.empty(E + 1, dtype=torch.int32, device="cuda")
    rows = torch.empty(moe.max_rows(s), dtype=torch.int32, device="cuda")
    inv = torch.empty(T, dtype=torch.int32, device="cuda")
    moe.align_permute(s, torch.from_numpy(ids).cuda(), counts, offsets, rows, inv, ws)
    c, o, r, v = orc.align(ids, E, 0, 16)
    assert np.array_equal(offsets.cpu().numpy(), o) and np.array_equal(inv.cpu().numpy(), v)
    assert np.array_equal(rows.cpu().numpy()[:o[-1]], r)


def test_align_rejects_out_of_range_id_via_device_status():
    ids = _ids(50, 8, 2, 1)
    ids[7, 1] = 8          # == E: invalid
    ids[9, 0] = -3
    wl = syn.Workload("a", T=50, H=128, I=128, E=8, k=2)
    s = _shape(wl)
    ws = moe.workspace(s)
    moe.reset_device_status(ws)
    counts = torch.empty(8, dtype=torch.int32, device="cuda")
    offsets = torch.empty(9, dtype=torch.int32, device="cuda")
    rows = torch.empty(moe.max_rows(s), dtype=torch.int32, device="cuda")
    inv = torch.empty(100, dtype=torch.int32, device="cuda")
    moe.align_permute(s, torch.from_numpy(ids).cuda(), counts, offsets, rows, inv, ws)
    assert moe.device_status(ws) == -5
    assert int(counts.sum()) == 98
    iv = inv.cpu().numpy()
    assert iv[15] == -1 and iv[18] == -1


# ------------------------------------------------------------------ gather
@pytest.mark.parametrize("adtype", [syn.BF16, syn.E4M3])
def test_gather_bit_exact(adtype):
    T, E, k, H = 200, 8, 2, 512
    wl = syn.Workload("g", T=T, H=H, I=128, E=E, k=k, n_shared=1, wdtype=adtype, adtype=adtype)
    x = syn.tokens(wl)
    ids = _ids(T, E, k, 5)
    c, o, r, v = orc.align(ids, E, 1, 16)
    s = _shape(wl)
    mr = moe.max_rows(s)
    rows = np.full(mr, -1, np.int32)
    rows[:len(r)] = r
    a1 = syn.activation_scale(x)
    esz = 2 if adtype == syn.BF16 else 1
    xp = torch.zeros((mr, H * esz), dtype=torch.uint8, device="cuda")
    moe.gather(s, dev_bf16(x), torch.from_numpy(rows).cuda(), torch.from_numpy(o).cuda(), a1, xp)
    got = xp.cpu().numpy()[:o[-1]]
    ref_bits = orc.gather(x, r, k, T, 1)
    if adtype == syn.BF16:
        assert np.array_equal(got.view(np.uint16), ref_bits)
    else:
        ref = orc.quant_e4m3_f32(syn.bf16_bits_to_f32(ref_bits), a1)
        assert np.array_equal(got, ref)


# ------------------------------------------------------------------ grouped GEMMs alone
def _segments(T, E, k, ns, pad, seed):
    ids = _ids(T, E, k, seed)
    return orc.align(ids, E, ns, pad)


GEMM_CASES = [  # (name, T, H, I, E, k, ns, variant, weight dtype, activation dtype)
    ("swap_tiny", 16, 256, 512, 8, 2, 0, moe.SWAP_AB, syn.BF16, syn.BF16),
    ("normal_tiny", 16, 256, 512, 8, 2, 0, moe.NORMAL, syn.BF16, syn.BF16),
    ("swap_decode", 64, 1024, 1024, 8, 2, 0, moe.SWAP_AB, syn.BF16, syn.BF16),
    ("normal_prefill", 700, 512, 384, 6, 2, 0, moe.NORMAL, syn.BF16, syn.BF16),
    ("swap_shared", 40, 256, 256, 16, 4, 1, moe.SWAP_AB, syn.BF16, syn.BF16),
    ("swap_fp8", 64, 512, 512, 8, 2, 0, moe.SWAP_AB, syn.E4M3, syn.E4M3),
    ("normal_fp8", 500, 512, 512, 8, 2, 0, moe.NORMAL, syn.E4M3, syn.E4M3),
    ("w8a16_decode", 32, 1024, 512, 16, 8, 1, moe.AUTO, syn.E4M3, syn.BF16),
    ("w8a16_t128", 128, 512, 256, 32, 8, 1, moe.AUTO, syn.E4M3, syn.BF16),
    ("w8a16_t1", 1, 768, 384, 8, 4, 1, moe.AUTO, syn.E4M3, syn.BF16),
    ("w8a16_multi_tile", 300, 256, 256, 4, 2, 0, moe.AUTO, syn.E4M3, syn.BF16),
]


def _act(dt, a):
    return dev_u8(a) if dt == syn.E4M3 else dev_bf16(a)


@pytest.mark.parametrize("case", GEMM_CASES, ids=lambda c: c[0])
def test_grouped_gemm_swiglu_matches_oracle(case):
    name, T, H, I, E, k, ns, variant, wdt, adt = case
    fp8a = adt == syn.E4M3
    wl = syn.Workload(name, T=T, H=H, I=I, E=E, k=k, n_shared=ns, wdtype=wdt, adtype=adt, seed=21)
    s = _shape(wl, variant=variant)
    c, o, r, v = _segments(T, E, k, ns, 16, 3)
    mr = moe.max_rows(s)
    xp = syn.random_rows(1, "xp", mr, H, adt)
    w13, s13 = syn.expert_weights(wl, "w13")
    a1 = 1.0 / 64 if fp8a else 1.0
    a2 = 0.02 if fp8a else 1.0
    h = torch.zeros((mr, I * (1 if fp8a else 2)), dtype=torch.uint8, device="cuda")
    ws = moe.workspace(s)
    moe.reset_device_status(ws)
    moe.grouped_gemm_swiglu(s, _act(adt, xp), dev_w(wl, w13),
                            torch.from_numpy(s13).cuda() if wdt == syn.E4M3 else None, a1, a2,
                            torch.from_numpy(o).cuda(), h, ws)
    torch.cuda.synchronize()
    assert moe.device_status(ws) == 0
    total = o[-1]
    ref = orc.expert_swiglu(xp[:total], o, w13, wdt, s13 if wdt == syn.E4M3 else None, adt, a1)
    hv = h.cpu().numpy()[:total]
    if fp8a:
        got = orc.e4m3_decode(hv.ravel()).reshape(total, I) * a2
        refq = orc.e4m3_decode(orc.e4m3_encode(ref / a2).ravel()).reshape(total, I) * a2
        assert rel_err(got, refq, "e4m3") <= FP8_TOL
    else:
        got = bf16_to_f64(hv.view(np.uint16))
        assert rel_err(got, ref, "bf16") <= BF16_TOL


@pytest.mark.parametrize("case", GEMM_CASES, ids=lambda c: c[0])
def test_grouped_gemm_down_matches_oracle(case):
    name, T, H, I, E, k, ns, variant, wdt, adt = case
    fp8a = adt == syn.E4M3
    wl = syn.Workload(name, T=T, H=H, I=I, E=E, k=k, n_shared=ns, wdtype=wdt, adtype=adt, seed=22)
    s = _shape(wl, variant=variant)
    c, o, r, v = _segments(T, E, k, ns, 16, 4)
    mr = moe.max_rows(s)
    hin = syn.random_rows(2, "h", mr, I, adt, std=0.5)
    w2, s2 = syn.expert_weights(wl, "w2")
    a2 = 0.01 if fp8a else 1.0
    y = torch.zeros((mr, H), dtype=torch.float32, device="cuda")
    ws = moe.workspace(s)
    moe.reset_device_status(ws)
    moe.grouped_gemm_down(s, _act(adt, hin), dev_w(wl, w2),
                          torch.from_numpy(s2).cuda() if wdt == syn.E4M3 else None, a2,
                          torch.from_numpy(o).cuda(), y, ws)
    torch.cuda.synchronize()
    assert moe.device_status(ws) == 0
    total = o[-1]
    ref = orc.expert_down(hin[:total], o, w2, wdt, s2 if wdt == syn.E4M3 else None, adt, a2)
    got = y.cpu().numpy()[:total].astype(np.float64)
    assert rel_err(got, ref) <= 1e-4


def test_combine_matches_oracle():
    T, E, k, ns, H = 90, 12, 3, 1, 384
    ids = _ids(T, E, k, 9)
    c, o, r, v = orc.align(ids, E, ns, 16)
    wl = syn.Workload("c", T=T, H=H, I=128, E=E, k=k, n_shared=ns)
    s = _shape(wl)
    mr = moe.max_rows(s)
    y = syn.random_f32(3, "y", (mr, H))
    w = np.abs(syn.random_f32(4, "w", (T, k)))
    out = torch.empty((T, H), dtype=torch.bfloat16, device="cuda")
    moe.combine(s, torch.from_numpy(y).cuda(), torch.from_numpy(w).cuda(), torch.from_numpy(v).cuda(),
                torch.from_numpy(o).cuda(), out)
    ref = orc.combine(y.astype(np.float64), w.astype(np.float64), v, o, E, ns)
    got = bf16_to_f64(host_bf16_bits(out))
    assert rel_err(got, ref, "bf16") <= 1e-3


# ------------------------------------------------------------------ the fused layer
def test_fused_tiny_all_tokens_both_variants_and_determinism():
    wl = W["tiny"]
    d = syn.make_inputs(wl)
    ref = oracle_forward(wl, d)
    outs = []
    for variant in (moe.SWAP_AB, moe.NORMAL, moe.AUTO):
        L = Layer(wl, d, variant=variant)
        got = L.run()
        assert L.status() == 0
        assert rel_err(got, ref, "bf16") <= BF16_TOL, variant
        outs.append(got)
        again = L.run()
        assert np.array_equal(got, again)          # bit-identical rerun
    assert rel_err(outs[0], outs[1], "bf16") <= 2e-2       # Swap-AB == normal up to summation order


@pytest.mark.parametrize("T", [1, 8, 64])
def test_fused_mixtral_decode_sampled(T):
    wl = W["mixtral_decode"].with_T(T)
    d = syn.make_inputs(wl)
    L = Layer(wl, d)
    got = L.run()
    assert L.status() == 0
    toks = np.unique(np.linspace(0, T - 1, min(T, 6)).astype(np.int32))
    ref = oracle_forward(wl, d, tokens=toks)
    assert rel_err(got[toks], ref, "bf16") <= BF16_TOL


def test_swap_ab_page_example_shape():
    """One token (M = 1), K = 4096, N = 8192 -- the decode GEMM the AWS post
    uses to motivate Swap-AB -- as a single expert with 2I = 8192."""
    wl = syn.Workload("m1", T=1, H=4096, I=4096, E=1, k=1, seed=5)
    d = syn.make_inputs(wl)
    ref = oracle_forward(wl, d)
    for variant in (moe.SWAP_AB, moe.NORMAL):
        got = Layer(wl, d, variant=variant).run()
        assert rel_err(got, ref, "bf16") <= BF16_TOL


EDGE = [
    syn.Workload("ragged", T=37, H=256, I=384, E=8, k=2, seed=1),
    syn.Workload("one_hot", T=200, H=256, I=256, E=8, k=1, logits="zipf", zipf_s=40.0, seed=2),
    syn.Workload("sigmoid_shared", T=24, H=256, I=256, E=256, k=8, n_shared=1, gate=syn.SIGMOID,
                 routed_scale=2.5, seed=3),
    syn.Workload("wide_prefill", T=600, H=512, I=256, E=6, k=2, logits="zipf", seed=4),
    syn.Workload("big_T_swapcap", T=300, H=256, I=256, E=4, k=4, seed=5),
]


@pytest.mark.parametrize("wl", EDGE, ids=lambda w: w.name)
@pytest.mark.parametrize("pad", [16, 64])
def test_fused_edge_cases(wl, pad):
    d = syn.make_inputs(wl)
    ref = oracle_forward(wl, d)
    for variant in (moe.SWAP_AB, moe.NORMAL):
        L = Layer(wl, d, pad=pad, variant=variant)
        got = L.run()
        assert L.status() == 0
        assert rel_err(got, ref, "bf16") <= BF16_TOL, (variant, pad)


def _random_shapes(n=16, seed=7, e_choices=(1, 2, 5, 8, 16, 33, 64), tag="rand"):
    """Seeded random layer shapes across the supported space (H, I multiples
    of 128; ragged T; 1 to 64 experts, or the given counts; top-1 to top-8;
    softmax or sigmoid gate; a shared expert or none; bf16 or E4M3 weights;
    both operand orders).  The list is fixed by the seed, so a failure names
    its shape."""
    rng = np.random.default_rng(seed)
    out = []
    for i in range(n):
        E = int(rng.choice(e_choices))
        k = int(rng.integers(1, min(E, 8) + 1))
        w8 = bool(rng.random() < 0.25)
        wl = syn.Workload(f"{tag}{i}", T=int(rng.integers(1, 700)), H=int(rng.choice([128, 256, 384, 640])),
                          I=int(rng.choice([128, 256, 512, 896])), E=E, k=k,
                          n_shared=int(rng.random() < 0.3),
                          gate=syn.SIGMOID if rng.random() < 0.3 else syn.SOFTMAX,
                          routed_scale=float(rng.choice([1.0, 2.5])),
                          wdtype=syn.E4M3 if w8 else syn.BF16, seed=100 + i)
        variant = moe.SWAP_AB if w8 else [moe.AUTO, moe.SWAP_AB, moe.NORMAL][int(rng.integers(0, 3))]
        pad = int(rng.choice([16, 32, 64]))
        out.append((wl, variant, pad))
    return out


@pytest.mark.parametrize("wl,variant,pad",
                         _random_shapes() + _random_shapes(12, seed=11, e_choices=(3, 24, 128, 256, 512), tag="randE"),
                         ids=lambda v: getattr(v, "name", str(v)))
def test_fused_random_shapes(wl, variant, pad):
    d = syn.make_inputs(wl)
    ref = oracle_forward(wl, d)
    L = Layer(wl, d, pad=pad, variant=variant)
    got = L.run()
    assert L.status() == 0
    assert rel_err(got, ref, "bf16") <= BF16_TOL, (wl, variant, pad)


def _fp8_small(T=300):
    wl = syn.Workload("fp8_small", T=T, H=512, I=512, E=8, k=2, wdtype=syn.E4M3, adtype=syn.E4M3, seed=7)
    d = syn.make_inputs(wl)
    xq = orc.quant_e4m3_f32(syn.bf16_bits_to_f32(d["x"]), d["a1"])
    a2 = float(np.float32(orc.hidden_amax(d["x"], d["logits"], d["w13"], E=8, k=2, wdtype=syn.E4M3,
                                          adtype=syn.E4M3, w13_scale=d["w13_scale"], a1=d["a1"]) / 448))
    del xq
    return wl, d, a2


@pytest.mark.parametrize("variant", [moe.SWAP_AB, moe.NORMAL])
def test_fused_fp8_weights_and_activations(variant):
    wl, d, a2 = _fp8_small()
    ref = oracle_forward(wl, d, a2=a2)
    L = Layer(wl, d, variant=variant, a2=a2)
    got = L.run()
    assert L.status() == 0
    assert rel_err(got, ref, "bf16") <= FP8_TOL


@pytest.mark.parametrize("T", [1, 8, 32, 128])
def test_fused_fp8_weights_bf16_activations_sigmoid_shared(T):
    """DeepSeek-V3-shaped routing (E=256, top-8 sigmoid x2.5, one shared
    expert, E4M3 weights, bf16 activations) at reduced H and I."""
    wl = syn.Workload("dsv3_small", T=T, H=1024, I=256, E=256, k=8, n_shared=1, gate=syn.SIGMOID,
                      routed_scale=2.5, wdtype=syn.E4M3, seed=8)
    d = syn.make_inputs(wl)
    ref = oracle_forward(wl, d)
    L = Layer(wl, d)
    got = L.run()
    assert L.status() == 0
    assert rel_err(got, ref, "bf16") <= FP8_TOL
    assert np.array_equal(got, L.run())


@pytest.mark.parametrize("mode", ["swiglu", "down"])
def test_e4m3_weight_expansion_is_exact(mode):
    """E4M3 weights drawn from every finite code (subnormals included), scale
    1: the E4M3-weight GEMM (bf16 activations split into hi/lo E4M3 planes)
    must equal the bf16-weight GEMM on the identical values up to fp32
    summation order and the split's sub-2^-11 remainders, which checks that
    every weight code and the activation split are taken exactly."""
    T, H, I, E, k = 32, 512, 256, 4, 2
    rng = np.random.default_rng(12)
    codes = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], dtype=np.uint8)
    rows_w = 2 * I if mode == "swiglu" else H
    cols_w = H if mode == "swiglu" else I
    q = rng.choice(codes, size=(E, rows_w, cols_w)).astype(np.uint8)
    wbits = orc.bf16_encode(orc.e4m3_decode(q.ravel())).reshape(q.shape)
    ones = torch.ones(E, dtype=torch.float32, device="cuda")
    c, o, r, v = _segments(T, E, k, 0, 16, 5)
    wl8 = syn.Workload("w8", T=T, H=H, I=I, E=E, k=k, wdtype=syn.E4M3)
    wl16 = syn.Workload("w16", T=T, H=H, I=I, E=E, k=k)
    s8, s16 = _shape(wl8), _shape(wl16, variant=moe.SWAP_AB)
    mr = moe.max_rows(s16)
    offs = torch.from_numpy(o).cuda()
    cols_a = H if mode == "swiglu" else I
    act = dev_bf16(syn.random_rows(6, "a", mr, cols_a, syn.BF16, std=0.05))
    outs = []
    for s, w, sc in ((s8, dev_u8(q), ones), (s16, dev_bf16(wbits), None)):
        ws = moe.workspace(s)
        moe.reset_device_status(ws)
        if mode == "swiglu":
            out = torch.zeros((mr, I), dtype=torch.bfloat16, device="cuda")
            moe.grouped_gemm_swiglu(s, act, w, sc, 1.0, 1.0, offs, out, ws)
        else:
            out = torch.zeros((mr, H), dtype=torch.float32, device="cuda")
            moe.grouped_gemm_down(s, act, w, sc, 1.0, offs, out, ws)
        torch.cuda.synchronize()
        assert moe.device_status(ws) == 0
        outs.append(out.float().cpu().numpy()[:o[-1]].astype(np.float64))
    if mode == "swiglu":
        assert rel_err(outs[0], outs[1], "bf16") <= 1e-3
    else:
        assert rel_err(outs[0], outs[1]) <= 1e-5


# ------------------------------------------------------------------ router (step 0+1)
ROUTER_CASES = [W["tiny"], W["mixtral_decode"],
                dataclasses.replace(W["dsv3_decode_fp8w"], wdtype=syn.BF16),
                syn.Workload("router_odd", T=77, H=136, I=128, E=45, k=3, seed=12)]


@pytest.mark.parametrize("wl", ROUTER_CASES, ids=lambda w: w.name)
def test_router_topk_bit_exact(wl):
    """Router logits bit for bit against the oracle's fixed-order sum, then
    ids bit-exact and weights within 2e-6 of the oracle's routing of those
    logits."""
    x = syn.tokens(wl)
    wg = syn.router_weight(wl)
    ref_l = orc.router_logits(x, wg)
    ref_ids, ref_w = orc.route(ref_l, k=wl.k, gate=wl.gate, renorm=wl.renorm, routed_scale=wl.routed_scale)
    s = _shape(wl)
    ws = moe.workspace(s)
    lg = torch.full((wl.T, wl.E), float("nan"), dtype=torch.float32, device="cuda")
    ids = torch.empty((wl.T, wl.k), dtype=torch.int32, device="cuda")
    w = torch.empty((wl.T, wl.k), dtype=torch.float32, device="cuda")
    for _ in range(2):                                # a rerun reuses the workspace tickets
        moe.router_topk(s, dev_bf16(x), dev_bf16(wg), lg, ids, w, ws)
        torch.cuda.synchronize()
        assert np.array_equal(lg.cpu().numpy().view(np.uint32), ref_l.view(np.uint32))
        assert np.array_equal(ids.cpu().numpy(), ref_ids)
        assert np.allclose(w.cpu().numpy(), ref_w, rtol=2e-6, atol=1e-7)


@pytest.mark.parametrize("wl", [W["tiny"], W["mixtral_decode"].with_T(8),
                                W["dsv3_decode_fp8w"].with_T(8)], ids=lambda w: f"{w.name}_T{w.T}")
def test_fused_forward_router_equals_logits_path(wl):
    """The layer started from the router weight equals, bit for bit, the layer
    given the oracle's router logits, and matches the oracle's layer."""
    d = syn.make_inputs(wl)
    wg = syn.router_weight(wl)
    d["logits"] = orc.router_logits(d["x"], wg)
    L = Layer(wl, d)
    via_logits = L.run()
    moe.reset_device_status(L.ws)
    out = torch.empty_like(L.out)
    moe.fused_forward_router(L.shape, L.x, dev_bf16(wg), L.w13, L.s13, L.w2, L.s2, L.a1, L.a2, out, L.ws)
    torch.cuda.synchronize()
    assert L.status() == 0
    via_router = bf16_to_f64(host_bf16_bits(out))
    assert np.array_equal(via_router, via_logits)
    toks = np.unique(np.linspace(0, wl.T - 1, min(wl.T, 6)).astype(np.int32))
    ref = oracle_forward(wl, d, tokens=toks)
    assert rel_err(via_router[toks], ref, "bf16") <= BF16_TOL


# ------------------------------------------------------------------ failure path
def test_bounded_wait_times_out_and_context_stays_usable():
    """A pipeline wait on a barrier that nothing arrives on gives up after the
    wait limit, the abort flag stops the block's other wait, the status word
    reads MOE_ERR_TIMEOUT, and the next layer call on the same context runs
    correctly."""
    import time
    wl = W["tiny"]
    d = syn.make_inputs(wl)
    L = Layer(wl, d)
    moe.reset_device_status(L.ws)
    gave_up = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    t0 = time.perf_counter()
    moe.selftest_wait_timeout(L.ws, gave_up)
    torch.cuda.synchronize()
    dt = time.perf_counter() - t0
    assert moe.device_status(L.ws) == -6
    assert int(gave_up.item()) == 2
    assert 1.5 < dt < 30.0
    got = L.run()                      # resets the status, runs the layer
    assert L.status() == 0
    assert rel_err(got, oracle_forward(wl, d), "bf16") <= BF16_TOL


def test_cta_pair_abort_times_out_and_context_stays_usable():
    """In every CTA pair of a prefill down projection the second CTA stops
    loading its operand halves after two stages.  The first CTA's waits run
    out after the wait limit, both CTAs take the pair's abort tear-down (no
    copy left in flight, tensor memory freed), the status word reads
    MOE_ERR_TIMEOUT, the call ends within seconds, and the next layer call on
    the same context is correct."""
    import time
    wl = W["tiny"].with_T(2048)            # 4096 routed rows over 8 experts: all on CTA pairs
    d = syn.make_inputs(wl)
    L = Layer(wl, d)
    s = L.shape
    E_t = wl.E + wl.n_shared
    mr = moe.max_rows(s)
    ids = torch.empty((wl.T, wl.k), dtype=torch.int32, device="cuda")
    w = torch.empty((wl.T, wl.k), dtype=torch.float32, device="cuda")
    counts = torch.empty(E_t, dtype=torch.int32, device="cuda")
    offsets = torch.empty(E_t + 1, dtype=torch.int32, device="cuda")
    rows = torch.empty(mr, dtype=torch.int32, device="cuda")
    inv = torch.empty(wl.T * wl.k, dtype=torch.int32, device="cuda")
    h = torch.zeros((mr, wl.I), dtype=torch.bfloat16, device="cuda")
    y = torch.empty((mr, wl.H), dtype=torch.float32, device="cuda")
    ws = moe.workspace(s)
    moe.reset_device_status(ws)
    moe.route_topk(s, L.logits, ids, w)
    moe.align_permute(s, ids, counts, offsets, rows, inv, ws)
    torch.cuda.synchronize()
    assert int(counts.min()) >= 256                       # every expert's segment goes to the pairs
    t0 = time.perf_counter()
    moe.selftest_pair_abort(s, h, L.w2, offsets, y, ws)
    torch.cuda.synchronize()
    dt = time.perf_counter() - t0
    assert moe.device_status(ws) == -6                     # MOE_ERR_TIMEOUT
    assert 1.5 < dt < 30.0
    got = L.run()                                          # resets the status, runs the layer
    assert L.status() == 0
    assert rel_err(got, oracle_forward(wl, d), "bf16") <= BF16_TOL


# ------------------------------------------------------------------ fused layer against the separate steps
# The fused layer routes and aligns in one kernel at decode sizes, skips pad
# slots, and combines inside GEMM2's epilogue on the Swap-AB path.  The
# arithmetic and its order are those of the separate steps, so the fused
# output must equal, bit for bit, the output of the step-by-step calls on the
# same inputs.
STEPWISE = [
    (W["tiny"], moe.SWAP_AB), (W["tiny"], moe.NORMAL),
    (EDGE[0], moe.SWAP_AB), (EDGE[0], moe.NORMAL),                  # ragged T=37
    (EDGE[2], moe.AUTO),                                              # E=256 top-8 sigmoid + shared
    (EDGE[3], moe.NORMAL),                                            # T=600 prefill, CTA-pair GEMM2
    (EDGE[4], moe.SWAP_AB), (EDGE[4], moe.NORMAL),                   # T=300: several row tiles
    (syn.Workload("fp8_small", T=300, H=512, I=512, E=8, k=2, wdtype=syn.E4M3, adtype=syn.E4M3, seed=7),
     moe.SWAP_AB),
    (syn.Workload("fp8_small", T=300, H=512, I=512, E=8, k=2, wdtype=syn.E4M3, adtype=syn.E4M3, seed=7),
     moe.NORMAL),
    (syn.Workload("dsv3_small", T=8, H=1024, I=256, E=256, k=8, n_shared=1, gate=syn.SIGMOID,
                  routed_scale=2.5, wdtype=syn.E4M3, seed=8), moe.AUTO),
    (syn.Workload("dsv3_small", T=128, H=1024, I=256, E=256, k=8, n_shared=1, gate=syn.SIGMOID,
                  routed_scale=2.5, wdtype=syn.E4M3, seed=8), moe.AUTO),
]


def _stepwise(L, a2):
    """The layer as separate entry-point calls (the unfused reference)."""
    wl, s = L.wl, L.shape
    E_t = wl.E + wl.n_shared
    mr = moe.max_rows(s)
    fp8a = wl.adtype == syn.E4M3
    ids = torch.empty((wl.T, wl.k), dtype=torch.int32, device="cuda")
    w = torch.empty((wl.T, wl.k), dtype=torch.float32, device="cuda")
    counts = torch.empty(E_t, dtype=torch.int32, device="cuda")
    offsets = torch.empty(E_t + 1, dtype=torch.int32, device="cuda")
    rows = torch.empty(mr, dtype=torch.int32, device="cuda")
    inv = torch.empty(wl.T * wl.k, dtype=torch.int32, device="cuda")
    xp = torch.empty((mr, wl.H * (1 if fp8a else 2)), dtype=torch.uint8, device="cuda")
    h = torch.empty((mr, wl.I * (1 if fp8a else 2)), dtype=torch.uint8, device="cuda")
    y = torch.empty((mr, wl.H), dtype=torch.float32, device="cuda")
    out = torch.empty((wl.T, wl.H), dtype=torch.bfloat16, device="cuda")
    ws = moe.workspace(s)
    moe.reset_device_status(ws)
    moe.route_topk(s, L.logits, ids, w)
    moe.align_permute(s, ids, counts, offsets, rows, inv, ws)
    moe.gather(s, L.x, rows, offsets, L.a1, xp)
    moe.grouped_gemm_swiglu(s, xp, L.w13, L.s13, L.a1, a2, offsets, h, ws)
    moe.grouped_gemm_down(s, h, L.w2, L.s2, a2, offsets, y, ws)
    moe.combine(s, y, w, inv, offsets, out)
    torch.cuda.synchronize()
    assert moe.device_status(ws) == 0
    return out


@pytest.mark.parametrize("wl,variant", STEPWISE, ids=lambda v: getattr(v, "name", str(v)))
def test_fused_gather_and_combine_equal_the_separate_steps_bit_for_bit(wl, variant):
    d = syn.make_inputs(wl)
    a2 = 1.0
    if wl.adtype == syn.E4M3:
        a2 = float(np.float32(orc.hidden_amax(d["x"], d["logits"], d["w13"], E=wl.E, k=wl.k, wdtype=syn.E4M3,
                                              adtype=syn.E4M3, w13_scale=d["w13_scale"], a1=d["a1"],
                                              tokens=np.arange(16, dtype=np.int32)) / 448))
    L = Layer(wl, d, variant=variant, a2=a2)
    L.run()
    assert L.status() == 0
    fused = L.out.clone()
    ref = _stepwise(L, a2)
    assert torch.equal(fused.view(torch.int16), ref.view(torch.int16))
    L.run()                                                     # and again: deterministic
    assert torch.equal(L.out.view(torch.int16), fused.view(torch.int16))
