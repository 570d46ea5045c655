"""Pins for the CPU oracle: each test checks the oracle against something other
than itself -- a format definition, a library routine the case reduces to, a
closed form, an invariant, or brute force on tiny inputs.  CPU only."""
import dataclasses
import itertools

import numpy as np
import pytest
import torch
from scipy.special import expit

import oracle as orc
from mixture_experts_layer_22_b200 import synthetic as syn


# ------------------------------------------------------------------ E4M3
def _torch_e4m3_decode(codes):
    return torch.tensor(codes, dtype=torch.uint8).view(torch.float8_e4m3fn).to(torch.float64).numpy()


def test_e4m3_decode_all_codes_match_library():
    codes = np.arange(256, dtype=np.uint8)
    ours = orc.e4m3_decode(codes)
    ref = _torch_e4m3_decode(codes)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(ours), nan)
    assert nan.sum() == 2 and nan[0x7F] and nan[0xFF]
    assert np.array_equal(ours[~nan], ref[~nan])


def test_e4m3_format_landmarks():
    # largest finite, smallest normal, smallest subnormal of the 1-4-3 format
    assert orc.e4m3_decode([0x7E])[0] == 448.0
    assert orc.e4m3_decode([0x08])[0] == 2.0 ** -6
    assert orc.e4m3_decode([0x01])[0] == 2.0 ** -9
    assert orc.e4m3_decode([0x38])[0] == 1.0
    assert orc.e4m3_decode([0xB8])[0] == -1.0


def test_e4m3_encode_roundtrip_every_finite_code():
    codes = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], dtype=np.uint8)
    back = orc.e4m3_encode(orc.e4m3_decode(codes))
    assert np.array_equal(back, codes)


def test_e4m3_encode_midpoints_ties_to_even():
    for c in range(0, 0x7E):
        lo, hi = orc.e4m3_decode([c, c + 1])
        mid = (lo + hi) / 2
        even = c if (c & 1) == 0 else c + 1
        assert orc.e4m3_encode([mid])[0] == even, hex(c)
        assert orc.e4m3_encode([np.nextafter(mid, 0)])[0] == c
        assert orc.e4m3_encode([np.nextafter(mid, 1e9)])[0] == c + 1
        assert orc.e4m3_encode([-mid])[0] == (even | 0x80)


def test_e4m3_encode_saturates():
    assert orc.e4m3_encode([449.0, 464.0, 480.0, 1e30])[:].tolist() == [0x7E] * 4
    assert orc.e4m3_encode([-1e30])[0] == 0xFE
    assert orc.e4m3_encode([2.0 ** -11])[0] == 0x00          # below half the smallest subnormal
    assert orc.e4m3_encode([-(2.0 ** -10)])[0] == 0x80       # exact tie with 0 -> even (zero)


def test_e4m3_encode_matches_library_cast():
    rng = np.random.default_rng(1)
    v = np.concatenate([rng.standard_normal(20000) * 40, rng.standard_normal(5000) * 0.01,
                        rng.uniform(-448, 448, 5000)]).astype(np.float32)
    ours = orc.e4m3_encode(v.astype(np.float64))
    ref = torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(ours, ref)


def test_quant_e4m3_fp32_quotient_matches_library():
    rng = np.random.default_rng(2)
    v = (rng.standard_normal(50000) * 3).astype(np.float32)
    scale = np.float32(np.abs(v).max() / 448.0)
    ours = orc.quant_e4m3_f32(v, float(scale))
    q = (torch.from_numpy(v) / torch.tensor(scale)).clamp(-448, 448)
    ref = q.to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(ours, ref)


# ------------------------------------------------------------------ bf16
def test_bf16_encode_matches_library_cast():
    rng = np.random.default_rng(3)
    v = np.concatenate([rng.standard_normal(30000), rng.standard_normal(3000) * 1e-38,
                        rng.standard_normal(3000) * 1e30]).astype(np.float32)
    ours = orc.bf16_encode(v.astype(np.float64))
    ref = torch.from_numpy(v).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)
    assert np.array_equal(orc.bf16_decode(ours), torch.from_numpy(v).to(torch.bfloat16).double().numpy())


# ------------------------------------------------------------------ routing
def _brute_topk(l, k):
    """The unique k-subset whose every member ranks above every non-member,
    ranking by (logit, then lower id)."""
    E = len(l)
    key = lambda e: (l[e], -e)
    found = []
    for S in itertools.combinations(range(E), k):
        rest = [e for e in range(E) if e not in S]
        if all(key(a) > key(b) for a in S for b in rest):
            found.append(S)
    assert len(found) == 1
    return sorted(found[0], key=key, reverse=True)


@pytest.mark.parametrize("E", [2, 3, 5, 8])
def test_route_matches_brute_force_with_ties(E):
    rng = np.random.default_rng(E)
    T = 200
    logits = rng.integers(-2, 3, size=(T, E)).astype(np.float32)   # many exact ties
    logits[0] = 1.0                                                   # all equal
    for k in range(1, E + 1):
        ids, w = orc.route(logits, k)
        for t in range(T):
            assert list(ids[t]) == _brute_topk(list(logits[t]), k)
        assert np.allclose(w.sum(1), 1.0, rtol=0, atol=1e-12)
    ids, w = orc.route(logits[:1], min(2, E))
    assert np.allclose(w, 1.0 / min(2, E))


def test_route_two_way_softmax_is_logistic():
    rng = np.random.default_rng(5)
    logits = rng.standard_normal((500, 8)).astype(np.float32) * 3
    ids, w = orc.route(logits, 2)
    l0 = logits[np.arange(500), ids[:, 0]].astype(np.float64)
    l1 = logits[np.arange(500), ids[:, 1]].astype(np.float64)
    assert np.allclose(w[:, 0], expit(l0 - l1), rtol=1e-13, atol=1e-15)


def test_route_softmax_without_renorm_is_full_softmax_entry():
    rng = np.random.default_rng(6)
    logits = rng.standard_normal((50, 6)).astype(np.float32)
    ids, w = orc.route(logits, 6, renorm=False)            # k = E: nothing dropped
    ids2, w2 = orc.route(logits, 6, renorm=True)
    assert np.array_equal(ids, ids2) and np.allclose(w, w2, atol=1e-14)
    ids, w = orc.route(logits, 2, renorm=False)
    assert np.all(w.sum(1) < 1.0)


def test_route_sigmoid_scaled():
    rng = np.random.default_rng(7)
    logits = rng.standard_normal((300, 16)).astype(np.float32) * 2
    ids, w = orc.route(logits, 4, gate=orc.SIGMOID, renorm=True, routed_scale=2.5)
    assert np.allclose(w.sum(1), 2.5, atol=1e-12)
    ids2, w2 = orc.route(logits, 4, gate=orc.SIGMOID, renorm=False, routed_scale=2.5)
    sel = np.take_along_axis(logits, ids2, 1).astype(np.float64)
    assert np.array_equal(ids, ids2)
    assert np.allclose(w2, 2.5 * expit(sel), rtol=1e-13)


def test_route_nan_ranks_last():
    l = np.array([[np.nan, -np.inf, 0.0, np.nan]], dtype=np.float32)
    ids, _ = orc.route(l, 4)
    assert ids[0].tolist() == [2, 1, 0, 3]


# ------------------------------------------------------------------ align
@pytest.mark.parametrize("T,E,k,n_shared,pad", [(16, 8, 2, 0, 16), (100, 60, 4, 0, 16),
                                                (37, 8, 2, 0, 1), (33, 256, 8, 1, 16),
                                                (64, 5, 3, 0, 128), (1, 8, 2, 0, 16)])
def test_align_counting_sort(T, E, k, n_shared, pad):
    rng = np.random.default_rng(T * E)
    ids = np.stack([rng.permutation(E)[:k] for _ in range(T)]).astype(np.int32)
    counts, offsets, rows, inv = orc.align(ids, E, n_shared, pad)
    R = T * k
    flat = ids.ravel()
    assert counts[:E].tolist() == np.bincount(flat, minlength=E).tolist()
    assert counts.sum() == R + n_shared * T
    seg = np.diff(offsets)
    assert np.all(seg % pad == 0) and np.all(seg == -(-counts // pad) * pad)
    # the library's stable sort gives the same order within each expert
    order = np.argsort(flat, kind="stable")
    got = np.concatenate([rows[offsets[e]:offsets[e] + counts[e]] for e in range(E)])
    assert np.array_equal(got, order)
    for e in range(E + n_shared):
        assert np.all(rows[offsets[e] + counts[e]:offsets[e + 1]] == -1)
    for s in range(n_shared):
        assert np.array_equal(rows[offsets[E + s]:offsets[E + s] + T], R + s * T + np.arange(T))
    assert np.array_equal(rows[inv], np.arange(R))                   # bijection onto routed slots
    assert len(set(inv.tolist())) == R


def test_align_empty_experts_and_one_hot_expert():
    ids = np.full((40, 1), 3, dtype=np.int32)
    counts, offsets, rows, inv = orc.align(ids, 8, 0, 16)
    assert counts.tolist() == [0, 0, 0, 40, 0, 0, 0, 0]
    assert offsets.tolist() == [0, 0, 0, 0, 48, 48, 48, 48, 48]
    assert np.array_equal(inv, np.arange(40))


# ------------------------------------------------------------------ expert math
def _bf16_round(v):
    """Round to bf16, nearest even (the library's cast), back to double."""
    return torch.from_numpy(np.asarray(v, dtype=np.float64)).to(torch.bfloat16).double().numpy()


def _dense_swiglu(xd, W1, W3, W2, round_h=True):
    """The textbook dense SwiGLU MLP; the hidden vector, an activation of a
    bf16 layer, is stored in bf16 (round_h) before the down projection."""
    g = xd @ W1.T
    u = xd @ W3.T
    h = g * expit(g) * u
    return (_bf16_round(h) if round_h else h) @ W2.T


def test_single_expert_top1_is_dense_swiglu_mlp():
    wl = syn.Workload("t", T=9, H=64, I=96, E=1, k=1, seed=3)
    d = syn.make_inputs(wl)
    out = orc.forward(d["x"], d["logits"], d["w13"], d["w2"], E=1, k=1)
    xd = orc.bf16_decode(d["x"])
    w13 = orc.bf16_decode(d["w13"][0])
    ref = _dense_swiglu(xd, w13[:96], w13[96:], orc.bf16_decode(d["w2"][0]))
    assert np.allclose(out, ref, rtol=1e-12, atol=1e-12)


def test_identical_experts_give_mlp_times_weight_sum():
    wl = syn.Workload("t", T=12, H=32, I=48, E=6, k=3, seed=4)
    d = syn.make_inputs(wl)
    w13 = np.repeat(d["w13"][:1], 6, axis=0)
    w2 = np.repeat(d["w2"][:1], 6, axis=0)
    out = orc.forward(d["x"], d["logits"], w13, w2, E=6, k=3)
    xd = orc.bf16_decode(d["x"])
    W = orc.bf16_decode(w13[0])
    mlp = _dense_swiglu(xd, W[:48], W[48:], orc.bf16_decode(w2[0]))
    assert np.allclose(out, mlp, rtol=1e-11, atol=1e-12)
    # sigmoid gate renormalised to 2.5 plus one shared expert: 3.5 * MLP
    w13s = np.repeat(d["w13"][:1], 7, axis=0)
    w2s = np.repeat(d["w2"][:1], 7, axis=0)
    out = orc.forward(d["x"], d["logits"], w13s, w2s, E=6, k=3, n_shared=1, gate=orc.SIGMOID,
                      routed_scale=2.5)
    assert np.allclose(out, 3.5 * mlp, rtol=1e-11, atol=1e-12)


def test_scalar_layer_closed_form():
    # H = I = 1: out = c * SiLU(a x) * (b x) with a, b, c exactly representable
    a, b, c = 0.5, -1.25, 3.0
    bits = orc.bf16_encode
    w13 = np.array([[[bits([a])[0]], [bits([b])[0]]]], dtype=np.uint16)
    w2 = np.array([[[bits([c])[0]]]], dtype=np.uint16)
    xs = np.array([-3.0, -0.5, 0.0, 0.75, 2.0, 6.0])
    x = bits(xs).reshape(-1, 1)
    out = orc.forward(x, np.zeros((6, 1), np.float32), w13, w2, E=1, k=1)[:, 0]
    ref = c * _bf16_round((a * xs) * expit(a * xs) * (b * xs))
    assert np.allclose(out, ref, rtol=1e-14, atol=1e-15)


def test_row_wise_pieces_compose_to_dense_definition():
    wl = syn.Workload("t", T=20, H=48, I=40, E=5, k=2, n_shared=1, gate=orc.SIGMOID,
                      routed_scale=2.5, seed=5)
    d = syn.make_inputs(wl)
    ids, w = orc.route(d["logits"], 2, gate=orc.SIGMOID, routed_scale=2.5)
    counts, offsets, rows, inv = orc.align(ids, 5, 1, 8)
    xp = orc.gather(d["x"], rows, 2, 20, 1)
    h = orc.expert_swiglu(xp, offsets, d["w13"], orc.BF16)
    # h is stored as bf16 between the two steps, as in the layer
    y = orc.expert_down(orc.bf16_encode(h), offsets, d["w2"], orc.BF16)
    out = orc.combine(y, w, inv, offsets, 5, 1)
    ref = orc.forward(d["x"], d["logits"], d["w13"], d["w2"], E=5, k=2, n_shared=1,
                      gate=orc.SIGMOID, routed_scale=2.5)
    assert np.allclose(out, ref, rtol=1e-11, atol=1e-13)


def _down_double(h, offsets, w2):
    y = np.zeros((h.shape[0], w2.shape[1]))
    for e in range(len(offsets) - 1):
        s0, s1 = offsets[e], offsets[e + 1]
        y[s0:s1] = h[s0:s1] @ orc.bf16_decode(w2[e]).T
    return y


def test_expert_down_matches_library_matmul():
    rng = np.random.default_rng(8)
    offsets = np.array([0, 16, 16, 48], np.int32)
    hbits = syn.to_bf16_bits(rng.standard_normal((48, 40)).astype(np.float32))
    w2 = syn.to_bf16_bits(rng.standard_normal((3, 24, 40)).astype(np.float32))
    y = orc.expert_down(hbits, offsets, w2, orc.BF16)
    assert np.allclose(y, _down_double(orc.bf16_decode(hbits), offsets, w2), rtol=1e-12, atol=1e-12)


# ------------------------------------------------------------------ FP8 plumbing
def test_fp8_weights_with_power_of_two_scale_equal_bf16_weights():
    """E4M3 values times 2^-j are exactly bf16 values, so the FP8-weight layer
    must equal the bf16 layer on those values exactly."""
    wl = syn.Workload("t", T=10, H=32, I=24, E=4, k=2, seed=6)
    d = syn.make_inputs(wl)
    rng = np.random.default_rng(9)
    c13 = rng.integers(0, 0x7E, size=(4, 48, 32)).astype(np.uint8) | (rng.integers(0, 2, (4, 48, 32)) << 7).astype(np.uint8)
    c2 = rng.integers(0, 0x7E, size=(4, 32, 24)).astype(np.uint8)
    s13 = np.full(4, 2.0 ** -8, np.float32)
    s2 = np.full(4, 2.0 ** -6, np.float32)
    b13 = orc.bf16_encode(orc.e4m3_decode(c13) * 2.0 ** -8)
    b2 = orc.bf16_encode(orc.e4m3_decode(c2) * 2.0 ** -6)
    out8 = orc.forward(d["x"], d["logits"], c13, c2, E=4, k=2, wdtype=orc.E4M3, w13_scale=s13, w2_scale=s2)
    out16 = orc.forward(d["x"], d["logits"], b13, b2, E=4, k=2)
    assert np.array_equal(out8, out16)


def test_fp8_activation_quantisation_path():
    wl = syn.Workload("t", T=10, H=32, I=24, E=4, k=2, seed=7)
    d = syn.make_inputs(wl)
    a1 = 2.0 ** -6                      # power of two: x_q * a1 is exactly bf16
    xq = orc.quant_e4m3_f32(syn.bf16_bits_to_f32(d["x"]), a1)
    xdeq = orc.bf16_encode(orc.e4m3_decode(xq) * a1)
    out_q = orc.forward(d["x"], d["logits"], d["w13"], d["w2"], E=4, k=2, adtype=orc.E4M3, a1=a1,
                        a2=2.0 ** 30)
    assert np.all(out_q == 0.0)        # every hidden value quantises to zero
    # with a2 calibrated to amax(h)/448 the layer differs from the bf16 layer on
    # the dequantised tokens only through the rounding of h to E4M3
    out_ref = orc.forward(xdeq, d["logits"], d["w13"], d["w2"], E=4, k=2)
    a2 = float(np.float32(orc.hidden_amax(xdeq, d["logits"], d["w13"], E=4, k=2) / 448))
    out_q = orc.forward(d["x"], d["logits"], d["w13"], d["w2"], E=4, k=2, adtype=orc.E4M3, a1=a1, a2=a2)
    err = np.abs(out_q - out_ref).max() / np.sqrt(np.mean(out_ref ** 2))
    assert 0 < err < 0.2


# ------------------------------------------------------------------ router logits
def _bf16(values) -> np.ndarray:
    return syn.to_bf16_bits(np.asarray(values, dtype=np.float32))


def test_router_logits_one_hot_picks_the_gate_column():
    """x_t = unit vector at h_t: l[t,e] = Wg[e, h_t] exactly, for positions in
    every lane and chunk of the fixed order (catches a dropped term, a wrong
    index or a transposed operand)."""
    T, E, H = 40, 5, 512
    rng = np.random.default_rng(21)
    wg = _bf16(rng.standard_normal((E, H)) * 0.02)
    hs = rng.choice(H, size=T, replace=False)
    x = np.zeros((T, H), dtype=np.float32)
    x[np.arange(T), hs] = 1.0
    lg = orc.router_logits(_bf16(x), wg)
    assert np.array_equal(lg, syn.bf16_bits_to_f32(wg)[:, hs].T)


def test_router_logits_within_rounding_of_the_exact_sum():
    """Against the exact rational sum: off by at most the double summation
    error plus half an fp32 ulp."""
    from fractions import Fraction
    T, E, H = 3, 4, 264
    rng = np.random.default_rng(22)
    x = _bf16(rng.standard_normal((T, H)))
    wg = _bf16(rng.standard_normal((E, H)) * 0.02)
    lg = orc.router_logits(x, wg)
    xf, wf = syn.bf16_bits_to_f32(x).astype(np.float64), syn.bf16_bits_to_f32(wg).astype(np.float64)
    for t in range(T):
        for e in range(E):
            exact = sum((Fraction(float(a)) * Fraction(float(b)) for a, b in zip(xf[t], wf[e])), Fraction(0))
            mag = float(np.sum(np.abs(xf[t] * wf[e])))
            err = abs(Fraction(float(lg[t, e])) - exact)
            ulp = float(np.spacing(np.float32(max(abs(float(exact)), abs(float(lg[t, e]))))))
            assert err <= Fraction(0.5 * ulp) + Fraction((H + 8) * 2.0 ** -53 * mag)


@pytest.mark.parametrize("hs,expect", [
    ((0, 256, 512), 0.0),     # one lane, ascending h: 2^60 + 1 loses the 1
    ((0, 8, 16), 1.0),        # lanes 0, 1, 2: (s0 + s2) + (s1 + s3) keeps it
    ((0, 8, 128), 1.0),       # lanes 0, 1, 16: (s0 + s16) + s1 keeps it
])
def test_router_logits_follow_the_fixed_order(hs, expect):
    """Products 2^60, 1, -2^60 at chosen positions: the result depends on the
    association, which pins the lane assignment and the xor tree."""
    H = 640
    x = np.zeros((1, H), dtype=np.float32)
    w = np.zeros((1, H), dtype=np.float32)
    x[0, hs[0]], w[0, hs[0]] = 2.0 ** 30, 2.0 ** 30
    x[0, hs[1]], w[0, hs[1]] = 1.0, 1.0
    x[0, hs[2]], w[0, hs[2]] = -(2.0 ** 30), 2.0 ** 30
    assert orc.router_logits(_bf16(x), _bf16(w))[0, 0] == np.float32(expect)


def test_router_logits_feed_routing_like_given_logits():
    """The synthetic router-logit recipe and the oracle's router agree to fp32
    rounding on the seeded Mixtral-shaped tokens, and route identically."""
    wl = syn.WORKLOADS["mixtral_decode"].with_T(16)
    x = syn.tokens(wl)
    lg = orc.router_logits(x, syn.router_weight(wl))
    ref = syn.router_logits(wl, x)
    assert np.allclose(lg, ref, rtol=1e-6, atol=1e-7)
    assert np.array_equal(orc.route(lg, k=2)[0], orc.route(ref, k=2)[0])


# ------------------------------------------------------------------ hi/lo split (E4M3 weights, bf16 activations)
def _split_scale(amax: float) -> float:
    """Smallest power of two s with amax <= 448 s."""
    if amax == 0.0:
        return 1.0
    s = 2.0 ** np.ceil(np.log2(amax / 448.0))
    while amax > 448.0 * s:          # guard the log2 rounding at exact powers
        s *= 2.0
    while amax <= 224.0 * s:
        s /= 2.0
    return s


def test_hilo_split_of_bf16_rows_is_exact_but_for_tiny_remainders():
    """The reading behind the E4M3-weight path: a bf16 row v with the power-of-
    two scale s splits as hi = e4m3(v/s), lo = e4m3(v/s - hi) with
    s (hi + lo) == v wherever the remainder is at least 2^-6, and within
    2^-10 s elsewhere (<= 2^-10 s / (224 s) of the row max), across 9 decades."""
    rng = np.random.default_rng(23)
    worst = 0.0
    for _ in range(200):
        v = orc.bf16_decode(syn.to_bf16_bits((rng.standard_normal(384) * 10.0 ** rng.uniform(-6, 3)).astype(np.float32)))
        amax = float(np.abs(v).max())
        s = _split_scale(amax)
        assert amax <= 448.0 * s and (amax > 224.0 * s or s == 1.0)
        q = v / s
        hi = orc.e4m3_decode(orc.e4m3_encode(q))
        rem = q - hi
        lo = orc.e4m3_decode(orc.e4m3_encode(rem))
        err = np.abs(s * (hi + lo) - v)
        assert np.all(err[np.abs(rem) >= 2.0 ** -6] == 0.0)
        assert np.all(err <= 2.0 ** -10 * s)
        worst = max(worst, float(err.max() / amax))
    assert worst <= 2.0 ** -10 / 224.0


# ------------------------------------------------------------------ E4M3 activations and weights
# "Tensor-quantised" FP8 (the AWS abstract, backend paragraph; the Russian
# summary, section "Triton вместо CUTLASS для FP8-квантования"): one fp32
# scale per expert weight matrix, one static scale per activation tensor,
# value = code * scale.  These pins rebuild the all-E4M3 layer from pieces
# that are pinned above (the codec against the format and the library cast,
# routing against brute force) and numpy matrix products, so that a dropped,
# doubled or misplaced scale, or a skipped quantisation, fails them.
def _e4m3_workload(seed=11, n_shared=1):
    return syn.Workload("t", T=10, H=64, I=48, E=4, k=2, n_shared=n_shared, gate=syn.SIGMOID,
                        routed_scale=2.5, wdtype=syn.E4M3, adtype=syn.E4M3, seed=seed)


def _decoded(codes, scale):
    return orc.e4m3_decode(codes) * float(scale)


def test_fp8_layer_composes_from_pinned_pieces():
    wl = _e4m3_workload()
    d = syn.make_inputs(wl)
    a1 = float(d["a1"])
    a2 = 0.0153                                   # not a power of two: a scale slip shows
    E, I = wl.E, wl.I
    # tokens quantised once with a1 (fp32 quotient), then dequantised
    xq = orc.quant_e4m3_f32(syn.bf16_bits_to_f32(d["x"]), a1)
    xd = orc.e4m3_decode(xq) * a1
    ids, w = orc.route(d["logits"], wl.k, gate=orc.SIGMOID, renorm=True, routed_scale=2.5)

    def mlp(e, xrow):
        W1 = _decoded(d["w13"][e][:I], d["w13_scale"][e])
        W3 = _decoded(d["w13"][e][I:], d["w13_scale"][e])
        W2 = _decoded(d["w2"][e], d["w2_scale"][e])
        g, u = W1 @ xrow, W3 @ xrow
        h = g * expit(g) * u
        hq = orc.e4m3_decode(orc.e4m3_encode(h / a2)) * a2
        return W2 @ hq

    ref = np.zeros((wl.T, wl.H))
    for t in range(wl.T):
        for j in range(wl.k):
            ref[t] += w[t, j] * mlp(ids[t, j], xd[t])
        ref[t] += mlp(E, xd[t])                     # the shared expert, weight 1
    out = orc.forward(d["x"], d["logits"], d["w13"], d["w2"], E=E, k=wl.k, n_shared=1, gate=orc.SIGMOID,
                      routed_scale=2.5, wdtype=orc.E4M3, adtype=orc.E4M3, w13_scale=d["w13_scale"],
                      w2_scale=d["w2_scale"], a1=a1, a2=a2)
    rms = np.sqrt(np.mean(ref ** 2))
    assert np.max(np.abs(out - ref)) <= 1e-12 * rms
    # the same layer with the hidden quantisation or the token quantisation
    # left out is far away: the pin would catch either slip
    assert np.max(np.abs(orc.forward(d["x"], d["logits"], d["w13"], d["w2"], E=E, k=wl.k, n_shared=1,
                                     gate=orc.SIGMOID, routed_scale=2.5, wdtype=orc.E4M3, adtype=orc.BF16,
                                     w13_scale=d["w13_scale"], w2_scale=d["w2_scale"]) - ref)) > 1e-4 * rms


def test_fp8_expert_gemm_references_row_by_row():
    """orc.expert_swiglu / orc.expert_down with E4M3 activations (scales a1,
    a2) and E4M3 weights with non-unit per-expert scales, against numpy on the
    decoded values, row by row of every segment (pad rows included)."""
    wl = _e4m3_workload(seed=12, n_shared=0)
    d = syn.make_inputs(wl)
    I, H = wl.I, wl.H
    offsets = np.array([0, 16, 16, 48, 64], np.int32)          # expert 1 empty
    rows = int(offsets[-1])
    a1, a2 = 0.0071, 0.0213
    xp = syn.random_rows(wl.seed, "xp", rows, H, syn.E4M3)
    hq = syn.random_rows(wl.seed, "hq", rows, I, syn.E4M3)
    h = orc.expert_swiglu(xp, offsets, d["w13"], orc.E4M3, d["w13_scale"], adtype=orc.E4M3, a1=a1)
    y = orc.expert_down(hq, offsets, d["w2"], orc.E4M3, d["w2_scale"], adtype=orc.E4M3, a2=a2)
    xd = orc.e4m3_decode(xp) * a1
    hd = orc.e4m3_decode(hq) * a2
    for e in range(wl.E):
        W1 = _decoded(d["w13"][e][:I], d["w13_scale"][e])
        W3 = _decoded(d["w13"][e][I:], d["w13_scale"][e])
        W2 = _decoded(d["w2"][e], d["w2_scale"][e])
        for s in range(offsets[e], offsets[e + 1]):
            g, u = W1 @ xd[s], W3 @ xd[s]
            hr = g * expit(g) * u
            assert np.allclose(h[s], hr, rtol=1e-12, atol=1e-14 * np.abs(hr).max())
            yr = W2 @ hd[s]
            assert np.allclose(y[s], yr, rtol=1e-12, atol=1e-14 * np.abs(yr).max())


# ------------------------------------------------------------------ inverse rotary + per-head E4M3
# The Russian summary (section "Убрать лишние JIT-перекомпиляции Triton")
# names a fused rotary-embedding + per-head FP8 quantisation kernel.  These
# pins tie the oracle's reading (inverse rotation, neox or interleaved pairs,
# scale = amax/448 per head) to a right-angle rotation, the identity at
# position 0, scipy's rotation matrices, and a layout permutation.
def _rope_case(T=6, nh=3, hd=16, rot=16, seed=31):
    rw = syn.RopeWorkload("pin", T=T, n_heads=nh, head_dim=hd, rot_dim=rot, max_pos=64, base=1e4, seed=seed)
    return rw, syn.rope_inputs(rw)


def _head_scale(v):
    amax = np.float32(np.max(np.abs(v)))
    return np.float32(amax / np.float32(448.0)) if amax > 0 else np.float32(1.0)


def test_inv_rope_position_zero_is_plain_per_head_quantisation():
    rw, d = _rope_case()
    pos = np.zeros(rw.T, np.int32)
    q, sc = orc.inv_rope_quant(d["x"], pos, d["cos_sin"], rw.rot_dim)
    xf = syn.bf16_bits_to_f32(d["x"])
    for t in range(rw.T):
        for h in range(rw.n_heads):
            s = _head_scale(xf[t, h])
            assert sc[t, h] == s
            assert np.array_equal(q[t, h], orc.quant_e4m3_f32(xf[t, h], float(s)))


@pytest.mark.parametrize("interleaved", [False, True])
def test_inv_rope_right_angle_swaps_and_negates(interleaved):
    """A table row with cos = 0, sin = 1 exactly (a quarter turn): the inverse
    rotation maps each pair (a', b') to (b', -a')."""
    rw, d = _rope_case()
    cs = np.zeros((2, rw.rot_dim), np.float32)
    cs[1, rw.rot_dim // 2:] = 1.0
    pos = np.ones(rw.T, np.int32)
    q, sc = orc.inv_rope_quant(d["x"], pos, cs, rw.rot_dim, interleaved)
    xf = syn.bf16_bits_to_f32(d["x"])
    half = rw.rot_dim // 2
    r = np.empty_like(xf)
    for i in range(half):
        a, b = (2 * i, 2 * i + 1) if interleaved else (i, i + half)
        r[..., a] = xf[..., b]
        r[..., b] = -xf[..., a]
    for t in range(rw.T):
        for h in range(rw.n_heads):
            s = _head_scale(r[t, h])
            assert sc[t, h] == s
            assert np.array_equal(q[t, h], orc.quant_e4m3_f32(r[t, h], float(s)))


def test_inv_rope_matches_scipy_rotation_by_minus_theta():
    """General angles: each pair rotated by -theta (theta from the table's
    cos/sin) with scipy's rotation matrices, in double; the oracle's codes
    decode to it within half an E4M3 step (plus fp32 rounding)."""
    from scipy.spatial.transform import Rotation
    rw, d = _rope_case(T=12, nh=2, hd=32, rot=32, seed=33)
    q, sc = orc.inv_rope_quant(d["x"], d["positions"], d["cos_sin"], rw.rot_dim)
    xf = syn.bf16_bits_to_f32(d["x"]).astype(np.float64)
    half = rw.rot_dim // 2
    for t in range(rw.T):
        row = d["cos_sin"][d["positions"][t]].astype(np.float64)
        theta = np.arctan2(row[half:], row[:half])
        for h in range(rw.n_heads):
            ref = np.empty(rw.head_dim)
            for i in range(half):
                v = np.array([xf[t, h, i], xf[t, h, i + half], 0.0])
                a, b, _ = Rotation.from_euler("z", -theta[i]).apply(v)
                ref[i], ref[i + half] = a, b
            got = orc.e4m3_decode(q[t, h]) * float(sc[t, h])
            step = np.exp2(np.floor(np.log2(np.maximum(np.abs(ref), 1e-30) / sc[t, h]))) * 2.0 ** -3
            tol = 0.5 * np.maximum(step, 2.0 ** -9) * sc[t, h] + 1e-5 * np.abs(ref).max()
            assert np.all(np.abs(got - ref) <= tol)
            assert np.abs(got).max() == pytest.approx(448.0 * float(sc[t, h]), rel=0, abs=0)


def test_inv_rope_neox_and_interleaved_layouts_are_a_permutation_apart():
    rw, d = _rope_case(T=8, nh=4, hd=32, rot=24, seed=35)
    half = rw.rot_dim // 2
    perm = np.arange(rw.head_dim)                 # interleaved slot -> neox slot
    perm[0:rw.rot_dim:2] = np.arange(half)
    perm[1:rw.rot_dim:2] = np.arange(half) + half
    q_n, s_n = orc.inv_rope_quant(d["x"], d["positions"], d["cos_sin"][:, :rw.rot_dim], rw.rot_dim, False)
    q_i, s_i = orc.inv_rope_quant(d["x"][..., perm], d["positions"], d["cos_sin"][:, :rw.rot_dim], rw.rot_dim, True)
    assert np.array_equal(s_n, s_i)
    assert np.array_equal(q_n[..., perm], q_i)


def test_inv_rope_partial_rotary_passes_the_rest_through():
    rw, d = _rope_case(T=5, nh=2, hd=32, rot=16, seed=37)
    cs = syn.rope_table(dataclasses.replace(rw, rot_dim=16))
    q, sc = orc.inv_rope_quant(d["x"], d["positions"], cs, 16)
    xf = syn.bf16_bits_to_f32(d["x"])
    for t in range(rw.T):
        for h in range(rw.n_heads):
            assert np.array_equal(q[t, h, 16:], orc.quant_e4m3_f32(xf[t, h, 16:], float(sc[t, h])))


def test_inv_rope_position_out_of_range_gives_zero_codes_and_scale():
    rw, d = _rope_case()
    pos = d["positions"].copy()
    pos[2], pos[4] = -1, 64
    q, sc = orc.inv_rope_quant(d["x"], pos, d["cos_sin"], rw.rot_dim)
    assert np.all(q[[2, 4]] == 0) and np.all(sc[[2, 4]] == 0)
    assert np.all(sc[[0, 1, 3, 5]] > 0)
