"""Generated cases for the oracle's integer steps (routing and alignment),
beside the fixed pins: hypothesis draws small shapes, gates and logits full of
exact ties, and every case is checked against brute force or against the
invariants that define the step (top-k by logit with ties to the lower id; a
stable counting sort into padded segments)."""
import itertools

import numpy as np
from hypothesis import given, settings, strategies as st
from scipy.special import expit

import oracle as orc


def _brute_topk(l, k):
    """The k experts ranked first by (logit, then lower id): the unique
    k-subset whose every member outranks every non-member."""
    key = lambda e: (l[e], -e)
    E = len(l)
    found = [S for S in itertools.combinations(range(E), k)
             if all(key(a) > key(b) for a in S for b in range(E) if b not in S)]
    assert len(found) == 1
    return sorted(found[0], key=key, reverse=True)


@st.composite
def _routing_case(draw):
    E = draw(st.integers(1, 7))
    k = draw(st.integers(1, E))
    T = draw(st.integers(1, 6))
    # small integer logits: many exact ties
    vals = draw(st.lists(st.integers(-3, 3), min_size=T * E, max_size=T * E))
    logits = np.array(vals, dtype=np.float32).reshape(T, E)
    gate = draw(st.sampled_from([orc.SOFTMAX, orc.SIGMOID]))
    renorm = draw(st.booleans())
    scale = draw(st.sampled_from([1.0, 2.5]))
    return logits, k, gate, renorm, scale


@settings(max_examples=150, deadline=None)
@given(_routing_case())
def test_route_generated_cases_match_brute_force(case):
    logits, k, gate, renorm, scale = case
    ids, w = orc.route(logits, k, gate=gate, renorm=renorm, routed_scale=scale)
    l64 = logits.astype(np.float64)
    for t in range(logits.shape[0]):
        assert list(ids[t]) == _brute_topk(list(logits[t]), k)
        sel = l64[t, ids[t]]
        if gate == orc.SOFTMAX:
            if renorm:
                p = np.exp(sel - sel.max())
                expect = p / p.sum()
            else:
                p = np.exp(l64[t] - l64[t].max())
                expect = np.exp(sel - l64[t].max()) / p.sum()
        else:
            s = expit(sel)
            expect = s / s.sum() if renorm else s
        assert np.allclose(w[t], scale * expect, rtol=1e-12, atol=1e-15)


@st.composite
def _align_case(draw):
    E = draw(st.integers(1, 40))
    k = draw(st.integers(1, min(E, 8)))
    T = draw(st.integers(1, 40))
    n_shared = draw(st.integers(0, 1))
    pad = draw(st.sampled_from([1, 2, 16, 64]))
    seed = draw(st.integers(0, 2 ** 32 - 1))
    rng = np.random.default_rng(seed)
    ids = np.stack([rng.permutation(E)[:k] for _ in range(T)]).astype(np.int32)
    return ids, E, n_shared, pad


@settings(max_examples=150, deadline=None)
@given(_align_case())
def test_align_generated_cases_are_a_stable_padded_counting_sort(case):
    ids, E, n_shared, pad = case
    T, k = ids.shape
    R = T * k
    counts, offsets, rows, inv = orc.align(ids, E, n_shared, pad)
    flat = ids.ravel()
    assert counts[:E].tolist() == np.bincount(flat, minlength=E).tolist()
    assert counts[E:].tolist() == [T] * n_shared
    assert offsets[0] == 0
    seg = np.diff(offsets)
    assert np.array_equal(seg, -(-counts // pad) * pad)
    order = np.argsort(flat, kind="stable")
    got = np.concatenate([rows[offsets[e]:offsets[e] + counts[e]] for e in range(E)])
    assert np.array_equal(got, order)
    for e in range(E + n_shared):
        assert np.all(rows[offsets[e] + counts[e]:offsets[e + 1]] == -1)
    for s in range(n_shared):
        assert np.array_equal(rows[offsets[E + s]:offsets[E + s] + T], R + s * T + np.arange(T))
    assert np.array_equal(rows[inv], np.arange(R))
    assert np.array_equal(np.sort(inv), np.sort(np.flatnonzero((rows >= 0) & (rows < R))))
