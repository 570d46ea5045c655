"""GPU parity of the attention-side step (inverse rotary embedding + per-head
E4M3 quantisation) against the oracle: codes and scales bit for bit, since
both decide each code in the same fp32 arithmetic."""
import dataclasses

import numpy as np
import pytest
import torch

import mixture_experts_layer_22_b200 as moe
import oracle as orc
from mixture_experts_layer_22_b200 import synthetic as syn

pytestmark = pytest.mark.gpu

R = syn.ROPE_WORKLOADS


def _run(rw, d, positions=None, status=None):
    pos = d["positions"] if positions is None else positions
    s = moe.RopeShape.of(rw)
    x = torch.from_numpy(d["x"].view(np.int16)).cuda().view(torch.bfloat16)
    q = torch.full((rw.T, rw.n_heads, rw.head_dim), 0xAA, dtype=torch.uint8, device="cuda")
    sc = torch.full((rw.T, rw.n_heads), -1.0, dtype=torch.float32, device="cuda")
    moe.inv_rope_quant(s, x, torch.from_numpy(pos).cuda(), torch.from_numpy(d["cos_sin"]).cuda(), q, sc, status)
    torch.cuda.synchronize()
    return q.cpu().numpy(), sc.cpu().numpy()


def _check(rw, d, positions=None):
    q, sc = _run(rw, d, positions)
    pos = d["positions"] if positions is None else positions
    rq, rs = orc.inv_rope_quant(d["x"], pos, d["cos_sin"], rw.rot_dim, rw.interleaved)
    assert np.array_equal(sc, rs)
    assert np.array_equal(q, rq)


@pytest.mark.parametrize("name", sorted(R))
def test_inv_rope_quant_full_size_bit_exact(name):
    rw = R[name]
    _check(rw, syn.rope_inputs(rw))


SMALL = [
    syn.RopeWorkload("t1", T=1, n_heads=1, head_dim=128, rot_dim=128),
    syn.RopeWorkload("odd_T", T=333, n_heads=5, head_dim=128, rot_dim=128, seed=1),
    syn.RopeWorkload("hd64_il", T=77, n_heads=3, head_dim=64, rot_dim=64, interleaved=True, seed=2),
    syn.RopeWorkload("hd256", T=40, n_heads=2, head_dim=256, rot_dim=256, seed=3),
    syn.RopeWorkload("partial", T=50, n_heads=4, head_dim=128, rot_dim=64, seed=4),
    syn.RopeWorkload("partial_il", T=50, n_heads=4, head_dim=256, rot_dim=96, interleaved=True, seed=5),
    syn.RopeWorkload("rot16", T=9, n_heads=2, head_dim=64, rot_dim=16, seed=6),
    syn.RopeWorkload("partial96", T=21, n_heads=3, head_dim=128, rot_dim=96, seed=12),
    syn.RopeWorkload("partial48_hd64", T=19, n_heads=9, head_dim=64, rot_dim=48, seed=13),
    syn.RopeWorkload("partial_il_odd", T=11, n_heads=2, head_dim=64, rot_dim=22, interleaved=True, seed=14),
    syn.RopeWorkload("rot2_il", T=9, n_heads=3, head_dim=128, rot_dim=2, interleaved=True, seed=10),
    syn.RopeWorkload("many_heads", T=3, n_heads=77, head_dim=64, rot_dim=64, seed=11),
]


# Larger shapes: many warp items per resident warp, ragged head chunks
LARGE = [
    syn.RopeWorkload("large_partial96", T=5000, n_heads=3, head_dim=128, rot_dim=96, seed=21),
    syn.RopeWorkload("large_il_hd256_ragged", T=2400, n_heads=20, head_dim=256, rot_dim=200, interleaved=True,
                     seed=22),
    syn.RopeWorkload("large_hd64_il_partial", T=2500, n_heads=40, head_dim=64, rot_dim=38, interleaved=True,
                     seed=23),
]


@pytest.mark.parametrize("rw", LARGE, ids=lambda r: r.name)
def test_inv_rope_quant_large_shapes_bit_exact(rw):
    _check(rw, syn.rope_inputs(rw))


def test_inv_rope_quant_large_reports_positions_out_of_range():
    rw = syn.RopeWorkload("badpos_large", T=6000, n_heads=4, head_dim=128, rot_dim=128, max_pos=4096, seed=24)
    d = syn.rope_inputs(rw)
    pos = d["positions"].copy()
    pos[[7, 4000, 5999]] = [-1, 4096, 99999]
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    q, sc = _run(rw, d, pos, status)
    assert int(status[0]) == -5                              # MOE_ERR_DEVICE_CHECK
    assert np.all(q[[7, 4000, 5999]] == 0) and np.all(sc[[7, 4000, 5999]] == 0)
    rq, rs = orc.inv_rope_quant(d["x"], pos, d["cos_sin"], rw.rot_dim)
    assert np.array_equal(q, rq) and np.array_equal(sc, rs)


@pytest.mark.parametrize("rw", SMALL, ids=lambda r: r.name)
def test_inv_rope_quant_shapes_bit_exact(rw):
    _check(rw, syn.rope_inputs(rw))


@pytest.mark.parametrize("rw", [
    syn.RopeWorkload("zeros_neox", T=40, n_heads=4, head_dim=128, rot_dim=96, seed=31),
    syn.RopeWorkload("zeros_il", T=40, n_heads=5, head_dim=64, rot_dim=38, interleaved=True, seed=32),
    syn.RopeWorkload("zeros_neox_large", T=5000, n_heads=3, head_dim=128, rot_dim=96, seed=33),
    syn.RopeWorkload("zeros_il_large", T=2500, n_heads=40, head_dim=64, rot_dim=38, interleaved=True, seed=34),
], ids=lambda r: r.name)
def test_inv_rope_quant_signed_zero_elements(rw):
    """Exact +0 and -0 elements inside heads of ordinary scale keep the sign
    of their quotient (IEEE division: -0 / scale = -0, code 0x80), rotated
    or passed through."""
    d = syn.rope_inputs(rw)
    x = d["x"].copy()
    half = rw.rot_dim // 2
    if rw.interleaved:
        x[:, :, 0] = 0x8000; x[:, :, 1] = 0x8000          # a pair of -0
        x[:, :, 2] = 0x8000; x[:, :, 3] = 0x0000          # -0 with a +0 partner
    else:
        x[:, :, 0] = 0x8000; x[:, :, half] = 0x8000
        x[:, :, 1] = 0x8000; x[:, :, half + 1] = 0x0000
    x[:, :, rw.rot_dim] = 0x8000                          # passed through
    x[:, :, rw.rot_dim + 1] = 0x0000
    d["x"] = x
    _check(rw, d)
    q, _ = _run(rw, d)
    assert np.all(q[:, :, rw.rot_dim] == 0x80) and np.all(q[:, :, rw.rot_dim + 1] == 0x00)


def test_inv_rope_quant_zero_head_and_extreme_values():
    rw = syn.RopeWorkload("ext", T=16, n_heads=4, head_dim=128, rot_dim=128, seed=7)
    d = syn.rope_inputs(rw)
    x = d["x"].copy()
    x[0, 0] = 0                                              # an all-zero head: scale 1, codes 0
    x[1] = syn.to_bf16_bits(syn.bf16_bits_to_f32(x[1]) * 1e30)
    x[2] = syn.to_bf16_bits(syn.bf16_bits_to_f32(x[2]) * 1e-30)
    d["x"] = x
    _check(rw, d)
    q, sc = _run(rw, d)
    # an all-zero head: scale 1, every code +0 or -0 (a zero times a negative
    # cosine is -0, code 0x80)
    assert sc[0, 0] == 1.0 and np.all((q[0, 0] & 0x7F) == 0)


def test_inv_rope_quant_reports_positions_out_of_range():
    rw = syn.RopeWorkload("badpos", T=64, n_heads=4, head_dim=128, rot_dim=128, max_pos=512, seed=8)
    d = syn.rope_inputs(rw)
    pos = d["positions"].copy()
    pos[[3, 40]] = [-5, 512]
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    q, sc = _run(rw, d, pos, status)
    assert int(status[0]) == -5                              # MOE_ERR_DEVICE_CHECK
    assert np.all(q[[3, 40]] == 0) and np.all(sc[[3, 40]] == 0)
    rq, rs = orc.inv_rope_quant(d["x"], pos, d["cos_sin"], rw.rot_dim)
    assert np.array_equal(q, rq) and np.array_equal(sc, rs)
    ok = torch.zeros(1, dtype=torch.int32, device="cuda")
    _run(rw, d, None, ok)
    assert int(ok[0]) == 0


def test_inv_rope_quant_token_count_is_a_runtime_value():
    """One library, every token count: T = 1..40 of the same inputs give the
    first T rows of the T = 40 result."""
    rw = syn.RopeWorkload("rt", T=40, n_heads=2, head_dim=128, rot_dim=128, seed=9)
    d = syn.rope_inputs(rw)
    q40, s40 = _run(rw, d)
    for T in (1, 2, 3, 17, 39):
        sub = dataclasses.replace(rw, T=T)
        dd = {"x": d["x"][:T], "positions": d["positions"][:T], "cos_sin": d["cos_sin"]}
        q, sc = _run(sub, dd)
        assert np.array_equal(q, q40[:T]) and np.array_equal(sc, s40[:T])
