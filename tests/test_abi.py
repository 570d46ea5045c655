"""The C-ABI library on the host, without a GPU: it loads, exports every entry
point include/moe.h declares, sizes buffers by the documented formulas and
rejects bad arguments before launching anything."""
import ctypes as C
import os
import re

import pytest

import mixture_experts_layer_22_b200 as moe
from mixture_experts_layer_22_b200 import build as mbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    mbuild.build()
    return moe.lib()


def _declared():
    src = open(os.path.join(ROOT, "include", "moe.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(moe_[a-z_0-9]+)\s*\(", src)))


def test_every_declared_symbol_is_exported(lib):
    names = _declared()
    assert len(names) >= 13
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(moe.EXPORTS)


def _shape(**kw):
    base = dict(T=64, H=4096, I=14336, E=8, k=2, n_shared=0, gate=0, renorm=1, routed_scale=1.0,
                wdtype=0, adtype=0, pad=16, variant=0)
    base.update(kw)
    return moe.Shape(**base)


@pytest.mark.parametrize("T,k,E,ns,pad", [(64, 2, 8, 0, 16), (1, 8, 256, 1, 16), (8192, 4, 60, 0, 128),
                                          (33, 3, 5, 0, 1)])
def test_max_rows_formula(lib, T, k, E, ns, pad):
    s = _shape(T=T, k=k, E=E, n_shared=ns, pad=pad, H=256, I=256)
    assert moe.max_rows(s) == T * k + ns * T + (E + ns) * (pad - 1)


def test_workspace_size_is_aligned_and_grows_with_T(lib):
    a = moe.workspace_size(_shape(T=8))
    b = moe.workspace_size(_shape(T=64))
    c = moe.workspace_size(_shape(T=4096))
    assert a % 256 == 0 and a < b < c


def test_status_strings(lib):
    for code in [0, -1, -2, -3, -4, -5, -6]:
        assert moe.status_string(code) and moe.status_string(code) != "unknown status"
    assert moe.status_string(-99) == "unknown status"


@pytest.mark.parametrize("bad", [dict(k=9), dict(k=0), dict(T=0), dict(E=513, k=2), dict(gate=2),
                                 dict(wdtype=0, adtype=1), dict(n_shared=2), dict(variant=3),
                                 dict(pad=0), dict(k=33, E=64)])
def test_invalid_shapes_rejected(lib, bad):
    s = _shape(**bad)
    assert lib.moe_workspace_size(C.byref(s), C.byref(C.c_size_t())) == -1


@pytest.mark.parametrize("bad", [dict(H=200), dict(I=100), dict(pad=8), dict(pad=512)])
def test_gemm_rejects_unbuilt_shapes_before_launch(lib, bad):
    s = _shape(**bad)
    r = lib.moe_grouped_gemm_swiglu(C.byref(s), 16, 16, 16, 1.0, 1.0, 16, 16, 256, 1 << 30, None)
    assert r == -2


def test_null_pointers_rejected_before_launch(lib):
    s = _shape()
    assert lib.moe_route_topk(C.byref(s), None, None, None, None) == -1
    assert lib.moe_combine(C.byref(s), None, None, None, None, None, None) == -1
    assert lib.moe_fused_forward(C.byref(s), None, None, None, None, None, None, 1.0, 1.0, None, None, 0,
                                 None) == -1
    assert lib.moe_align_permute(None, None, None, None, None, None, None, 0, None) == -1


def test_router_entry_points_reject_bad_arguments(lib):
    s = _shape(H=256, I=256)
    need = moe.workspace_size(s)
    assert lib.moe_router_topk(C.byref(s), None, 256, 256, 256, 256, 256, need, None) == -1
    assert lib.moe_router_topk(C.byref(s), 264, 256, 256, 256, 256, 256, need, None) == -1   # misaligned x
    assert lib.moe_router_topk(C.byref(s), 256, 256, 256, 256, 256, 256, need - 1, None) == -3
    assert lib.moe_fused_forward_router(C.byref(s), 256, None, 256, None, 256, None, 1.0, 1.0, 256, 256, need,
                                        None) == -1
    assert lib.moe_fused_forward_router(C.byref(s), 256, 264, 256, None, 256, None, 1.0, 1.0, 256, 256, need,
                                        None) == -1


def test_workspace_too_small_rejected(lib):
    s = _shape()
    need = moe.workspace_size(s)
    r = lib.moe_fused_forward(C.byref(s), 256, 256, 256, None, 256, None, 1.0, 1.0, 256, 256, need - 1, None)
    assert r == -3


def test_fp8_requires_scales(lib):
    s = _shape(wdtype=1, adtype=1, H=256, I=256)
    need = moe.workspace_size(s)
    r = lib.moe_fused_forward(C.byref(s), 256, 256, 256, None, 256, None, 1.0, 1.0, 256, 256, need, None)
    assert r == -1


def test_misaligned_pointers_rejected(lib):
    s = _shape(H=256, I=256)
    need = moe.workspace_size(s)
    r = lib.moe_fused_forward(C.byref(s), 258, 256, 256, None, 256, None, 1.0, 1.0, 256, 256, need, None)
    assert r == -1
    r = lib.moe_fused_forward(C.byref(s), 256, 256, 256, None, 256, None, 1.0, 1.0, 256, 272, need, None)
    assert r == -1


def _rope(**kw):
    base = dict(num_tokens=8, n_heads=4, head_dim=128, rot_dim=128, max_pos=64, interleaved=0)
    base.update(kw)
    return moe.RopeShape(**base)


@pytest.mark.parametrize("kw,code", [({"head_dim": 96, "rot_dim": 96}, -2), ({"rot_dim": 7}, -1),
                                     ({"rot_dim": 24}, -2), ({"rot_dim": 24, "interleaved": 1, "num_tokens": 0}, 0),
                                     ({"rot_dim": 130}, -1), ({"n_heads": 0}, -1), ({"interleaved": 2}, -1),
                                     ({"num_tokens": -1}, -1), ({"max_pos": 0}, -1)])
def test_inv_rope_rejects_bad_shapes_before_launch(lib, kw, code):
    assert lib.moe_inv_rope_quant_per_head(C.byref(_rope(**kw)), 16, 16, 16, 16, 16, None, None) == code


def test_inv_rope_rejects_null_and_misaligned_pointers(lib):
    s = _rope()
    assert lib.moe_inv_rope_quant_per_head(C.byref(s), None, 16, 16, 16, 16, None, None) == -1
    assert lib.moe_inv_rope_quant_per_head(C.byref(s), 8, 16, 16, 16, 16, None, None) == -1   # x not 16-aligned
    assert lib.moe_inv_rope_quant_per_head(C.byref(s), 16, 16, 16, 4, 16, None, None) == -1   # q not 8-aligned
    assert lib.moe_inv_rope_quant_per_head(C.byref(_rope(num_tokens=0)), None, None, None, None, None, None,
                                           None) == 0                                        # nothing to do
