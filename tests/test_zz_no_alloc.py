"""The workspace-free align/permute entry point, for callers that cannot
allocate device memory (an engine that owns all of it through its own
allocator, or a loop where cudaMalloc may not run).  Its results must equal
those of the regular moe_align_permute, call after call, even though every call
reuses the library's one fixed scratch array.  Collected last on purpose."""
import numpy as np
import pytest
import torch

import mixture_experts_layer_22_b200 as moe
from mixture_experts_layer_22_b200 import synthetic as syn

pytestmark = pytest.mark.gpu


def _ids(T, E, k, seed):
    rng = np.random.default_rng(seed)
    return np.stack([rng.permutation(E)[:k] for _ in range(T)]).astype(np.int32)


def _buffers(s, T, k, E, ns):
    mr = moe.max_rows(s)
    return (torch.empty(E + ns, dtype=torch.int32, device="cuda"),
            torch.empty(E + ns + 1, dtype=torch.int32, device="cuda"),
            torch.full((mr,), -7, dtype=torch.int32, device="cuda"),
            torch.empty(T * k, dtype=torch.int32, device="cuda"))


@pytest.mark.parametrize("calls", [[(3000, 60, 4, 0, 16, 1), (64, 8, 2, 0, 16, 2)],
                                   [(128, 256, 8, 1, 16, 3), (128, 256, 8, 1, 16, 4)]])
def test_noalloc_align_equals_workspace_align_on_consecutive_calls(calls):
    for T, E, k, ns, pad, seed in calls:                     # two calls in a row
        wl = syn.Workload("na", T=T, H=128, I=128, E=E, k=k, n_shared=ns)
        s = moe.Shape.of(wl, pad=pad)
        ids = torch.from_numpy(_ids(T, E, k, seed)).cuda()
        ref = _buffers(s, T, k, E, ns)
        ws = moe.workspace(s)
        moe.reset_device_status(ws)
        moe.align_permute(s, ids, *ref, ws)
        got = _buffers(s, T, k, E, ns)
        status = torch.full((1,), 99, dtype=torch.int32, device="cuda")
        moe.align_permute_noalloc(s, ids, *got, status)
        torch.cuda.synchronize()
        total = int(ref[1][-1])
        assert torch.equal(got[0], ref[0])
        assert torch.equal(got[1], ref[1])
        assert torch.equal(got[2][:total], ref[2][:total])
        assert torch.equal(got[3], ref[3])
        assert int(status[0]) == 0 and moe.device_status(ws) == 0


def test_noalloc_align_rejects_shapes_beyond_its_scratch():
    wl = syn.Workload("na", T=20000, H=128, I=128, E=8, k=4)    # 80000 routed rows > 65536
    s = moe.Shape.of(wl)
    dummy = torch.empty(16, dtype=torch.int32, device="cuda")
    with pytest.raises(moe.MoeError) as e:
        moe.align_permute_noalloc(s, dummy, dummy, dummy, dummy, dummy)
    assert e.value.code == -2


@pytest.mark.parametrize("T,E,k", [(64, 8, 2), (3000, 60, 4)])       # one-kernel and two-kernel paths
def test_noalloc_align_reports_a_bad_id_then_starts_clean(T, E, k):
    """An expert id outside 0..E-1 is reported through the optional status
    output; the next call on the same shared array starts from a clear status
    and matches moe_align_permute again.  The launch count is this call's."""
    wl = syn.Workload("na", T=T, H=128, I=128, E=E, k=k)
    s = moe.Shape.of(wl)
    ids_np = _ids(T, E, k, 5)
    bad = ids_np.copy()
    bad[T // 2, 0] = E                                           # one id out of range
    status = torch.full((1,), 99, dtype=torch.int32, device="cuda")
    got = _buffers(s, T, k, E, 0)
    moe.align_permute_noalloc(s, torch.from_numpy(bad).cuda(), *got, status)
    torch.cuda.synchronize()
    assert int(status[0]) == -5                                  # MOE_ERR_DEVICE_CHECK
    assert moe.last_launch_count() == (1 if T * k <= 1024 else 2)
    ids = torch.from_numpy(ids_np).cuda()
    ref = _buffers(s, T, k, E, 0)
    ws = moe.workspace(s)
    moe.reset_device_status(ws)
    moe.align_permute(s, ids, *ref, ws)
    got = _buffers(s, T, k, E, 0)
    moe.align_permute_noalloc(s, ids, *got, status)
    torch.cuda.synchronize()
    assert int(status[0]) == 0
    total = int(ref[1][-1])
    for g, r in zip(got[:2], ref[:2]):
        assert torch.equal(g, r)
    assert torch.equal(got[2][:total], ref[2][:total])
    assert torch.equal(got[3], ref[3])
