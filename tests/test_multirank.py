"""The N > 1 host path of bench.py on CPU: two gloo ranks ("replicas only" --
every rank runs its own copy of the layer, there is no data-path
collective).  The job's time is the slowest rank's and its throughput counts
every rank's tokens; the reference arm runs on rank 0 only."""
import os
import socket
import sys

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        local_ms = [120.0, 80.0][rank]                    # rank 0 is the slow one
        ms, value = bench.aggregate_over_ranks(local_ms, tokens_per_rank=64, steps=10, dist_mod=dist)
        q.put((rank, ms, value))
    finally:
        dist.destroy_process_group()


def test_two_rank_aggregation_takes_the_slowest_rank():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(2))
    for rank, ms, value in res:
        assert ms == 120.0                               # max over ranks, on every rank
        assert value == pytest.approx(2 * 64 * 10 / 0.120)


def test_single_rank_aggregation():
    sys.path.insert(0, ROOT)
    import bench
    ms, value = bench.aggregate_over_ranks(50.0, tokens_per_rank=8, steps=4)
    assert ms == 50.0 and value == pytest.approx(8 * 4 / 0.05)


def test_reference_arm_runs_on_rank0_only(monkeypatch, capsys):
    sys.path.insert(0, ROOT)
    import bench
    from mixture_experts_layer_22_b200 import synthetic as syn
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    args = type("A", (), {"steps": 1, "warmup": 3, "gpus": 2, "ref_budget": 1.0})()
    assert bench.reference_main(args, syn.WORKLOADS["tiny"]) == 0
    assert capsys.readouterr().out == ""


def test_reference_arm_prints_the_contract_line(monkeypatch, capsys):
    sys.path.insert(0, ROOT)
    import json
    import bench
    from mixture_experts_layer_22_b200 import synthetic as syn
    monkeypatch.setenv("RANK", "0")
    monkeypatch.setenv("WORLD_SIZE", "1")
    args = type("A", (), {"steps": 1, "warmup": 3, "gpus": 1, "ref_budget": 0.2})()
    assert bench.reference_main(args, syn.WORKLOADS["tiny"]) == 0
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["unit"] == "tokens/s" and line["value"] > 0
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["cpu_baseline"]["kind"] == "oracle"
