"""Throughput of the fused-MoE layer on B200.

Headline workload: the DeepSeek-V3-shaped decode layer at T=128 tokens (H=7168,
I=2048, E=256 routed experts top-8 with sigmoid scores renormalised x2.5, one
shared expert, 11.3 GB of E4M3 weights with per-expert scales, bf16
activations), the largest configuration that runs on one GPU: one
moe_fused_forward per step with inputs resident in HBM.  At N=1 the same JSON
line also carries `per_workload`, the same measurements for every other
configuration (tiny layer; Mixtral decode T=1/8/64; Mixtral E4M3 prefill
T=4096; DeepSeek-V3 decode T=1/8/32, with E4M3 weights and with E4M3
activations too; Qwen2-MoE skewed prefill T=8192) and for the attention-side
inverse-rotary + per-head E4M3 step.  Prints one JSON line.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                  [--workload NAME] [--T T] [--no-sweep]

N > 1 (under torchrun): every rank runs an independent replica of the
headline layer ("replicas only": the single-GPU layer has no exchange step);
value is the tokens of all ranks over the slowest rank's device time.
--impl reference times the CPU oracle (the reference arm of this project) on
a bounded sample of the headline workload.
"""
from __future__ import annotations

import argparse
import dataclasses
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from mixture_experts_layer_22_b200 import synthetic as syn  # noqa: E402

METRIC = "fused-MoE layer tokens/s"
UNIT = "tokens/s"
HEADLINE = ("dsv3_decode_fp8w", 128)
# (workload, T) measured in the per-workload sweep, besides the headline
SWEEP = [("dsv3_decode_fp8w", 1), ("dsv3_decode_fp8w", 8), ("dsv3_decode_fp8w", 32),
         ("dsv3_decode_fp8", 1), ("dsv3_decode_fp8", 8), ("dsv3_decode_fp8", 32), ("dsv3_decode_fp8", 128),
         ("tiny", 16), ("mixtral_decode", 1), ("mixtral_decode", 8), ("mixtral_decode", 64),
         ("mixtral_prefill_fp8", 4096), ("qwen2_skewed_prefill", 8192)]
L2_BYTES = 126 * 2 ** 20


def workload_desc(wl) -> str:
    dt = {(0, 0): "bf16", (1, 1): "fp8 e4m3 w+a", (1, 0): "fp8 e4m3 w, bf16 a"}[(wl.wdtype, wl.adtype)]
    gate = "softmax" if wl.gate == syn.SOFTMAX else f"sigmoid x{wl.routed_scale}"
    sh = f" +{wl.n_shared} shared" if wl.n_shared else ""
    return (f"{wl.name}: T={wl.T} H={wl.H} I={wl.I} E={wl.E} top-{wl.k} {gate}{sh}, {dt}")


def config_of(wl, parallelism: str, launch: str = "", l2: str = "") -> dict:
    return {"workload": workload_desc(wl), "T": wl.T, "H": wl.H, "I": wl.I, "E": wl.E, "k": wl.k,
            "n_shared": wl.n_shared, "parallelism": parallelism, "launch": launch, "l2": l2,
            "inputs": "seeded synthetic (seed 0), resident in HBM before timing"}


def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def aggregate_over_ranks(ms_local: float, tokens_per_rank: int, steps: int, dist_mod=None):
    """Slowest rank's timed-region milliseconds and the whole-job tokens/s:
    every rank contributes `tokens_per_rank * steps` tokens, the job takes as
    long as its slowest rank.  With dist_mod (torch.distributed, initialised)
    the max is an all-reduce over the process group; every rank returns the
    same numbers."""
    import torch
    world = 1
    ms = float(ms_local)
    if dist_mod is not None and dist_mod.is_initialized():
        world = dist_mod.get_world_size()
        dev = torch.device("cuda", torch.cuda.current_device()) if dist_mod.get_backend() == "nccl" else "cpu"
        t = torch.tensor([ms], dtype=torch.float64, device=dev)
        dist_mod.all_reduce(t, op=dist_mod.ReduceOp.MAX)
        ms = float(t.item())
    return ms, world * tokens_per_rank * steps / (ms / 1e3)


def weight_bytes_per_expert(wl) -> int:
    esz = 2 if wl.wdtype == syn.BF16 else 1
    return 3 * wl.H * wl.I * esz


def workload_of(name: str, T: int):
    return syn.WORKLOADS[name].with_T(T)


# ---------------------------------------------------------------- reference arm
def cpu_oracle_rate(wl, d, budget_s: float = 15.0, a2: float = 1.0):
    """Tokens/s of the oracle on this host, from a bounded token sample."""
    import oracle as orc

    def run(toks):
        t0 = time.perf_counter()
        orc.forward(d["x"], d["logits"], d["w13"], d["w2"], E=wl.E, k=wl.k, n_shared=wl.n_shared,
                    gate=wl.gate, renorm=wl.renorm, routed_scale=wl.routed_scale, wdtype=wl.wdtype,
                    adtype=wl.adtype, w13_scale=d["w13_scale"], w2_scale=d["w2_scale"],
                    a1=float(d.get("a1", 1.0)), a2=a2, tokens=np.asarray(toks, np.int32))
        return time.perf_counter() - t0

    cores = orc.num_threads()
    n = min(wl.T, cores)
    dt = run(list(range(n)))
    while dt < budget_s / 3 and n < wl.T:
        n = min(wl.T, max(n + 1, int(n * min(4.0, budget_s / max(dt, 1e-3)))))
        dt = run(list(range(n)))
    return n / dt, cores, f"first {n} of {wl.T} tokens, {dt:.1f} s of host time"


def reference_main(args, wl):
    ws_n, rank, _ = dist_env()
    if rank != 0:
        return 0
    d = syn.make_inputs(wl)
    a2 = static_hidden_scale(wl)
    for _ in range(args.warmup):
        cpu_oracle_rate(wl, d, budget_s=2.0, a2=a2)
    rates = []
    # each step a bounded sample, so that the whole run ends in a few minutes
    budget = min(args.ref_budget, max(1.0, 150.0 / max(1, args.steps)))
    for _ in range(args.steps):
        r, cores, sample = cpu_oracle_rate(wl, d, budget_s=budget, a2=a2)
        rates.append(r)
    value = statistics.median(rates)
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * wl.T / value,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": config_of(wl, "cpu oracle"),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------- clocks
class ClockSampler:
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.idx = gpu_index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.idx}", f"--query-gpu={self.QUERY}",
                                          "--format=csv,noheader,nounits", "-lms", "50"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except (OSError, FileNotFoundError):
            self.proc = None

    def _read(self):
        for ln in self.proc.stdout:
            self.lines.append(ln.strip())

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.1)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        sm, smax, reasons, power = [], [], set(), []
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                smax.append(float(f[2]))
                power.append(float(f[3]))
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm),
                "power_w_median": statistics.median(power) if power else None}


# ---------------------------------------------------------------- measurement helpers
def measured_peaks():
    """(hbm GB/s, bf16 TF/s burst, bf16 TF/s sustained, kind)."""
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            m = json.load(f)
        return float(m["hbm_gbs"]), float(m["bf16_tflops"]), float(m["bf16_tflops_sustained"]), "measured"
    except (OSError, KeyError, ValueError):
        return 6650.0, 1590.0, 1400.0, "fallback"


def source_sha256(names) -> str:
    """sha256 over the named kernel source files, concatenated in order."""
    import hashlib
    h = hashlib.sha256()
    for name in names:
        with open(os.path.join(ROOT, "mixture_experts_layer_22_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def captured_traffic(key: str):
    """DRAM bytes per launch of a kernel from a committed ncu capture
    (profiles/traffic.json, keyed "<workload> T=<T> <kernel>"), or None when
    no capture exists for it or its kernel sources have changed since."""
    try:
        with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
            t = json.load(f)
    except (OSError, ValueError):
        return None
    for cap in t.get("captures", []):
        if key in cap.get("kernels", {}):
            try:
                if source_sha256(cap["sources"]) != cap.get("source_sha256"):
                    return None
            except OSError:
                return None
            return cap["kernels"][key]
    return None


def static_hidden_scale(wl) -> float:
    """The oracle-calibrated static E4M3 scale of h (tests/golden), else 1."""
    if wl.adtype != syn.E4M3:
        return 1.0
    path = os.path.join(ROOT, "tests", "golden", f"{wl.name}_hidden_scale.json")
    with open(path) as f:
        return float(json.load(f)["a2"])


def moe_plan_is_normal(shape) -> bool:
    """The operand order the library picks for this shape (mirrors its rule:
    Swap-AB for T <= 128 or E4M3 weights with bf16 activations)."""
    if shape.variant:
        return shape.variant == 2
    return not (shape.T <= 128 or (shape.wdtype == 1 and shape.adtype == 0))


class DeviceLayer:
    """One workload's inputs on the device plus the calls bench.py times."""

    def __init__(self, wl, d, dev, weights=None):
        import torch
        import mixture_experts_layer_22_b200 as moe
        self.moe, self.torch = moe, torch
        self.wl, self.d, self.dev = wl, d, dev
        self.shape = moe.Shape.of(wl)
        self.esz = 2 if wl.wdtype == syn.BF16 else 1
        self.x = self.to_dev(d["x"])
        self.logits = torch.from_numpy(d["logits"]).to(dev)
        if weights is None:
            weights = (self.to_dev(d["w13"], u8=self.esz == 1), self.to_dev(d["w2"], u8=self.esz == 1),
                       torch.from_numpy(d["w13_scale"]).to(dev) if self.esz == 1 else None,
                       torch.from_numpy(d["w2_scale"]).to(dev) if self.esz == 1 else None)
        self.weights = weights
        self.w13, self.w2, self.s13, self.s2 = weights
        self.a1 = float(d["a1"])
        self.a2 = static_hidden_scale(wl)
        self.out = torch.empty((wl.T, wl.H), dtype=torch.bfloat16, device=dev)
        self.ws = moe.workspace(self.shape, device=dev)
        self.stream = torch.cuda.Stream(dev)      # graphs cannot be captured on the legacy stream
        self.graph = None

    def to_dev(self, a, u8=False):
        t = self.torch.from_numpy(np.ascontiguousarray(a).view(np.int16 if not u8 else np.uint8)).to(self.dev)
        return t if u8 else t.view(self.torch.bfloat16)

    def call(self, x=None, logits=None, out=None):
        self.moe.fused_forward(self.shape, self.x if x is None else x, self.logits if logits is None else logits,
                               self.w13, self.s13, self.w2, self.s2, self.a1, self.a2,
                               self.out if out is None else out, self.ws, self.stream)

    def capture(self):
        """One layer call as a CUDA graph (the library issues no host sync, so
        the whole kernel sequence is capturable)."""
        torch = self.torch
        with torch.cuda.stream(self.stream):
            self.call()
        torch.cuda.synchronize(self.dev)
        self.graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(self.graph, stream=self.stream):
            self.call()
        torch.cuda.synchronize(self.dev)

    def step(self, graph=True):
        # a graph replays on torch's current stream: make that the layer's stream
        with self.torch.cuda.stream(self.stream):
            if graph:
                self.graph.replay()
            else:
                self.call()

    def check_graph_matches_direct(self):
        """The replayed graph does the layer's work: its output equals a direct
        call's, bit for bit."""
        torch = self.torch
        self.out.fill_(0)
        self.step(True)
        torch.cuda.synchronize(self.dev)
        g = self.out.clone()
        self.out.fill_(0)
        self.call()
        torch.cuda.synchronize(self.dev)
        if not torch.equal(g.view(torch.int16), self.out.view(torch.int16)):
            raise SystemExit(f"{self.wl.name} T={self.wl.T}: graph replay output differs from a direct call")

    def routing_facts(self):
        """Distinct active experts (routed with >= 1 row, plus shared) and
        permuted slots, from the library's own routing and alignment."""
        torch, moe, wl = self.torch, self.moe, self.wl
        E_t = wl.E + wl.n_shared
        ids = torch.empty((wl.T, wl.k), dtype=torch.int32, device=self.dev)
        wts = torch.empty((wl.T, wl.k), dtype=torch.float32, device=self.dev)
        counts = torch.empty(E_t, dtype=torch.int32, device=self.dev)
        offsets = torch.empty(E_t + 1, dtype=torch.int32, device=self.dev)
        rows = torch.empty(moe.max_rows(self.shape), dtype=torch.int32, device=self.dev)
        inv = torch.empty(wl.T * wl.k, dtype=torch.int32, device=self.dev)
        moe.route_topk(self.shape, self.logits, ids, wts, self.stream)
        moe.align_permute(self.shape, ids, counts, offsets, rows, inv, self.ws, self.stream)
        torch.cuda.synchronize(self.dev)
        self.rows, self.offsets = rows, offsets
        return int((counts.cpu() > 0).sum()), int(offsets[-1].item())

    def time_gemms(self, steps):
        """Mean device time of each grouped GEMM call alone (with E4M3 weights
        and bf16 activations a call is the hi/lo split kernel plus the GEMM)."""
        torch, moe, wl = self.torch, self.moe, self.wl
        mr = moe.max_rows(self.shape)
        xp = torch.empty((mr, wl.H * (1 if wl.adtype else 2)), dtype=torch.uint8, device=self.dev)
        hb = torch.empty((mr, wl.I * (1 if wl.adtype else 2)), dtype=torch.uint8, device=self.dev)
        yb = torch.empty((mr, wl.H), dtype=torch.float32, device=self.dev)
        st = self.stream
        moe.gather(self.shape, self.x, self.rows, self.offsets, self.a1, xp, st)
        ev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(steps)]
        for i in range(steps + 1):
            e = ev[i - 1] if i > 0 else None
            if e:
                e[0].record(st)
            moe.grouped_gemm_swiglu(self.shape, xp, self.w13, self.s13, self.a1, self.a2, self.offsets, hb,
                                    self.ws, st)
            if e:
                e[1].record(st)
                e[2].record(st)
            moe.grouped_gemm_down(self.shape, hb, self.w2, self.s2, self.a2, self.offsets, yb, self.ws, st)
            if e:
                e[3].record(st)
        torch.cuda.synchronize(self.dev)
        t1 = statistics.mean(e[0].elapsed_time(e[1]) for e in ev)
        t2 = statistics.mean(e[2].elapsed_time(e[3]) for e in ev)
        del xp, hb, yb
        return t1, t2

    def host_us_per_call(self, n=50):
        """Host time to enqueue one direct moe_fused_forward (binding + C ABI +
        launches), the cost graph replay removes."""
        torch = self.torch
        torch.cuda.synchronize(self.dev)
        t0 = time.perf_counter()
        for _ in range(n):
            self.call()
        t1 = time.perf_counter()
        torch.cuda.synchronize(self.dev)
        return 1e6 * (t1 - t0) / n


class L2Flush:
    """Empties L2 between timed steps, outside the timed intervals: a 256 MB
    buffer (twice L2) is written, which evicts the step's data, and then, with
    `clean`, a second 256 MB buffer is read.  The read makes L2 write back the
    first buffer's dirty lines before the timed step starts; without it the
    step would begin by writing back up to 126 MB that are not its own."""

    MB = 256

    def __init__(self, torch, dev):
        n = self.MB * 2 ** 20 // 4
        self.torch = torch
        self.w = torch.empty(n, dtype=torch.float32, device=dev)
        self.r = torch.zeros(n, dtype=torch.float32, device=dev)
        self.s = torch.empty((), dtype=torch.float32, device=dev)

    def __call__(self, stream, clean=True):
        with self.torch.cuda.stream(stream):
            self.w.add_(1)
            if clean:
                self.torch.sum(self.r, dim=0, out=self.s)

    def describe(self, clean=True):
        return (f"flushed between timed steps: {self.MB} MB written" +
                (f", then {self.MB} MB read (no dirty lines left in L2)" if clean else " (L2 left dirty)"))


def time_steps(L, steps, graph, flush=None, clean=True):
    """Device milliseconds of `steps` layer steps on L's stream.  With `flush`
    (an L2Flush) each step is timed alone and L2 is emptied between steps,
    outside the timed intervals."""
    torch = L.torch
    st = L.stream
    if flush is None:
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(st)
        for _ in range(steps):
            L.step(graph)
        e1.record(st)
        torch.cuda.synchronize(L.dev)
        return e0.elapsed_time(e1)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    for a, b in ev:
        flush(st, clean)
        a.record(st)
        L.step(graph)
        b.record(st)
    torch.cuda.synchronize(L.dev)
    return sum(a.elapsed_time(b) for a, b in ev)


def time_e2e(L, steps, warmup, graph):
    """Tokens/s end to end through the C ABI with host buffers: every step
    copies its x and logits from pinned host memory, runs the layer and copies
    out back to pinned host memory, and the host reads every step's result.
    Device inputs and outputs are double-buffered so that step i+1's H2D and
    step i-1's D2H (each on its own copy stream) overlap step i's layer."""
    torch, wl, dev = L.torch, L.wl, L.dev
    nbuf = 2
    hx = torch.from_numpy(L.d["x"].view(np.int16)).view(torch.bfloat16).pin_memory()
    hl = torch.from_numpy(L.d["logits"]).pin_memory()
    ho = [torch.empty((wl.T, wl.H), dtype=torch.bfloat16).pin_memory() for _ in range(nbuf)]
    dx = [torch.empty_like(L.x) for _ in range(nbuf)]
    dl = [torch.empty_like(L.logits) for _ in range(nbuf)]
    dout = [torch.empty_like(L.out) for _ in range(nbuf)]
    graphs = [None] * nbuf
    if graph:
        torch.cuda.synchronize(dev)
        for b in range(nbuf):
            with torch.cuda.stream(L.stream):
                L.call(dx[b], dl[b], dout[b])
            torch.cuda.synchronize(dev)
            graphs[b] = torch.cuda.CUDAGraph()
            with torch.cuda.graph(graphs[b], stream=L.stream):
                L.call(dx[b], dl[b], dout[b])
        torch.cuda.synchronize(dev)
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev_in = [torch.cuda.Event() for _ in range(nbuf)]
    ev_layer = [torch.cuda.Event() for _ in range(nbuf)]
    ev_out = [torch.cuda.Event() for _ in range(nbuf)]

    def enqueue(i):
        b = i % nbuf
        s_in.wait_event(ev_layer[b])          # the layer of step i-2 is done reading dx[b], dl[b]
        with torch.cuda.stream(s_in):
            dx[b].copy_(hx, non_blocking=True)
            dl[b].copy_(hl, non_blocking=True)
        ev_in[b].record(s_in)
        L.stream.wait_event(ev_in[b])
        L.stream.wait_event(ev_out[b])        # step i-2's D2H is done reading dout[b]
        with torch.cuda.stream(L.stream):
            if graphs[b] is not None:
                graphs[b].replay()
            else:
                L.call(dx[b], dl[b], dout[b])
        ev_layer[b].record(L.stream)
        s_out.wait_event(ev_layer[b])
        with torch.cuda.stream(s_out):
            ho[b].copy_(dout[b], non_blocking=True)
        ev_out[b].record(s_out)

    def run(n):
        for i in range(n):
            enqueue(i)
            if i > 0:
                ev_out[(i - 1) % nbuf].synchronize()   # the host reads step i-1's result
        ev_out[(n - 1) % nbuf].synchronize()

    run(warmup)
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(s_in)
    run(steps)
    e1.record(s_out)
    torch.cuda.synchronize(dev)
    ms = e0.elapsed_time(e1)
    return ms, {"h2d_bytes_per_step": int(hx.numel() * 2 + hl.numel() * 4), "d2h_bytes_per_step": int(ho[0].numel() * 2)}


def measure_workload(wl, d, dev, args, weights=None, full=False, flush=None):
    """Layer throughput, the two GEMMs against their rooflines, and the end-to-
    end rate, for one workload (graph replay; with `full`, also direct calls)."""
    torch = __import__("torch")
    L = DeviceLayer(wl, d, dev, weights)
    active, slots = L.routing_facts()
    L.capture()
    for _ in range(args.warmup):
        L.step(True)
    torch.cuda.synchronize(dev)
    L.call()
    torch.cuda.synchronize(dev)
    launches = L.moe.last_launch_count()
    st = L.moe.device_status(L.ws, L.stream)
    if st != 0:
        raise SystemExit(f"{wl.name} T={wl.T}: device status after warm-up: {L.moe.status_string(st)}")
    L.check_graph_matches_direct()
    # flush L2 between steps when the weights of one step would stay in it
    wbytes = active * weight_bytes_per_expert(wl)
    use_flush = flush if (flush is not None and wbytes < 4 * L2_BYTES) else None
    ms = time_steps(L, args.steps, True, use_flush)
    # the same steps after a write-only flush, whose dirty lines the step
    # itself must write back (for comparison with the usual practice)
    ms_dirty = time_steps(L, args.steps, True, use_flush, clean=False) if use_flush is not None else None
    t_g1, t_g2 = L.time_gemms(args.steps)
    e2e_ms, e2e_bytes = time_e2e(L, args.steps, args.warmup, graph=True)
    res = {"T": wl.T, "ms_per_step": ms / args.steps, "tokens_per_s": wl.T * args.steps / (ms / 1e3),
           "active_experts": active, "launches_per_step": launches,
           "l2": use_flush.describe() if use_flush is not None else
                 "not flushed: each step streams the active experts' weights (> 4x L2)",
           "e2e": {"value": wl.T * args.steps / (e2e_ms / 1e3), "unit": UNIT, **e2e_bytes,
                   "launch": "CUDA graph replay"}}
    if ms_dirty is not None:
        res["ms_per_step_after_write_only_flush"] = ms_dirty / args.steps
    if full:
        ms_direct = time_steps(L, args.steps, False, use_flush)
        e2e_d_ms, _ = time_e2e(L, args.steps, args.warmup, graph=False)
        res["direct"] = {"ms_per_step": ms_direct / args.steps, "host_us_per_call": L.host_us_per_call(),
                         "e2e_tokens_per_s": wl.T * args.steps / (e2e_d_ms / 1e3)}
    hbm_peak, tc_burst, _, peak_kind = measured_peaks()
    esz = L.esz
    aesz = 1 if wl.adtype else 2
    real_rows = wl.T * wl.k + wl.n_shared * wl.T
    g1_bytes = active * 2 * wl.H * wl.I * esz + slots * wl.H * aesz + slots * wl.I * aesz
    g2_bytes = active * wl.H * wl.I * esz + slots * wl.I * aesz + slots * wl.H * 4
    g1_flops = 2.0 * 2 * wl.H * wl.I * real_rows
    g2_flops = 2.0 * wl.H * wl.I * real_rows
    layer_bytes = wbytes + wl.T * wl.H * 2 * 2 + wl.T * wl.E * 4
    layer_flops = g1_flops + g2_flops
    tc_peak = tc_burst * (2.0 if wl.adtype == syn.E4M3 else 1.0)
    decode = not moe_plan_is_normal(L.shape)
    res["layer"] = {"gbs": layer_bytes / (res["ms_per_step"] * 1e-3) / 1e9,
                    "tflops": layer_flops / (res["ms_per_step"] * 1e-3) / 1e12}
    if decode:
        res["layer"]["frac"] = res["layer"]["gbs"] / hbm_peak
        g1 = {"bound": "hbm", "achieved": g1_bytes / (t_g1 * 1e-3) / 1e9, "peak": hbm_peak, "unit": "GB/s",
              "algorithmic_bytes": g1_bytes}
        g2 = {"bound": "hbm", "achieved": g2_bytes / (t_g2 * 1e-3) / 1e9, "peak": hbm_peak, "unit": "GB/s",
              "algorithmic_bytes": g2_bytes}
    else:
        res["layer"]["frac"] = res["layer"]["tflops"] / tc_peak
        g1 = {"bound": "tensor", "achieved": g1_flops / (t_g1 * 1e-3) / 1e12, "peak": tc_peak,
              "unit": "TFLOP/s", "algorithmic_flops": g1_flops}
        g2 = {"bound": "tensor", "achieved": g2_flops / (t_g2 * 1e-3) / 1e12, "peak": tc_peak,
              "unit": "TFLOP/s", "algorithmic_flops": g2_flops}
    for g, t in ((g1, t_g1), (g2, t_g2)):
        g["frac"] = g["achieved"] / g["peak"]
        g["ms"] = t
        g["peak_kind"] = peak_kind
    g1["kernel"] = "grouped_gemm gate/up + SwiGLU" + (" (+ hi/lo split)" if (wl.wdtype, wl.adtype) == (1, 0) else "")
    g2["kernel"] = "grouped_gemm down" + (" (+ hi/lo split)" if (wl.wdtype, wl.adtype) == (1, 0) else "")
    g1["traffic"] = captured_traffic(f"{wl.name} T={wl.T} gemm1")
    g2["traffic"] = captured_traffic(f"{wl.name} T={wl.T} gemm2")
    res["gemm1"], res["gemm2"] = g1, g2
    return res, L


def ours_main(args, wl):
    import torch
    import torch.distributed as dist

    world, rank, local = dist_env()
    if world > 1:
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", init_method="env://",
                                timeout=__import__("datetime").timedelta(seconds=120))
    dev = torch.device("cuda", local if world > 1 else 0)
    torch.cuda.set_device(dev)
    d = syn.make_inputs(wl)
    L = DeviceLayer(wl, d, dev)
    active, slots = L.routing_facts()
    L.capture()
    for _ in range(args.warmup):
        L.step(True)
    torch.cuda.synchronize(dev)
    L.call()
    torch.cuda.synchronize(dev)
    launches_per_step = L.moe.last_launch_count()
    st = L.moe.device_status(L.ws, L.stream)
    if st != 0:
        raise SystemExit(f"device status after warm-up: {L.moe.status_string(st)}")
    L.check_graph_matches_direct()

    # clocks: sampled through a soak of about half a second of steps and the
    # timed region right after it
    clocks = ClockSampler(dev.index)
    clocks.start()
    time.sleep(0.2)
    t_end = time.perf_counter() + 0.5
    while time.perf_counter() < t_end:
        for _ in range(20):
            L.step(True)
        torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    ms_local = time_steps(L, args.steps, True)
    if world > 1:
        dist.barrier()
    clk = clocks.stop()
    ms, value = aggregate_over_ranks(ms_local, wl.T, args.steps, dist if world > 1 else None)
    ms_per_step = ms / args.steps

    # the same measurements the sweep reports, for the headline workload
    weights = L.weights
    del L
    torch.cuda.empty_cache()
    detail, L = measure_workload(wl, d, dev, args, weights=weights, full=True)
    e2e_ms, e2e_bytes = time_e2e(L, args.steps, args.warmup, graph=True)
    ems, e2e_val = aggregate_over_ranks(e2e_ms, wl.T, args.steps, dist if world > 1 else None)

    # the optional router step (logits = x . W_g^T and top-k in one launch)
    router = None
    if wl.logits == "router":
        moe = L.moe
        wg = L.to_dev(syn.router_weight(wl))
        rl = torch.empty((wl.T, wl.E), dtype=torch.float32, device=dev)
        rids = torch.empty((wl.T, wl.k), dtype=torch.int32, device=dev)
        rw = torch.empty((wl.T, wl.k), dtype=torch.float32, device=dev)
        moe.router_topk(L.shape, L.x, wg, rl, rids, rw, L.ws, L.stream)
        r0, r1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        r0.record(L.stream)
        for _ in range(args.steps):
            moe.router_topk(L.shape, L.x, wg, rl, rids, rw, L.ws, L.stream)
        r1.record(L.stream)
        torch.cuda.synchronize(dev)
        router = {"kernel": "router_topk (x . W_g^T in fp64, fixed order, + top-k)",
                  "ms": r0.elapsed_time(r1) / args.steps,
                  "bytes": wl.T * wl.H * 2 + wl.E * wl.H * 2 + wl.T * wl.E * 4 + wl.T * wl.k * 8}
    roof = dict(detail["gemm1"])
    roof["down"] = detail["gemm2"]
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None,
        "dtype": {(0, 0): "bf16", (1, 1): "e4m3", (1, 0): "e4m3w-bf16a"}[(wl.wdtype, wl.adtype)],
        "data": "synthetic",
        "config": config_of(wl, f"replicas x{world}" if world > 1 else "1 GPU",
                            "CUDA graph of one moe_fused_forward per step",
                            "not flushed: each step streams the active experts' weights (GBs, > L2)"),
        "hbm_gbs": detail["layer"]["gbs"] * detail["ms_per_step"] / ms_per_step,
        "layer_frac_of_hbm": detail["layer"]["gbs"] * detail["ms_per_step"] / ms_per_step / roof["peak"]
        if roof["bound"] == "hbm" else None,
        "active_experts": active,
        "roofline": roof,
        "e2e": {"value": e2e_val, "unit": UNIT, **e2e_bytes,
                "overlap": "double-buffered: H2D and D2H on their own copy streams overlap the layer of "
                           "the neighbouring step; the host reads every step's result; graph replay"},
        "direct_calls": detail["direct"],
        "gpu_launches": launches_per_step * args.steps,
        "router": router,
        "clocks": clk,
    }
    del L
    torch.cuda.empty_cache()
    if world == 1 and not args.no_sweep:
        line["per_workload"] = sweep(args, dev, d, weights, wl)
    if rank == 0 and world == 1 and not args.no_cpu:
        r, cores, sample = cpu_oracle_rate(wl, d, budget_s=args.ref_budget, a2=static_hidden_scale(wl))
        line["cpu_baseline"] = {"value": r, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": sample}
    if world > 1:
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


ROPE_SWEEP = [("rope_mixtral", 8192), ("rope_mixtral", 64), ("rope_dsv3", 8192)]


def measure_rope(rw, dev, args, flush):
    """The attention-side step (inverse rotary + per-head E4M3, one launch):
    tokens/s and HBM GB/s of its algorithmic bytes (x in, codes and scales
    out, positions and the table rows it reads), each step timed alone with L2
    emptied in between (its data fits in L2)."""
    import torch
    import mixture_experts_layer_22_b200 as moe
    d = syn.rope_inputs(rw)
    s = moe.RopeShape.of(rw)
    x = torch.from_numpy(d["x"].view(np.int16)).to(dev).view(torch.bfloat16)
    pos = torch.from_numpy(d["positions"]).to(dev)
    cs = torch.from_numpy(d["cos_sin"]).to(dev)
    q = torch.empty((rw.T, rw.n_heads, rw.head_dim), dtype=torch.uint8, device=dev)
    sc = torch.empty((rw.T, rw.n_heads), dtype=torch.float32, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    st = torch.cuda.Stream(dev)
    for _ in range(args.warmup):
        moe.inv_rope_quant(s, x, pos, cs, q, sc, status, st)
    torch.cuda.synchronize(dev)
    if int(status.item()) != 0:
        raise SystemExit(f"{rw.name}: device status {int(status.item())}")
    def timed(clean):
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(args.steps)]
        for a, b in ev:
            flush(st, clean)
            a.record(st)
            moe.inv_rope_quant(s, x, pos, cs, q, sc, status, st)
            b.record(st)
        torch.cuda.synchronize(dev)
        return sum(a.elapsed_time(b) for a, b in ev) / args.steps

    ms = timed(True)
    ms_dirty = timed(False)
    heads = rw.T * rw.n_heads
    nbytes = heads * rw.head_dim * 3 + heads * 4 + rw.T * 4 + rw.T * rw.rot_dim * 4
    hbm_peak = measured_peaks()[0]
    return {"T": rw.T, "n_heads": rw.n_heads, "head_dim": rw.head_dim, "rot_dim": rw.rot_dim,
            "interleaved": rw.interleaved, "ms_per_step": ms, "tokens_per_s": rw.T / (ms * 1e-3),
            "roofline": {"bound": "hbm", "achieved": nbytes / (ms * 1e-3) / 1e9, "peak": hbm_peak, "unit": "GB/s",
                         "frac": nbytes / (ms * 1e-3) / 1e9 / hbm_peak, "algorithmic_bytes": nbytes,
                         "traffic": captured_traffic(f"{rw.name} T={rw.T} rope")},
            "ms_per_step_after_write_only_flush": ms_dirty,
            "l2": flush.describe(), "launches_per_step": 1}


def rope_main(args):
    """The inverse-rotary + per-head E4M3 step alone (one GPU): a JSON line
    with its tokens/s and HBM roofline."""
    import torch
    rw = syn.ROPE_WORKLOADS[args.workload]
    if args.T is not None:
        rw = rw.with_T(args.T)
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    flush = L2Flush(torch, dev)
    r = measure_rope(rw, dev, args, flush)
    line = {"metric": "inverse-RoPE + per-head E4M3 tokens/s", "value": r["tokens_per_s"], "unit": UNIT,
            "n_gpus": 1, "steps": args.steps, "warmup": args.warmup, "ms_per_step": r["ms_per_step"],
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16-in e4m3-out",
            "data": "synthetic", "config": {"workload": f"{rw.name}: T={rw.T} heads={rw.n_heads} head_dim={rw.head_dim} "
                                                        f"rot_dim={rw.rot_dim} {'interleaved' if rw.interleaved else 'neox'}",
                                            "l2": r["l2"]},
            "roofline": r["roofline"], "gpu_launches": args.steps}
    print(json.dumps(line), flush=True)
    return 0


def sweep(args, dev, d_head, weights_head, wl_head):
    """Every configuration besides the headline, measured the same way."""
    import torch
    flush = L2Flush(torch, dev)
    out = {}
    cache = {"key": (wl_head.name, wl_head.wdtype, wl_head.adtype), "weights": weights_head,
             "host": {k: d_head[k] for k in ("w13", "w13_scale", "w2", "w2_scale")}}
    clocks = ClockSampler(dev.index)
    clocks.start()
    for name, T in SWEEP:
        wl = workload_of(name, T)
        if (wl.name, wl.T) == (wl_head.name, wl_head.T):
            continue
        key = (wl.name, wl.wdtype, wl.adtype)
        d = syn.make_inputs(wl, weights=False)
        same_w = cache["key"][0].startswith("dsv3") and wl.name.startswith("dsv3")
        if key != cache["key"] and not same_w:
            cache["weights"] = None
            torch.cuda.empty_cache()
            dw = syn.make_inputs(wl)
            cache["host"] = {k: dw[k] for k in ("w13", "w13_scale", "w2", "w2_scale")}
            cache["key"] = key
        d.update(cache["host"])
        res, L = measure_workload(wl, d, dev, args, weights=cache["weights"],
                                  full=wl.T in (1, 64) and wl.name == "mixtral_decode", flush=flush)
        cache["weights"] = L.weights
        out[f"{wl.name} T={wl.T}"] = res
        del L
    cache["weights"] = None
    torch.cuda.empty_cache()
    for name, T in ROPE_SWEEP:
        rw = syn.ROPE_WORKLOADS[name].with_T(T)
        out[f"{rw.name} T={rw.T}"] = measure_rope(rw, dev, args, flush)
    out["_clocks"] = clocks.stop()
    return out


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=HEADLINE[0], choices=sorted(syn.WORKLOADS) + sorted(syn.ROPE_WORKLOADS),
                    help="a layer workload, or an attention-side rope_* workload (that step alone)")
    ap.add_argument("--T", type=int, default=None)
    ap.add_argument("--E", type=int, default=None, help="override the routed expert count (small profiling cases)")
    ap.add_argument("--ref-budget", type=float, default=15.0, help="seconds of host time per oracle sample")
    ap.add_argument("--no-cpu", action="store_true", help="skip the cpu_baseline leg")
    ap.add_argument("--no-sweep", action="store_true", help="headline workload only")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.workload in syn.ROPE_WORKLOADS:
        return rope_main(args)
    wl = syn.WORKLOADS[args.workload]
    T = args.T if args.T is not None else (HEADLINE[1] if args.workload == HEADLINE[0] else wl.T)
    wl = wl.with_T(T)
    if args.E is not None:
        wl = dataclasses.replace(wl, E=args.E, name=f"{wl.name}_E{args.E}")
        args.no_sweep = True
    if args.impl == "reference":
        return reference_main(args, wl)
    return ours_main(args, wl)


if __name__ == "__main__":
    sys.exit(main())
