#!/usr/bin/env python
"""Benchmark of the activation-sparse gated FFN on B200.

One step = one sparse forward (gate -> select -> up -> down) over one batch
of the workload's tokens.  Default workload: Llama-7B-shaped FFN decode
(d=4096, d_ff=11008, one token, dense gate, tau for 90 % sparsity), the shape
of the headline metric.  Prints one JSON line (rank 0).

Timing: W warm-up steps, then every captured graph is replayed once untimed
(its first launch uploads it), then at least 50 ms of untimed replays run
straight into the timed region, so the timed steps start in steady state.
Exactly K steps are then replayed from CUDA graphs on one stream, bracketed by
a barrier and device synchronisation, timed with CUDA events; the max over
ranks is taken.  Consecutive steps use different weight replicas whose total
footprint exceeds 3x the L2, so no step finds its weights in L2.  A second
series times each replay of the graph on its own (median, p10, p90 per step),
and a third times the same steps with one weight copy reused every step
(weights warm in L2; labelled as such, not the headline).  Multi-GPU runs are
independent replicas (weak scaling).

Also reported: the same metric end to end through sffn_forward_host (host
buffers, copies in the timed region), the library's dense FFN on the same
weights, the roofline of the dominant kernel (from stage events around each
kernel in a second pass over the same steps), SM clocks during the run, and the
CPU oracle's time per token on a bounded sample (rank 0 only).

`--impl reference` times the CPU oracle as it stands (the reference arm).
"""
from __future__ import annotations

import argparse
import hashlib
import glob
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

import workloads  # noqa: E402

METRIC = "sparse-FFN us/token at 90% sparsity (HBM GB/s in roofline) vs dense FFN"
UNIT = "us/token"
KERNEL_SOURCES = os.path.join(ROOT, "activation_sparse_gated_gemv_b200", "csrc")


def parse():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20000)
    ap.add_argument("--warmup", type=int, default=500)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="llama7b-decode",
                    choices=["llama7b-decode", "lopa7b", "moc-topk", "llama70b", "llama70b-lopa", "heavy7b", "tiny"])
    ap.add_argument("--sparsity", type=float, default=0.9)
    ap.add_argument("--tokens", type=int, default=0, help="batch size (0: the workload's)")
    ap.add_argument("--top-p", type=float, default=0.0,
                    help="select by top-p with this softmax-mass budget instead of the workload's rule")
    ap.add_argument("--graph-steps", type=int, default=256, help="steps per captured graph")
    ap.add_argument("--e2e-steps", type=int, default=2000)
    ap.add_argument("--cpu-seconds", type=float, default=12.0, help="CPU oracle sample budget")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-dense", action="store_true")
    ap.add_argument("--dense-step", action="store_true",
                    help="time the library's dense FFN as the step (the comparator on its own, e.g. for ncu)")
    ap.add_argument("--no-hot", action="store_true", help="heavy7b: run without the heavy-hitter set")
    ap.add_argument("--replicas", type=int, default=0,
                    help="weight copies rotated across steps (0: enough to exceed 3x the L2); 1 keeps ncu "
                         "captures small (ncu flushes the caches between its passes anyway)")
    ap.add_argument("--json-out", default="")
    return ap.parse_args()


def make_workload(a) -> workloads.Workload:
    if a.workload == "llama7b-decode":
        wl = workloads.llama7b_decode(a.sparsity)
    elif a.workload == "lopa7b":
        wl = workloads.lopa7b(a.sparsity)
    elif a.workload == "moc-topk":
        wl = workloads.moc_topk()
    elif a.workload == "llama70b":
        wl = workloads.llama70b(1, "dense", a.sparsity)
    elif a.workload == "llama70b-lopa":
        wl = workloads.llama70b(1, "lopa", a.sparsity)
    elif a.workload == "heavy7b":
        wl = workloads.heavy7b()
    else:
        wl = workloads.tiny()
    if a.tokens:
        wl.n = a.tokens
    if a.top_p:
        wl.select, wl.p = "topp", a.top_p
    return wl


def bytes_per_elem(dtype):
    return 2 if dtype == "bf16" else 4


def algorithmic_bytes(wl, union, gate_kernel_only=False):
    """Gate weights + the union's W_up and W_down rows + x in and y out
    (gate kernel: gate weights + W_up rows + x)."""
    w = bytes_per_elem(wl.dtype)
    gate = (wl.r * (wl.d + wl.d_ff) if wl.gate == "lopa" else wl.d * wl.d_ff) * w
    if gate_kernel_only:
        return gate + union * wl.d * w + wl.n * wl.d * w
    return gate + 2 * union * wl.d * w + 2 * wl.n * wl.d * w


def dense_bytes(wl):
    w = bytes_per_elem(wl.dtype)
    return 3 * wl.d * wl.d_ff * w + 2 * wl.n * wl.d * w


def select_args(wl):
    if wl.select == "threshold":
        return dict(select="threshold", tau=wl.tau)
    if wl.select == "topp":
        return dict(select="topp", p=wl.p)
    return dict(select="topk", k=wl.k)


def code_only(src: str) -> str:
    """C/C++/CUDA source without its comments and blank space, so that a change
    to comments alone does not count as a change of the kernels (string and
    character literals are kept as they are)."""
    out, i, n = [], 0, len(src)
    while i < n:
        c = src[i]
        if src.startswith("//", i):
            j = src.find("\n", i)
            i = n if j < 0 else j
        elif src.startswith("/*", i):
            j = src.find("*/", i + 2)
            i = n if j < 0 else j + 2
            out.append(" ")
        elif c in "\"'":
            j = i + 1
            while j < n and src[j] != c:
                j += 2 if src[j] == "\\" else 1
            out.append(src[i:j + 1])
            i = j + 1
        else:
            out.append(c)
            i += 1
    return " ".join("".join(out).split())


# The device sources each kernel family is built from (plus the shared
# header); the launch geometry of the decode and tensor-core kernels is
# computed in their own files.
KERNEL_FAMILY_FILES = {
    "decode": ["fused.cu", "dot.cuh"],
    "tc": ["tc.cu"],
    "topk": ["topk.cu"],
    "gate": ["gate.cu", "dot.cuh"],
    "down": ["down.cu"],
}
COMMON_KERNEL_FILES = ["common.cuh"]


def kernel_family(kernel: str) -> str:
    if kernel.startswith("decode"):
        return "decode"
    if kernel.startswith("tc_") or kernel == "union_list":
        return "tc"
    if kernel in ("topk", "topp"):
        return "topk"
    if kernel == "down":
        return "down"
    return "gate"


def kernel_hash(family: str) -> str:
    """Hash of the code (comments and layout left out) of one kernel family's
    sources."""
    h = hashlib.sha256()
    for name in sorted(set(KERNEL_FAMILY_FILES[family] + COMMON_KERNEL_FILES)):
        with open(os.path.join(KERNEL_SOURCES, name), encoding="utf-8") as f:
            h.update(name.encode() + code_only(f.read()).encode())
    return h.hexdigest()[:16]


def traffic_for(kernel: str, workload: str, tokens: int):
    """Per-launch DRAM bytes from a committed ncu capture, if it was taken on
    the current code of the kernel's sources (keyed by workload and token
    count)."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            data = json.load(f)
    except (OSError, ValueError):
        return None
    ent = (data.get(f"{workload}:n{tokens}") or data.get(workload, {}) if tokens > 1 else
           data.get(workload, {})).get(kernel)
    if not ent or ent.get("kernel_hash") != kernel_hash(kernel_family(kernel)):
        return None
    return ent.get("dram_bytes_per_launch")


def measured_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return json.load(f), "measured"
    except (OSError, ValueError):
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0}, "fallback"


class ClockSampler:
    """nvidia-smi SM clocks and throttle reasons every 100 ms."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.path = None
        self.t0 = self.t1 = None

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None

    def mark(self, which):
        setattr(self, which, time.time())

    def stop(self):
        if not self.proc:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"], "samples": 0}
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = set()
        sm = []
        for r in rows:
            try:
                sm.append(float(r[1]))
            except ValueError:
                pass
            for i, nm in enumerate(names):
                if r[5 + i].lower().startswith("active"):
                    reasons.add(nm)
        try:
            smax = float(rows[-1][2])
        except ValueError:
            smax = None
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": smax,
                "reasons": sorted(reasons), "samples": len(rows)}


def init_dist(a):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    elif torch.cuda.is_available():
        torch.cuda.set_device(local)
    return world, rank, local


def reduce_max(v: float, world: int) -> float:
    if world == 1:
        return v
    import torch.distributed as dist
    t = torch.tensor([v], dtype=torch.float64, device="cuda" if torch.cuda.is_available() else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


# ---------------------------------------------------------------------------
# CPU oracle (the reported baseline / the reference arm)

def cpu_oracle_run(wl, weights, budget_s: float, max_tokens: int = 4096):
    """Time the oracle's sparse path token by token for about budget_s."""
    import oracle
    oracle.build()
    done, t_total = 0, 0.0
    tag = 0
    while t_total < budget_s and done < max_tokens:
        x = wl.x(tag=f"cpu{tag}")
        t0 = time.perf_counter()
        oracle.forward(x, weights, wl.gate, wl.select, tau=wl.tau or 0.0, k=wl.k, p=wl.p)
        t_total += time.perf_counter() - t0
        done += x.shape[0]
        tag += 1
    return {"value": t_total / done * 1e6, "unit": UNIT, "cores": oracle.num_threads(), "kind": "oracle",
            "sample": f"{done} tokens of {wl.describe()}, fp64 oracle sparse path (gate, select, up, "
                      f"down) in {t_total:.1f} s with {oracle.num_threads()} OpenMP threads"}


def run_reference(a, world, rank):
    if rank != 0:
        return
    wl = make_workload(a)
    weights = wl.weights()
    budget = max(5.0, min(60.0, a.cpu_seconds))
    t_all0 = time.perf_counter()
    per_step = []
    import oracle
    oracle.build()
    steps = max(1, a.steps)
    # each step is a bounded sample of the workload: one batch of tokens
    steps = min(steps, max(1, int(budget / 0.05)))
    for i in range(a.warmup and 1 or 0):
        oracle.forward(wl.x(tag="refw"), weights, wl.gate, wl.select, tau=wl.tau or 0.0, k=wl.k, p=wl.p)
    for i in range(steps):
        x = wl.x(tag=f"ref{i}")
        t0 = time.perf_counter()
        oracle.forward(x, weights, wl.gate, wl.select, tau=wl.tau or 0.0, k=wl.k, p=wl.p)
        per_step.append(time.perf_counter() - t0)
        if time.perf_counter() - t_all0 > budget:
            break
    ms = statistics.mean(per_step) * 1e3
    value = ms * 1e3 / wl.n
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": a.gpus,
        "steps": len(per_step), "warmup": a.warmup, "ms_per_step": ms, "higher_is_better": False,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": wl.describe(), "tokens_per_step": wl.n},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": oracle.num_threads(), "kind": "oracle",
                         "sample": f"{len(per_step)} steps of {wl.n} token(s) each, fp64 oracle sparse path"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------
# GPU arm

def main():
    a = parse()
    world, rank, local = init_dist(a)
    if a.impl == "reference":
        run_reference(a, world, rank)
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
        return

    from activation_sparse_gated_gemv_b200 import build
    build.build()
    import activation_sparse_gated_gemv_b200 as sffn

    wl = make_workload(a)
    dev = torch.device("cuda", local)
    props = torch.cuda.get_device_properties(dev)
    l2 = getattr(props, "L2_cache_size", 126 * 2**20) or 126 * 2**20
    sel = select_args(wl)
    weights = wl.weights()
    dense_gate_w = None
    if wl.gate == "lopa":
        # the uncast comparator: a dense gate holding A B rounded to the storage type
        prod = (weights["A"].to(dev, torch.float32) @ weights["B"].to(dev, torch.float32))
        dense_gate_w = prod.to(workloads.DTYPES[wl.dtype]).contiguous()

    # token pool: P batches, different per rank
    P = 8
    xs = [wl.x(tag=f"r{rank}p{i}").to(dev) for i in range(P)]
    ys = [torch.empty((wl.n, wl.d), dtype=xs[0].dtype, device=dev) for _ in range(P)]

    # one probe handle to measure the active union for each pool batch
    probe = sffn.SparseFFN(wl.d, wl.d_ff, wl.r, wl.n, wl.dtype, device=local)
    probe.set_weights(**weights)
    hot = wl.hot().numpy() if wl.hot_frac > 0.0 and not a.no_hot else None
    if hot is not None:
        probe.set_hot(hot)
    unions = []
    for i in range(P):
        probe.forward(xs[i], gate=wl.gate, out=ys[i], **sel)
        unions.append(probe.active(wl.n)[1])
    probe.close()
    union = statistics.mean(unions)
    fwd_bytes = dense_bytes(wl) if a.dense_step else algorithmic_bytes(wl, union)
    R = max(2, math.ceil(3 * l2 / fwd_bytes))
    R = min(R, 64) if a.replicas <= 0 else a.replicas
    ffns = []
    for i in range(R):
        f = sffn.SparseFFN(wl.d, wl.d_ff, wl.r, wl.n, wl.dtype, device=local)
        f.set_weights(**weights)
        if hot is not None:
            f.set_hot(hot)
        ffns.append(f)

    stream = torch.cuda.Stream(dev)

    def step(i, dense=False):
        ffns[i % R].forward(xs[i % P], gate=wl.gate, out=ys[i % P], dense=dense or a.dense_step, stream=stream,
                            **sel)

    def capture(first, count, dense=False):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream, capture_error_mode="thread_local"):
            for i in range(first, first + count):
                step(i, dense)
        return g

    sampler = ClockSampler(local)
    sampler.start()                            # sampling from the warm-up on: no idle gap before the timing

    G = max(1, min(a.graph_steps, a.steps))
    G = max(R, G - G % R) if G >= R else G
    graphs = [capture(0, G)]
    rem = a.steps % G
    rem_graph = capture(0, rem) if rem else None

    # warm-up (untimed), then one untimed replay of each graph (the first
    # launch of a graph uploads it)
    with torch.cuda.stream(stream):
        for i in range(a.warmup):
            step(i)
        graphs[0].replay()
        if rem_graph is not None:
            rem_graph.replay()
    torch.cuda.synchronize()

    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    # pre-roll: untimed replays worth at least 50 ms of GPU time, queued
    # straight ahead of the timed region, so it starts with the GPU busy
    t_one = time.perf_counter()
    with torch.cuda.stream(stream):
        graphs[0].replay()
    torch.cuda.synchronize()
    t_one = time.perf_counter() - t_one
    pre_replays = max(2, min(5000, int(0.05 / max(t_one, 1e-6)) + 1))
    sampler.mark("t0")
    with torch.cuda.stream(stream):
        for _ in range(pre_replays):
            graphs[0].replay()
        ev0.record(stream)
        for _ in range(a.steps // G):
            graphs[0].replay()
        if rem_graph is not None:
            rem_graph.replay()
        ev1.record(stream)
    torch.cuda.synchronize()
    sampler.mark("t1")
    barrier(world)
    ms_total = reduce_max(ev0.elapsed_time(ev1), world)
    ms_per_step = ms_total / a.steps
    us_per_token = ms_total * 1e3 / (a.steps * wl.n * world)

    # -- spread: each replay of the G-step graph timed on its own, back to back
    M = 50
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(M + 1)]
    with torch.cuda.stream(stream):
        graphs[0].replay()
        evs[0].record(stream)
        for j in range(M):
            graphs[0].replay()
            evs[j + 1].record(stream)
    torch.cuda.synchronize()
    per_rep = sorted(evs[j].elapsed_time(evs[j + 1]) * 1e3 / (G * wl.n) for j in range(M))
    q = lambda f: per_rep[min(M - 1, int(round(f * (M - 1))))]
    spread = {"median": round(statistics.median(per_rep), 4), "p10": round(q(0.1), 4), "p90": round(q(0.9), 4),
              "unit": UNIT, "replays": M, "steps_per_replay": G,
              "how": "CUDA events between back-to-back replays of the timed graph, per-step mean of each replay"}

    # -- warm L2: the same steps with one weight copy reused every step
    gw = torch.cuda.CUDAGraph()
    with torch.cuda.graph(gw, stream=stream, capture_error_mode="thread_local"):
        for i in range(G):
            ffns[0].forward(xs[i % P], gate=wl.gate, out=ys[i % P], stream=stream, **sel)
    ew0, ew1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    Mw = max(1, min(20, 2000 // G))
    with torch.cuda.stream(stream):
        gw.replay()
        gw.replay()
        ew0.record(stream)
        for _ in range(Mw):
            gw.replay()
        ew1.record(stream)
    torch.cuda.synchronize()
    warm = {"value": round(ew0.elapsed_time(ew1) * 1e3 / (Mw * G * wl.n), 4), "unit": UNIT,
            "note": f"L2-warm: one weight copy reused by every step ({algorithmic_bytes(wl, union) / 1e6:.0f} MB "
                    f"touched per step, L2 {l2 / 2**20:.0f} MiB); not the headline"}
    del gw

    # -- second pass: stage events around each kernel, same steps, replayed
    #    from a graph (events become external record nodes between kernels)
    launches = ffns[0].last_launches()
    nev = launches + 1
    K2 = min(a.steps, 512)
    stage = []
    for j in range(K2):
        evs = [torch.cuda.Event(enable_timing=True) for _ in range(nev)]
        for e in evs:
            e.record(stream)
        stage.append(evs)
    torch.cuda.synchronize()
    gs = torch.cuda.CUDAGraph()
    with torch.cuda.graph(gs, stream=stream, capture_error_mode="thread_local"):
        for j in range(K2):
            ffns[j % R].set_stage_events(stage[j])
            step(j)
    for f in ffns:
        f.set_stage_events([])
    with torch.cuda.stream(stream):
        gs.replay()
    torch.cuda.synchronize()
    per_kernel = np.zeros(launches)
    for evs in stage:
        for i in range(launches):
            per_kernel[i] += evs[i].elapsed_time(evs[i + 1])
    per_kernel /= K2
    kernel_names = ffns[0].last_kernel_names()
    # launches of the same kernel (a batch above 128 tokens takes one
    # tensor-core pass per 128 tokens) are counted together
    names = [kernel_names[i] if i < len(kernel_names) else f"k{i}" for i in range(launches)]
    per_name = {}
    for i, nm in enumerate(names):
        per_name[nm] = per_name.get(nm, 0.0) + per_kernel[i]
    launch_count = {nm: names.count(nm) for nm in per_name}
    dom_name = max(per_name, key=per_name.get)
    peaks, peak_kind = measured_peaks()
    w = bytes_per_elem(wl.dtype)
    if dom_name == "decode_dense":
        dom_bytes = dense_bytes(wl)
    elif dom_name == "decode_fused":
        # everything (LoPA's stage 1 runs inside the same launch)
        dom_bytes = algorithmic_bytes(wl, union) - (
            wl.d * wl.r * bytes_per_elem(wl.dtype) if "lopa_u" in kernel_names else 0)
    elif dom_name == "gate_select_up":
        dom_bytes = algorithmic_bytes(wl, union, gate_kernel_only=True)
    elif dom_name == "down":
        dom_bytes = union * wl.d * w + 4 * union * wl.n + wl.n * wl.d * w
    elif dom_name == "gate_z":
        dom_bytes = (wl.d * wl.d_ff * w if wl.gate == "dense" else wl.r * wl.d_ff * w) + wl.n * wl.d * w
    elif dom_name == "preselected_up":
        dom_bytes = union * wl.d * w + wl.n * wl.d * w
    elif dom_name == "tc_gate":
        dom_bytes = (wl.d * wl.d_ff if wl.gate == "dense" else wl.r * wl.d_ff) * w + wl.n * wl.d * w
    elif dom_name == "tc_up":
        dom_bytes = union * wl.d * w + wl.n * wl.d * w
    elif dom_name == "tc_down":
        dom_bytes = union * wl.d * w + wl.n * wl.d * w
    elif dom_name in ("topk", "topp"):
        dom_bytes = wl.n * wl.d_ff * 4                     # z read (the masks written are overhead)
    elif dom_name == "tc_lopa_u":
        dom_bytes = wl.d * wl.r * w + wl.n * wl.d * w
    elif dom_name == "union_list":
        dom_bytes = wl.d_ff // 8 + 4 * union                # union bitmap read, list written
    else:
        dom_bytes = wl.d * wl.r * w + wl.n * wl.d * w
    # Stage events put an event node between kernels, which stops the next
    # kernel's early (programmatic) launch, so each kernel is timed there
    # without its overlap with its neighbours.  The steady-state launch time
    # is the timed region's time per step apportioned by those shares; for a
    # one-kernel step it is exactly the timed region divided by the steps.
    total = sum(per_name.values())
    share = {nm: v / total for nm, v in per_name.items()}
    avg_launch_ms = ms_per_step * share[dom_name]
    achieved = dom_bytes / (avg_launch_ms * 1e-3) / 1e9
    roofline = {"bound": "hbm", "kernel": dom_name, "achieved": round(achieved, 1),
                "peak": peaks["hbm_gbs"], "peak_kind": peak_kind, "unit": "GB/s",
                "frac": round(achieved / peaks["hbm_gbs"], 4),
                "traffic": traffic_for(dom_name, a.workload, wl.n),
                "algorithmic_bytes_per_launch": int(dom_bytes),
                "avg_launch_us": round(avg_launch_ms * 1e3, 3),
                "kernel_timing": (f"timed region per step x the kernel's share of the step; shares from "
                                  f"CUDA events around each kernel over {K2} steps replayed from a graph"),
                "share": {nm: round(float(v), 4) for nm, v in share.items()},
                "isolated_launch_us": {nm: round(v * 1e3, 3) for nm, v in per_name.items()}}
    if any(c > 1 for c in launch_count.values()):
        roofline["launches_per_step"] = launch_count
        roofline["kernel_timing"] += "; a kernel launched several times per step counts all its launches"
    step_gbs = fwd_bytes / (ms_per_step * 1e-3) / 1e9

    # -- dense FFN on the same weights (the library's dense path)
    dense = None
    if not a.no_dense:
        dffns = ffns
        if dense_gate_w is not None:
            dffns = []
            for i in range(min(R, max(2, math.ceil(3 * l2 / dense_bytes(wl))))):
                f = sffn.SparseFFN(wl.d, wl.d_ff, 0, wl.n, wl.dtype, device=local)
                f.set_weights(w_gate=dense_gate_w, w_up=weights["w_up"].to(dev), w_down=weights["w_down"].to(dev))
                dffns.append(f)
        Rd = len(dffns)
        gate_d = "dense"
        Kd = 2000                  # a comparator outside the timed region: always enough steps
        with torch.cuda.stream(stream):
            for i in range(min(a.warmup, 50)):
                dffns[i % Rd].forward(xs[i % P], gate=gate_d, out=ys[i % P], dense=True, stream=stream, **sel)
        gd = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gd, stream=stream, capture_error_mode="thread_local"):
            for i in range(min(Kd, 64)):
                dffns[i % Rd].forward(xs[i % P], gate=gate_d, out=ys[i % P], dense=True, stream=stream, **sel)
        reps = max(1, Kd // 64)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            gd.replay()                # untimed: a graph's first launch uploads it
        torch.cuda.synchronize()
        with torch.cuda.stream(stream):
            e0.record(stream)
            for _ in range(reps):
                gd.replay()
            e1.record(stream)
        torch.cuda.synchronize()
        dms = e0.elapsed_time(e1) / (reps * min(Kd, 64))
        dense = {"value": dms * 1e3 / wl.n, "unit": UNIT, "gbs": round(dense_bytes(wl) / (dms * 1e-3) / 1e9, 1),
                 "gate": "dense (A B materialised)" if dense_gate_w is not None else "dense"}
        if dffns is not ffns:
            for f in dffns:
                f.close()

    # -- end to end through the C ABI with host buffers
    xs_host = [x.cpu().pin_memory() for x in xs]
    ys_host = [torch.empty((wl.n, wl.d), dtype=xs[0].dtype).pin_memory() for _ in range(P)]
    Ke = max(20, a.e2e_steps)     # host-timed, so not tied to the (possibly short) timed region
    # the C entry point itself, its arguments built once (what a caller with
    # its own buffers does); each call copies x in, runs the forward, copies y
    # out and synchronises
    import ctypes
    sel_c = sffn.make_select(**sel)
    sel_ref = ctypes.byref(sel_c)
    gcode = sffn.gate_code(wl.gate)
    calls = [(ffns[i % R].handle, xs_host[i % P].data_ptr(), wl.n, gcode, sel_ref, ys_host[i % P].data_ptr(),
              stream.cuda_stream) for i in range(math.lcm(R, P))]
    fwd_host = sffn.sffn_forward_host
    for i in range(20):
        sffn.check(fwd_host(*calls[i % len(calls)]), "sffn_forward_host")
    torch.cuda.synchronize()
    barrier(world)
    rcs = 0
    t0 = time.perf_counter()
    for i in range(Ke):
        rcs |= fwd_host(*calls[i % len(calls)])
    e2e_s = reduce_max(time.perf_counter() - t0, world)
    sffn.check(rcs, "sffn_forward_host")
    xbytes = wl.n * wl.d * bytes_per_elem(wl.dtype)
    e2e = {"value": e2e_s * 1e6 / (Ke * wl.n * world), "unit": UNIT, "h2d_bytes_per_step": xbytes,
           "d2h_bytes_per_step": xbytes, "steps": Ke,
           "timer": "host wall clock around synchronous sffn_forward_host calls (pinned host x and y)"}

    clocks = sampler.stop()
    gpu_launches = a.steps * launches

    cpu = None
    if rank == 0 and world == 1 and not a.no_cpu_baseline:
        cpu = cpu_oracle_run(wl, weights, a.cpu_seconds)

    for f in ffns:
        f.close()
    if rank == 0:
        line = {
            "metric": METRIC, "value": round(us_per_token, 4), "unit": UNIT, "n_gpus": world,
            "steps": a.steps, "warmup": a.warmup, "ms_per_step": ms_per_step, "higher_is_better": False,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16" if wl.dtype == "bf16" else "f32",
            "data": "synthetic",
            "config": {"workload": wl.describe() + (" (hot set off)" if wl.hot_frac > 0.0 and hot is None else "")
                       + (" -- DENSE FFN comparator as the step" if a.dense_step else ""),
                       "tokens_per_step": wl.n, "parallelism": f"replicas x{world}",
                       "l2": (f"{R} weight replicas rotated ({R * dense_bytes(wl) / 1e9:.2f} GB > L2 "
                              f"{l2 / 2**20:.0f} MiB), no step reuses L2-resident weights"
                              if R * fwd_bytes >= 3 * l2 else
                              f"{R} weight replica(s) only ({R * fwd_bytes / 1e6:.0f} MB touched per cycle, "
                              f"L2 {l2 / 2**20:.0f} MiB): steps may reuse L2-resident weights (profiling runs)"),
                       "mean_union": union, "timed_with": "CUDA graphs of "
                       f"{G} steps, CUDA events on the launch stream, after one untimed replay of each graph "
                       f"and {pre_replays} untimed pre-roll replays (>= 50 ms) queued straight ahead of it"},
            "spread": spread,
            "warm_l2": warm,
            "tokens_per_s": round(wl.n * world / (ms_per_step * 1e-3), 1),
            "step_gbs": round(step_gbs, 1),
            "step_frac_of_hbm": round(step_gbs / peaks["hbm_gbs"], 4),
            "algorithmic_bytes_per_step": int(fwd_bytes),
            "roofline": roofline,
            "dense_ffn": dense,
            "speedup_vs_dense": round(dense["value"] / (us_per_token * world), 3) if dense else None,
            "e2e": e2e,
            "gpu_launches": gpu_launches,
            "clocks": clocks,
            "cpu_baseline": cpu,
        }
        s = json.dumps(line)
        print(s, flush=True)
        if a.json_out:
            with open(a.json_out, "w") as f:
                f.write(s + "\n")
    if world > 1:
        import torch.distributed as dist
        barrier(world)
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
