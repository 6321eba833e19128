"""Benchmark of the routed MoE layer (route + dispatch + expert MLP + combine).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

One step = one moe_forward over one batch of the workload.  The default is the
largest single-GPU workload, the skewed Kimi-K2-shaped batch: N=16384 tokens,
d=7168, 384 experts, top-8, d_ff=2048, a correction bias calibrated so that
expert popularity follows Zipf(1.2) with 20 experts receiving no token (the
other workloads are selected with --workload).  Inputs are seeded and
synthetic, drawn on the device; the expert weights (33.8 GB) are larger than
L2 and L2 is also flushed (256 MB write) between steps, outside the per-step
events.  Under torchrun every rank runs its own batch (token rows rank*N ..
rank*N+N-1) with the same weights: weak scaling with no collective on the
data path; the step time is the max over ranks.  Rank 0 prints one JSON line.
`--workload k3_block_decode` (or tiny_block) times the whole MoE block instead
(moe_block_forward: gate, shared experts, latent projections and norm around
the routed layer).

`value` is tokens over the mean of the K per-step CUDA-event times (the
median is reported beside it); `stages_ms` comes from a second pass of K
steps with an event after every stage.  `gpu_launches` is the library's own
count of the kernels it launched in the timed region (moe_launch_count).

The `e2e` figure is the same step through the public API from pinned host
memory, each step uploading its tokens and downloading its output; the
copies of neighbouring steps overlap on two copy streams (double-buffered),
and the timed region spans the first upload to the last download.

--impl reference times the CPU reference (oracle/) on the host cores on a
bounded sample of the same workload (its line says which sample and that the
figure is extrapolated from it); it is the slow reference arm, not a target.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "routed tokens/sec per MoE layer (route+dispatch+FFN+combine)"
UNIT = "tokens/s"
DEFAULT_WORKLOAD = "k2_skew"
# nominal B200 figures, reported beside the measured peaks for context
NOMINAL_HBM_GBS = 7700.0
NOMINAL_BF16_TFLOPS = 2250.0


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=20)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--workload", default=DEFAULT_WORKLOAD)
    p.add_argument("--impl", default="ours", choices=["ours", "reference"])
    p.add_argument("--no-cpu-baseline", action="store_true")
    # time replays of one moe_forward captured in a CUDA graph (the routed
    # layer only; the stage breakdown and the end-to-end pass stay eager)
    p.add_argument("--graph", action="store_true")
    # profiling cases: the same workload with fewer tokens / experts
    p.add_argument("--tokens", type=int, default=None)
    p.add_argument("--experts", type=int, default=None)
    p.add_argument("--ffn", type=int, default=None)
    # router variants ("DeepSeek-V3.2-Exp · Affinities", gate-forward)
    p.add_argument("--score-func", default="sigmoid", choices=["sigmoid", "softmax"])
    p.add_argument("--group-score", default="top2_sum", choices=["top2_sum", "max"])
    return p.parse_args()


def route_cfg(moe, wl, args):
    return moe.RouteConfig(wl.E, wl.G, wl.TG, wl.K, wl.route_scale, wl.norm,
                           score_func=args.score_func, group_score=args.group_score)


def workload_of(args):
    from synth.workloads import BLOCKS, WORKLOADS, scaled
    wl = WORKLOADS[args.workload] if args.workload in WORKLOADS else BLOCKS[args.workload]
    kw = {}
    if args.tokens:
        kw["N"] = args.tokens
    if args.experts:
        kw["E"] = args.experts
    if args.ffn:
        kw["F"] = args.ffn
    return scaled(wl, **kw) if kw else wl


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "bf16_tflops_sustained": float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "source": "fallback"}


# ------------------------------------------------------------------ clocks
class ClockSampler:
    """nvidia-smi sampling of SM clock and throttle reasons during a region."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.path = None
        # raw samples go to a temporary file unless MOE_BENCH_CLOCKS_DIR names
        # a folder to keep them in
        self.keep_dir = os.environ.get("MOE_BENCH_CLOCKS_DIR")

    def __enter__(self):
        if self.keep_dir:
            os.makedirs(self.keep_dir, exist_ok=True)
            self.path = os.path.join(self.keep_dir, f"clocks_{os.getpid()}.csv")
        else:
            fd, self.path = tempfile.mkstemp(prefix="moe_clocks_", suffix=".csv")
            os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.Q}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except OSError:
            self.proc = None
        return self

    def __exit__(self, *a):
        if self.proc is not None:
            time.sleep(0.2)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        if self.proc is None or not os.path.exists(self.path):
            if not self.keep_dir and self.path and os.path.exists(self.path):
                os.remove(self.path)
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not self.keep_dir:
            os.remove(self.path)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(sm)}


# ------------------------------------------------------------ multi-rank
def max_over_ranks(values, world, device="cpu"):
    """Element-wise max of per-rank timings (the slowest rank sets the step)."""
    if world <= 1:
        return list(values)
    import torch
    import torch.distributed as dist
    t = torch.tensor(values, dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def aggregate_throughput(tokens_per_rank, world, step_ms_max):
    """Whole-job routed tokens/s: every rank's tokens over the slowest rank's time."""
    return world * tokens_per_rank / (step_ms_max * 1e-3)


def e2e_pipelined(torch, steps, hosts, run, out_like):
    """Milliseconds per step end to end through the public API from pinned
    host memory.  Every step uploads its inputs (`hosts`) and downloads its
    output; the upload of step i runs on one copy stream while step i-1
    computes and its download on another while step i+1 computes (two device
    buffers each), the way a serving loop would run.  The timed region spans
    the first upload to the last download, so every copy is inside it."""
    comp = torch.cuda.current_stream()
    up, down = torch.cuda.Stream(), torch.cuda.Stream()
    devs = [[torch.empty(h.shape, dtype=h.dtype, device="cuda") for h in hosts] for _ in range(2)]
    outs = [torch.empty_like(out_like) for _ in range(2)]
    outs_h = [torch.empty(tuple(out_like.shape), dtype=out_like.dtype, pin_memory=True)
              for _ in range(2)]
    uploaded = [torch.cuda.Event() for _ in range(2)]
    computed = [torch.cuda.Event() for _ in range(2)]
    downloaded = [torch.cuda.Event() for _ in range(2)]

    def one(i):
        b = i & 1
        with torch.cuda.stream(up):
            if i >= 2:
                up.wait_event(computed[b])  # the step that read buffer b is done
            for d, h in zip(devs[b], hosts):
                d.copy_(h, non_blocking=True)
            uploaded[b].record(up)
        comp.wait_event(uploaded[b])
        if i >= 2:
            comp.wait_event(downloaded[b])  # output buffer b has been read back
        run(devs[b], outs[b])
        computed[b].record(comp)
        with torch.cuda.stream(down):
            down.wait_event(computed[b])
            outs_h[b].copy_(outs[b], non_blocking=True)
            downloaded[b].record(down)

    for i in range(3):
        one(i)
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(comp)
    up.wait_stream(comp)
    for i in range(steps):
        one(i)
    comp.wait_stream(down)
    t1.record(comp)
    t1.synchronize()
    return t0.elapsed_time(t1) / steps


# ---------------------------------------------------------------- our arm
def run_ours(args, rank, world, local_rank):
    import torch
    import moe_routing_expert_fp32_b200 as moe
    import synth
    from synth.workloads import dev_inputs

    wl = workload_of(args)
    torch.cuda.set_device(local_rank)
    dev = dev_inputs(wl, rank=rank)
    cfg = route_cfg(moe, wl, args)
    act = moe.ActConfig(wl.act, wl.beta, wl.lbeta)
    x_e = dev["x_e"] if wl.latent else None
    ws = moe.workspace(moe.workspace_size(wl.N, wl.d_r, wl.d_e, cfg, wl.F))
    out = torch.empty((wl.N, wl.d_e), dtype=torch.bfloat16, device="cuda")
    counts_probe = torch.empty((wl.N, wl.K), dtype=torch.int32, device="cuda")
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
    names = ["after_route", "after_dispatch", "after_gate_up", "after_down", "after_combine"]

    def step(events=None, idx=None):
        moe.forward(dev["x"], dev["W"], dev["bias"], cfg, dev["w1"], dev["w3"], dev["w2"], act,
                    x_e=x_e, ws=ws, out=out, topk_idx=idx, events=events)

    torch.cuda.synchronize()
    for _ in range(max(args.warmup, 3)):
        flush.zero_()
        step()
    torch.cuda.synchronize()

    def barrier():
        if world > 1:
            import torch.distributed as dist
            dist.barrier()

    # with --graph the timed steps replay one captured moe_forward (the same
    # kernels and arguments; the library counts launches at capture, so the
    # timed region's count is the graph's kernels times the steps)
    graph, per_graph = None, 0
    if args.graph:
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            step()
        torch.cuda.current_stream().wait_stream(side)
        torch.cuda.synchronize()
        graph = torch.cuda.CUDAGraph()
        c0 = moe.launch_count()
        with torch.cuda.graph(graph):
            step()
        per_graph = moe.launch_count() - c0
        for _ in range(max(args.warmup, 3)):
            flush.zero_()
            graph.replay()
        torch.cuda.synchronize()

    # timed region: K steps, one start/end event pair around each moe_forward
    ev0 = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(args.steps)]
    with ClockSampler(local_rank) as clk:
        barrier()
        torch.cuda.synchronize()
        n0 = moe.launch_count()
        t0 = time.perf_counter()
        for i in range(args.steps):
            flush.zero_()
            ev0[i][0].record()
            if graph is not None:
                graph.replay()
            else:
                step()
            ev0[i][1].record()
        torch.cuda.synchronize()
        barrier()
        wall = time.perf_counter() - t0
        launches = moe.launch_count() - n0 + per_graph * args.steps
    del graph
    per_step = [a.elapsed_time(b) for a, b in ev0]
    ms = statistics.mean(per_step)

    # breakdown pass: the same steps with an event after every stage (events
    # between the two expert kernels hold back the second one's early start,
    # so this pass is used for the per-stage times only)
    ev = [{"start": torch.cuda.Event(enable_timing=True),
           **{n: torch.cuda.Event(enable_timing=True) for n in names}} for _ in range(args.steps)]
    for e in ev:  # create the CUDA events before handing their handles to the library
        for v in e.values():
            v.record()
    torch.cuda.synchronize()
    for i in range(args.steps):
        flush.zero_()
        ev[i]["start"].record()
        step(events={n: ev[i][n] for n in names})
    torch.cuda.synchronize()
    stage_ms = {}
    prev = "start"
    for n in names:
        stage_ms[n.replace("after_", "")] = statistics.mean(
            e[prev].elapsed_time(e[n]) for e in ev)
        prev = n

    # routing statistics of the timed batch (for the algorithmic byte count)
    step(idx=counts_probe)
    torch.cuda.synchronize()
    counts = np.bincount(counts_probe.cpu().numpy().ravel(), minlength=wl.E)
    touched = int((counts > 0).sum())

    # end to end through the public API from pinned host buffers (weights
    # larger than L2; copies of neighbouring steps overlapped)
    hosts = [torch.empty((wl.N, wl.d_r), dtype=torch.bfloat16, pin_memory=True)]
    hosts[0].copy_(dev["x"].cpu())
    if wl.latent:
        hosts.append(torch.empty((wl.N, wl.d_e), dtype=torch.bfloat16, pin_memory=True))
        hosts[1].copy_(dev["x_e"].cpu())

    def e2e_run(xs_dev, o):
        moe.forward(xs_dev[0], dev["W"], dev["bias"], cfg, dev["w1"], dev["w3"], dev["w2"], act,
                    x_e=xs_dev[1] if wl.latent else None, ws=ws, out=o)

    e2e_ms = [e2e_pipelined(torch, args.steps, hosts, e2e_run, out)]
    h2d = wl.N * wl.d_r * 2 + (wl.N * wl.d_e * 2 if wl.latent else 0)
    d2h = wl.N * wl.d_e * 2

    ms_max, e2e_max, gu_ms, wall_max = max_over_ranks(
        [ms, statistics.mean(e2e_ms), stage_ms["gate_up"], wall], world, "cuda")

    srt = np.sort(counts)[::-1]
    top10 = float(srt[: max(1, wl.E // 10)].sum() / max(1, counts.sum()))
    res = {
        "ms": ms_max, "e2e_ms": e2e_max, "stage_ms": stage_ms, "gate_up_ms": gu_ms,
        "step_ms": [min(per_step), statistics.median(per_step), max(per_step)],
        "touched": touched, "counts_max": int(counts.max()), "top10_share": top10,
        "clocks": clk.summary(), "h2d": h2d, "d2h": d2h, "wall_s": wall_max,
        "launches": launches,
    }
    return wl, res


# ------------------------------------------------------ whole-block arm
BLOCK_METRIC = "tokens/sec per MoE block (route+shared experts+latent projections+routed experts)"


def block_bytes(wl, touched):
    """Algorithmic HBM bytes of one block step: every weight byte read once
    (gate fp32; projections, norm, shared and touched routed experts bf16) and
    the activations each stage must write and read back."""
    N, S = wl.N, wl.N * wl.K
    w = wl.E * wl.d_r * 4 + touched * 3 * wl.F * wl.d_e * 2
    if wl.latent:
        w += 2 * wl.d_e * wl.d_r * 2 + wl.d_e * 2
    if wl.F_shared:
        w += 3 * wl.F_shared * wl.d_r * 2
    act = N * wl.d_r * 2 + N * wl.d_r * 2                # x read, out written
    act += 2 * (S * wl.d_e * 2) + 2 * (S * wl.F * 2) + 2 * (S * wl.d_e * 2)  # xs, h, y
    if wl.latent:
        act += 2 * N * wl.d_e * 2 * 2                     # x_e and the combined rows
    if wl.F_shared:
        act += 2 * N * wl.F_shared * 2 + 2 * N * wl.d_r * 2  # shared h and output
    return w + act


def run_block(args, rank, world, local_rank):
    import torch
    import moe_routing_expert_fp32_b200 as moe
    from synth.workloads import dev_block, dev_inputs

    wl = workload_of(args)
    torch.cuda.set_device(local_rank)
    dev = dev_inputs(wl, rank=rank)
    blk = dev_block(wl)
    sh = blk["shared"] or (None, None, None)
    W = moe.BlockWeights(gate_weight=dev["W"], gate_bias=dev["bias"], w1=dev["w1"], w3=dev["w3"],
                         w2=dev["w2"], down_proj=blk["down_proj"], norm_weight=blk["norm_w"],
                         up_proj=blk["up_proj"], shared_w1=sh[0], shared_w3=sh[1],
                         shared_w2=sh[2])
    cfg = route_cfg(moe, wl, args)
    act = moe.ActConfig(wl.act, wl.beta, wl.lbeta)
    out = torch.empty((wl.N, wl.d_r), dtype=torch.bfloat16, device="cuda")
    idx = torch.empty((wl.N, wl.K), dtype=torch.int32, device="cuda")
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
    ws = [None]

    def step(x=None):
        o = moe.block_forward(dev["x"] if x is None else x, W, cfg, act, norm_eps=wl.norm_eps,
                              ws=ws[0], out=out, topk_idx=idx)
        return o

    # first call sizes the workspace; keep it
    import ctypes
    dims = moe._BlockDims(wl.d_r, wl.d_e, wl.F, wl.F_shared, wl.norm_eps)
    wc, c = W._c(), cfg._c()
    ws[0] = moe.workspace(moe.lib().moe_block_workspace_size(wl.N, ctypes.byref(dims),
                                                             ctypes.byref(wc), ctypes.byref(c)))
    torch.cuda.synchronize()
    for _ in range(max(args.warmup, 3)):
        flush.zero_()
        step()
    torch.cuda.synchronize()

    def barrier():
        if world > 1:
            import torch.distributed as dist
            dist.barrier()

    ev0 = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(args.steps)]
    with ClockSampler(local_rank) as clk:
        barrier()
        torch.cuda.synchronize()
        n0 = moe.launch_count()
        t0 = time.perf_counter()
        for i in range(args.steps):
            flush.zero_()
            ev0[i][0].record()
            step()
            ev0[i][1].record()
        torch.cuda.synchronize()
        barrier()
        wall = time.perf_counter() - t0
        launches = moe.launch_count() - n0
    per_step = [a.elapsed_time(b) for a, b in ev0]
    ms = statistics.mean(per_step)
    counts = np.bincount(idx.cpu().numpy().ravel(), minlength=wl.E)
    touched = int((counts > 0).sum())

    hosts = [torch.empty((wl.N, wl.d_r), dtype=torch.bfloat16, pin_memory=True)]
    hosts[0].copy_(dev["x"].cpu())

    def e2e_run(xs_dev, o):
        moe.block_forward(xs_dev[0], W, cfg, act, norm_eps=wl.norm_eps, ws=ws[0], out=o)

    e2e_ms = [e2e_pipelined(torch, args.steps, hosts, e2e_run, out)]
    ms_max, e2e_max, wall_max = max_over_ranks([ms, statistics.mean(e2e_ms), wall], world, "cuda")
    return wl, {"ms": ms_max, "e2e_ms": e2e_max, "touched": touched, "clocks": clk.summary(),
                "h2d": wl.N * wl.d_r * 2, "d2h": wl.N * wl.d_r * 2, "wall_s": wall_max,
                "launches": launches,
                "step_ms": [min(per_step), statistics.median(per_step), max(per_step)]}


def block_line(args, wl, r, world):
    peaks = load_peaks()
    achieved = block_bytes(wl, r["touched"]) / (r["ms"] * 1e-3) / 1e9
    return {
        "metric": BLOCK_METRIC, "value": aggregate_throughput(wl.N, world, r["ms"]),
        "unit": UNIT, "n_gpus": world, "steps": args.steps, "warmup": max(args.warmup, 3),
        "ms_per_step": r["ms"], "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": wl.name, "N": wl.N, "d_r": wl.d_r, "d_e": wl.d_e, "E": wl.E,
                   "K": wl.K, "F": wl.F, "F_shared": wl.F_shared, "act": wl.act,
                   "router": f"{args.score_func}/{args.group_score}",
                   "global_batch": world * wl.N, "parallelism": f"dp{world}",
                   "l2": "weights > L2, plus a 256 MB write between steps outside the "
                         "per-step events"},
        "roofline": {"kernel": "whole block step (HBM-bound weight stream)", "bound": "hbm",
                     "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                     "frac": achieved / peaks["hbm_gbs"], "traffic": None,
                     "peak_source": peaks["source"], "touched_experts": r["touched"],
                     "peak_nominal": NOMINAL_HBM_GBS,
                     "frac_of_nominal": achieved / NOMINAL_HBM_GBS},
        "e2e": {"value": aggregate_throughput(wl.N, world, r["e2e_ms"]), "unit": UNIT,
                "h2d_bytes_per_step": r["h2d"], "d2h_bytes_per_step": r["d2h"]},
        "step_ms_min_median_max": r["step_ms"],
        "step_ms_stat": "mean of the K per-step CUDA-event times",
        "gpu_launches": r["launches"],
        "clocks": r["clocks"],
    }


def source_sha256(source):
    """sha256 of a record's kernel source: one path, or the bytes of several
    (the kernel file and the headers it includes) in the listed order."""
    import hashlib
    h = hashlib.sha256()
    for rel in ([source] if isinstance(source, str) else source):
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def gate_up_traffic(workload, touched, bound, path=None):
    # workload: the bench's Workload (name and sizes must match a same-workload record)
    """DRAM bytes of one gate_up launch from a committed ncu capture: for an
    HBM-bound launch the decode-shaped capture scaled by touched experts, for a
    tensor-bound one the capture of the same workload; None when there is no
    such record or the kernel source has changed since it was taken."""
    path = path or os.path.join(ROOT, "profiles", "expert_gemm_traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        records = json.load(f)["records"]
    for rec in records:
        if bound == "hbm" and rec["scaling"] == "touched":
            scale = touched / rec["touched_experts"]
        elif bound == "tensor" and rec["scaling"] == "same-workload" and \
                (rec["workload"], rec["N"], rec["E"]) == (workload.name, workload.N, workload.E):
            scale = 1.0
        else:
            continue
        if source_sha256(rec["source"]) != rec["source_sha256"]:
            return None
        return (rec["dram_bytes_read"] + rec["dram_bytes_write"]) * scale
    return None


def gate_up_bytes(wl, touched):
    """Algorithmic HBM bytes of one w1/w3 launch: both weight matrices of every
    touched expert, the gathered rows read, the h rows written."""
    S = wl.N * wl.K
    return touched * 2 * wl.F * wl.d_e * 2 + S * wl.d_e * 2 + S * wl.F * 2


def gate_up_flops(wl):
    """Algorithmic flops of one w1/w3 launch: g and u for every slot."""
    return 4 * wl.N * wl.K * wl.F * wl.d_e


def gate_up_roofline(wl, touched, gate_up_ms, peaks):
    """The roofline object of the w1/w3 kernel.  Its bound is the one with the
    longer ideal time: the algorithmic bytes at the measured copy bandwidth,
    or the algorithmic flops at the sustained bf16 peak (the kernel runs for
    milliseconds inside a long step).  DRAM traffic comes from the committed
    captures (gate_up_traffic)."""
    nbytes, flops = gate_up_bytes(wl, touched), gate_up_flops(wl)
    t_hbm = nbytes / (peaks["hbm_gbs"] * 1e9)
    t_tensor = flops / (peaks["bf16_tflops_sustained"] * 1e12)
    sec = gate_up_ms * 1e-3
    obj = {"kernel": "expert w1/w3 (gate_up) grouped GEMM"}
    if t_tensor > t_hbm:
        achieved = flops / sec / 1e12
        obj.update({"bound": "tensor", "achieved": achieved,
                    "peak": peaks["bf16_tflops_sustained"], "unit": "TFLOP/s",
                    "frac": achieved / peaks["bf16_tflops_sustained"],
                    "traffic": gate_up_traffic(wl, touched, "tensor"),
                    "peak_kind": "sustained bf16", "peak_nominal": NOMINAL_BF16_TFLOPS,
                    "frac_of_nominal": achieved / NOMINAL_BF16_TFLOPS})
    else:
        achieved = nbytes / sec / 1e9
        obj.update({"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"],
                    "unit": "GB/s", "frac": achieved / peaks["hbm_gbs"],
                    "traffic": gate_up_traffic(wl, touched, "hbm"),
                    "peak_nominal": NOMINAL_HBM_GBS,
                    "frac_of_nominal": achieved / NOMINAL_HBM_GBS})
    obj.update({"peak_source": peaks["source"], "touched_experts": touched})
    return obj


# ------------------------------------------------------------ oracle arm
ROUTE_SAMPLE_TOKENS = 2048   # tokens routed, sorted and combined per sample
FFN_SAMPLE_ROWS = 240        # expert-MLP rows per sample
FFN_SAMPLE_EXPERTS = 8       # at most this many experts' weights drawn per sample
SUBSET_TOKENS = 256          # the single-threaded subset
SUBSET_FFN_ROWS = 24


def _router_codes(router):
    import oracle
    return ({"sigmoid": oracle.SCORE_SIGMOID, "softmax": oracle.SCORE_SOFTMAX}[router[0]],
            {"top2_sum": oracle.GROUP_TOP2_SUM, "max": oracle.GROUP_MAX}[router[1]])


def _oracle_step(wl, inp, n_tok, n_rows, router):
    """One bounded pass of the CPU reference over the first `n_tok` tokens of
    the batch: route, sort + gather and combine run on all of them; the
    expert MLP runs on up to `n_rows` of their sorted rows, taken from the
    least-, median- and most-loaded experts they touch and, while those hold
    too few rows, the next most-loaded ones (the cost of a row does not
    depend on its expert).
    Returns the measured seconds of each stage, each scaled to the whole
    batch (route, sort and combine by N / n_tok, the MLP by N*K / n_rows),
    and what was sampled."""
    import oracle
    from synth.workloads import host_expert

    score, group = _router_codes(router)
    x = np.ascontiguousarray(inp["x"][:n_tok])
    xe = np.ascontiguousarray(inp["x_e"][:n_tok])
    raw = {}
    t0 = time.perf_counter()
    idx, w, _ = oracle.route(x, inp["W"], inp["bias"], wl.G, wl.TG, wl.K, wl.route_scale,
                             wl.norm, score=score, group=group)
    raw["route"] = time.perf_counter() - t0
    t0 = time.perf_counter()
    counts, offsets, perm, pos = oracle.dispatch(idx, wl.E)
    xs = oracle.gather(xe, perm, wl.K)
    raw["dispatch"] = time.perf_counter() - t0
    touched = [int(e) for e in np.argsort(counts, kind="stable") if counts[e] > 0]
    # the least-, median- and most-loaded experts, then the next most-loaded
    # ones (at most FFN_SAMPLE_EXPERTS) while their rows fall short of n_rows
    picks = list(dict.fromkeys([touched[0], touched[len(touched) // 2], touched[-1]]))
    for e in reversed(touched):
        if len(picks) >= FFN_SAMPLE_EXPERTS or int(counts[picks].sum()) >= n_rows:
            break
        if e not in picks:
            picks.append(e)
    # an equal share each, the lighter experts' shortfall taken by the heavier
    spans, left = [], min(n_rows, int(counts[picks].sum()))
    for i, e in enumerate(picks):
        take = min(int(counts[e]), left // (len(picks) - i))
        spans.append((e, int(offsets[e]), int(offsets[e]) + take))
        left -= take
    weights = {e: host_expert(wl, e) for e in picks}  # inputs, not timed
    ys = np.zeros_like(xs)
    done = 0
    t0 = time.perf_counter()
    for e, a, b in spans:
        ys[a:b] = oracle.expert_ffn(xs[a:b], *weights[e], wl.act, wl.beta, wl.lbeta)
        done += b - a
    raw["ffn"] = time.perf_counter() - t0
    t0 = time.perf_counter()
    oracle.combine(ys, pos, w, wl.K)
    raw["combine"] = time.perf_counter() - t0
    scale_tok = wl.N / n_tok
    scaled_s = {"route": raw["route"] * scale_tok, "dispatch": raw["dispatch"] * scale_tok,
                "ffn": raw["ffn"] * wl.N * wl.K / max(done, 1),
                "combine": raw["combine"] * scale_tok}
    what = (f"route, sort+gather and combine of the first {n_tok} of {wl.N} tokens (time x "
            f"{scale_tok:g}); expert MLP on {done} of their sorted rows from experts "
            f"{[(e, b - a) for e, a, b in spans]} ((expert, rows): least-, median-, most-loaded, "
            f"then the next most-loaded; "
            f"time x {wl.N * wl.K}/{done} slots)")
    return scaled_s, raw, what


def oracle_sample(wl, router=("sigmoid", "top2_sum")):
    """The CPU reference on all host cores over a bounded sample of one step
    (_oracle_step with ROUTE_SAMPLE_TOKENS tokens and FFN_SAMPLE_ROWS MLP
    rows), extrapolated to the whole batch.  Returns tokens/s, the cores
    used, the per-stage seconds (extrapolated and as measured) and the
    sample's description."""
    import oracle
    from synth.workloads import host_inputs

    oracle.set_threads(os.cpu_count() or 1)
    cores = oracle.max_threads()
    n_tok = min(wl.N, ROUTE_SAMPLE_TOKENS)
    inp = host_inputs(wl, n_tokens=n_tok)
    sc, raw, what = _oracle_step(wl, inp, n_tok, FFN_SAMPLE_ROWS, router)
    total = sum(sc.values())
    return {"value": wl.N / total, "cores": cores, "seconds": sc, "sample_seconds": raw,
            "sample": what}


def oracle_subset_single(wl, router=("sigmoid", "top2_sum")):
    """The single-threaded CPU reference on the first SUBSET_TOKENS tokens
    (route, sort, combine on all of them; the expert MLP on SUBSET_FFN_ROWS
    of their rows, scaled to their slots): tokens/s of that subset, labelled
    as such and not extrapolated to the batch."""
    import oracle
    from synth.workloads import host_inputs, scaled

    n_tok = min(wl.N, SUBSET_TOKENS)
    sub = scaled(wl, N=n_tok)
    inp = host_inputs(wl, n_tokens=n_tok)
    oracle.set_threads(1)
    try:
        sc, raw, what = _oracle_step(sub, inp, n_tok, SUBSET_FFN_ROWS, router)
    finally:
        oracle.set_threads(os.cpu_count() or 1)
    return {"value": n_tok / sum(sc.values()), "cores": 1, "tokens": n_tok, "seconds": sc,
            "sample": "subset: " + what}


def cpu_baseline_obj(cb, subset=None):
    """The line's cpu_baseline object: the all-core sample as the value, its
    per-stage seconds, and the single-threaded subset beside it."""
    obj = {"value": cb["value"], "unit": UNIT, "cores": cb["cores"], "kind": "oracle",
           "sample": cb["sample"], "extrapolated": True,
           "stage_seconds": {k: round(v, 6) for k, v in cb["seconds"].items()}}
    if "sample_seconds" in cb:
        obj["sample_stage_seconds"] = {k: round(v, 6) for k, v in cb["sample_seconds"].items()}
    if subset is not None:
        obj["single_thread_subset"] = {
            "value": subset["value"], "unit": UNIT, "cores": 1, "tokens": subset["tokens"],
            "stage_seconds": {k: round(v, 6) for k, v in subset["seconds"].items()},
            "sample": subset["sample"]}
    return obj


def oracle_sample_block(wl, n_tokens=4, router=("sigmoid", "top2_sum")):
    """The CPU reference on a bounded sample of a whole-block step: the routed
    layer as oracle_sample; the latent projections and the norm on all
    tokens; the shared experts on `n_tokens` tokens, scaled to all."""
    import oracle
    from synth.workloads import host_block, host_inputs

    r = oracle_sample(wl, router)
    hb = host_block(wl)
    x = host_inputs(wl)["x"]
    t = dict(r["seconds"])
    if wl.latent:
        t0 = time.perf_counter()
        xe = oracle.linear(x, hb["down_proj"])
        y = oracle.rms_norm(xe, hb["norm_w"], wl.norm_eps)  # a stand-in row block of the width
        oracle.linear(y, hb["up_proj"])
        t["projections_norm"] = time.perf_counter() - t0
    if wl.F_shared:
        n = min(n_tokens, wl.N)
        t0 = time.perf_counter()
        oracle.expert_ffn(np.ascontiguousarray(x[:n]), *hb["shared"], wl.act, wl.beta, wl.lbeta)
        t["shared"] = (time.perf_counter() - t0) * wl.N / n
    total = sum(t.values())
    return {"value": wl.N / total, "cores": r["cores"], "seconds": t,
            "sample": r["sample"] + (f"; down/up projections and norm on all {wl.N} tokens"
                                     if wl.latent else "") +
                      (f"; shared experts on {min(n_tokens, wl.N)} tokens, time scaled to "
                       f"{wl.N}" if wl.F_shared else "")}


def run_reference(args, rank, world):
    """The reference arm: the CPU reference (oracle/) as it stands, timed on
    the host cores, each step one bounded sample of the workload (the same
    sample as the cpu_baseline leg), W untimed sample steps first.  The
    figure is extrapolated from the sample and says so."""
    if rank != 0:
        return
    wl = workload_of(args)
    from synth.workloads import BLOCKS
    block = args.workload in BLOCKS
    rt = (args.score_func, args.group_score)

    def one():
        return oracle_sample_block(wl, router=rt) if block else oracle_sample(wl, router=rt)

    for _ in range(args.warmup):
        one()
    vals = []
    t_start = time.perf_counter()
    res = None
    for _ in range(args.steps):
        res = one()
        vals.append(res["value"])
    wall = time.perf_counter() - t_start
    v = statistics.mean(vals)
    cb = cpu_baseline_obj(res)
    cb["value"] = v
    line = {
        "impl": "reference", "metric": BLOCK_METRIC if block else METRIC, "value": v,
        "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * wl.N / v,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": {"workload": wl.name, "N": wl.N, "d_r": wl.d_r,
                                        "d_e": wl.d_e, "E": wl.E, "K": wl.K, "F": wl.F,
                                        "router": f"{args.score_func}/{args.group_score}"},
        "extrapolated": True,
        "cpu_baseline": cb,
        "e2e": {"value": v, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "wall_s": wall,
    }
    print(json.dumps(line), flush=True)


def main():
    args = parse()
    rank = int(os.environ.get("RANK", 0))
    world = int(os.environ.get("WORLD_SIZE", 1))
    local_rank = int(os.environ.get("LOCAL_RANK", 0))
    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    import torch
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    from synth.workloads import BLOCKS
    if args.workload in BLOCKS:
        wl, r = run_block(args, rank, world, local_rank)
        line = block_line(args, wl, r, world)
        if rank == 0 and world == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline_obj(
                oracle_sample_block(wl, router=(args.score_func, args.group_score)))
        if world > 1:
            import torch.distributed as dist
            dist.barrier()
            dist.destroy_process_group()
        if rank == 0:
            print(json.dumps(line), flush=True)
        return
    wl, r = run_ours(args, rank, world, local_rank)
    peaks = load_peaks()
    line = {
        "metric": METRIC,
        "value": aggregate_throughput(wl.N, world, r["ms"]),
        "unit": UNIT,
        "n_gpus": world,
        "steps": args.steps,
        "warmup": max(args.warmup, 3),
        "ms_per_step": r["ms"],
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": wl.name, "N": wl.N, "d_r": wl.d_r, "d_e": wl.d_e, "E": wl.E,
                   "n_group": wl.G, "topk_group": wl.TG, "K": wl.K, "F": wl.F, "act": wl.act,
                   "router": f"{args.score_func}/{args.group_score}",
                   "global_batch": world * wl.N, "parallelism": f"dp{world}",
                   "l2": "expert weights > L2, plus a 256 MB write between steps outside the "
                         "per-step events",
                   "launch": "CUDA graph replay" if args.graph else "eager"},
        "roofline": gate_up_roofline(wl, r["touched"], r["gate_up_ms"], peaks),
        "stages_ms": r["stage_ms"],
        "stages_pass": "a second pass of K steps with a CUDA event after every stage",
        "step_ms_min_median_max": r["step_ms"],
        "step_ms_stat": "mean of the K per-step CUDA-event times",
        "routing": {"touched_experts": r["touched"], "max_rows_per_expert": r["counts_max"],
                    "top10pct_expert_share": r["top10_share"]},
        "e2e": {"value": aggregate_throughput(wl.N, world, r["e2e_ms"]), "unit": UNIT,
                "h2d_bytes_per_step": r["h2d"], "d2h_bytes_per_step": r["d2h"]},
        "gpu_launches": r["launches"],
        "clocks": r["clocks"],
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline_obj(
            oracle_sample(wl, router=(args.score_func, args.group_score)),
            oracle_subset_single(wl, router=(args.score_func, args.group_score)))
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
