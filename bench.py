#!/usr/bin/env python
"""Benchmark of the grouped 4-bit MoE GEMM (one JSON line on rank 0).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]
                    [--op gemm|swiglu|combine]

A step is one pass of the hot path over one routed batch: for every token count
of the workload, the gate_up projection (reads token rows, writes sorted rows)
and the down projection (reads sorted rows, weights them, scatters to t*k+slot),
each one grouped GEMM call through the C ABI. Inputs are synthetic (seeded);
the weights are N(0, 0.02) quantized on the device by the library's quantizer.

Metric: packed-weight GB/s = nibble + scale bytes of the experts each call
touches, divided by device time (decode workloads); TFLOP/s = 2*R*N*K / time
for the prefill workload. L2: the timed steps rotate over enough copies of the
weight stacks that the bytes between two uses of one copy exceed twice the L2
size. Multi-GPU: one independent replica per rank (the path has no exchange
step), value = all ranks' work / the slowest rank's time.

``--op swiglu`` / ``--op combine`` time instead the memory-bound kernel on one
side of the GEMM, at the workload's largest token count: bf16 bytes read and
written per call over device time (HBM roofline), inputs rotated past L2 or L2
flushed before each call.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402
from synth.workloads import WORKLOADS, expert_bytes  # noqa: E402

METRIC = "grouped 4-bit MoE GEMM: packed-weight GB/s (decode), TFLOP/s (prefill)"
GLUE_OPS = {"swiglu": "MoE SwiGLU over gate_up rows: HBM GB/s (bf16 read + written)",
            "combine": "MoE top-k combine (fp32 slot-order sum): HBM GB/s (bf16 read + written)"}
DEFAULT_WORKLOAD = "olmoe_decode_nf4"
PREFILL_WORKLOADS = {"qwen3_prefill_nf4"}


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--absmax", default="f32", choices=["f32", "bf16"],
                    help="NF4 absmax storage: f32, or bf16 (the weights are then drawn as bf16 values, a "
                         "bf16 source, so the cast is lossless)")
    ap.add_argument("--x-dtype", default="bf16", choices=["bf16", "f16"],
                    help="activations (and output) type")
    ap.add_argument("--unfused-swiglu", action="store_true",
                    help="--op layer: run gate_up and the SwiGLU as two kernels (default: fused)")
    ap.add_argument("--no-sub-records", action="store_true",
                    help="default workload only: skip the prefill and MXFP4 sub-records")
    ap.add_argument("--top-k", type=int, default=None, help="sweep workload: top_k (default first)")
    ap.add_argument("--tokens", type=str, default=None, help="comma list overriding the token counts")
    ap.add_argument("--op", default="gemm", choices=["gemm", "dgrad", "layer"] + list(GLUE_OPS),
                    help="gemm: the grouped GEMM step (default); dgrad: its input gradient, every "
                         "call of the step; layer: the whole MoE layer (device routing, gate_up, "
                         "SwiGLU, down, combine) as one CUDA graph per token count; swiglu / combine: "
                         "the glue kernel either side of the GEMM, on the workload's largest token count")
    return ap.parse_args()


def workload_calls(wl, seed, top_k=None, tokens=None):
    """The grouped GEMM calls of one step: (T, projection, routed batch)."""
    k = top_k if top_k is not None else wl.top_k[-1 if wl.name != "olmoe_sweep_nf4" else 0]
    Ts = tokens if tokens is not None else wl.T
    calls = []
    for T in Ts:
        b = synth.make_routed_batch(seed, T, wl.E, k, routing=wl.routing)
        for proj in wl.projections:
            calls.append((T, proj, b))
    return calls, k


def call_bytes(fmt, proj, b, absmax="f32"):
    """Algorithmic bytes of one call: the packed codes and scales of the experts it
    touches (bf16 absmax: 2 bytes a block instead of 4)."""
    pb = expert_bytes(fmt, proj.N, proj.K)
    if fmt == "nf4" and absmax == "bf16":
        pb = dict(pb, scales=pb["scales"] // 2)
    n_act = int((np.diff(b.offsets) > 0).sum())
    return n_act * (pb["nibbles"] + pb["scales"]), n_act * pb["nibbles"]


def describe(wl, k):
    projs = ", ".join(f"{p.name} K={p.K} N={p.N}" for p in wl.projections)
    return (f"{wl.name}: {wl.note}; E={wl.E}, top_k={k}, {projs}, T in {list(wl.T)}, "
            f"{wl.fmt}, routing {wl.routing}")


# --------------------------------------------------------------------------
# clocks sampled during the timed region
# --------------------------------------------------------------------------
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu_index = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu_index}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = []
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) >= 9:
                rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        return {"sm_mhz": float(np.median(sm)) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons, "samples": len(rows)}


# --------------------------------------------------------------------------
# replicas across ranks (one process per GPU; no collective on the data path)
# --------------------------------------------------------------------------
def max_over_ranks(values, device):
    """The per-rank timings, each replaced by its maximum over all ranks (the job
    takes as long as its slowest replica). Every rank calls this once, in the same
    order; with one rank it returns the values unchanged."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return [float(v) for v in values]
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t.cpu()]


def replica_rate(world, work_per_rank, seconds):
    """Whole-job rate of `world` replicas that each did `work_per_rank` units in
    `seconds` (the max over ranks): weak scaling, work grows with the ranks."""
    return world * work_per_rank / seconds


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d.get("hbm_gbs", 6650.0), d.get("bf16_tflops", 1590.0), \
            d.get("bf16_tflops_sustained", 1400.0), "measured"
    return 6650.0, 1590.0, 1400.0, "fallback"


def _code_only(text):
    """C++/CUDA source without comments and whitespace: what a kernel is made of."""
    out, i, n = [], 0, len(text)
    while i < n:
        if text.startswith("//", i):
            j = text.find("\n", i)
            i = n if j < 0 else j
        elif text.startswith("/*", i):
            j = text.find("*/", i + 2)
            i = n if j < 0 else j + 2
        elif text[i] in "\"'":
            q, j = text[i], i + 1
            while j < n and text[j] != q:
                j += 2 if text[j] == "\\" else 1
            out.append(text[i:j + 1])
            i = j + 1
        else:
            if not text[i].isspace():
                out.append(text[i])
            i += 1
    return "".join(out)


def kernel_source_hash(names):
    """Hash of the kernel sources' code (comments and whitespace do not count)."""
    h = hashlib.sha256()
    for n in names:
        text = open(os.path.join(ROOT, "bit_grouped_moe_gnf4_b200", "csrc", n), encoding="utf-8").read()
        h.update(_code_only(text).encode())
    return h.hexdigest()[:16]


def recorded_traffic(kernel, workload):
    """DRAM bytes per launch from a committed ncu summary, if it was taken on the
    current kernel source (else None)."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    d = json.load(open(p)).get(f"{kernel}:{workload}")
    if not d:
        return None
    if d.get("source_hash") != kernel_source_hash(d.get("sources", [])):
        return None
    return d.get("bytes_per_launch")


# --------------------------------------------------------------------------
# the oracle on the host cores (CPU baseline and the reference arm)
# --------------------------------------------------------------------------
def oracle_sample(wl, calls, budget_s=15.0, seed=0):
    """Run the oracle's grouped GEMM over whole calls of the step (smallest token
    counts first) until ~budget_s of host time. The oracle's own quantization of
    the inputs is untimed. Returns (bytes, flops, calls, gemm_seconds, cores)."""
    from oracle import gnf4_oracle as O
    from synth import generators as G
    try:
        from threadpoolctl import threadpool_info
        cores = max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    except Exception:
        cores = 1
    done_bytes = done_flop = gemm_s = 0.0
    ncalls = 0
    t_begin = time.perf_counter()
    sdiv = 64 if wl.fmt == "nf4" else 32
    q = O.quantize_nf4 if wl.fmt == "nf4" else O.quantize_mxfp4
    for T, proj, b in sorted(calls, key=lambda c: c[0]):
        Wh = np.zeros((wl.E, proj.N, proj.K // 2), np.uint8)
        Sh = np.zeros((wl.E, proj.N, proj.K // sdiv), np.float32 if wl.fmt == "nf4" else np.uint8)
        for e in b.active_experts():
            Wh[e], Sh[e] = q(G.expert_weights(seed, int(e), proj.N, proj.K))
        if proj.name == "gate_up":
            x = synth.activations_bf16(seed, T, proj.K)
            tok = b.row_token
            if wl.gate_up_input == "a_cat":
                x, tok = x[b.row_token], None          # rows already in routed order
            t1 = time.perf_counter()
            O.grouped_gemm(wl.fmt, x, Wh, Sh, b.offsets, tok, None, None, T_out=b.R)
        else:
            x = synth.activations_bf16(seed, b.R, proj.K, tag="x_down")
            t1 = time.perf_counter()
            O.grouped_gemm(wl.fmt, x, Wh, Sh, b.offsets, None, b.row_weight, b.row_dest, T_out=T * b.k)
        gemm_s += time.perf_counter() - t1
        nb, _ = call_bytes(wl.fmt, proj, b)
        done_bytes += nb
        done_flop += 2.0 * b.R * proj.N * proj.K
        ncalls += 1
        if time.perf_counter() - t_begin > budget_s:
            break
    return done_bytes, done_flop, ncalls, gemm_s, cores


def oracle_one_core(wl, calls, seed, prefill, budget_s=4.0):
    """The same oracle sample with its BLAS limited to one thread (None if that limit
    cannot be set): the single-core figure beside the all-cores one."""
    try:
        from threadpoolctl import threadpool_limits
        with threadpool_limits(limits=1):
            nb, nf, nc, dt, _ = oracle_sample(wl, calls, budget_s=budget_s, seed=seed)
        return (nf / dt / 1e12) if prefill else (nb / dt / 1e9)
    except Exception:
        return None


def run_reference(args, wl):
    """The reference arm: the oracle as it stands, timed on the host cores."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    calls, k = workload_calls(wl, args.seed, args.top_k, _tokens(args))
    prefill = wl.name in PREFILL_WORKLOADS
    from oracle import gnf4_oracle as O  # noqa: F401
    times, vals = [], []
    cores = 1
    for i in range(args.warmup + args.steps):
        nb, nf, nc, dt, cores = oracle_sample(wl, calls, budget_s=4.0, seed=args.seed)
        if i >= args.warmup:
            times.append(dt)
            vals.append((nf / dt / 1e12) if prefill else (nb / dt / 1e9))
    v = float(np.median(vals))
    unit = "TFLOP/s" if prefill else "GB/s"
    line = {"metric": METRIC, "value": v, "unit": unit, "n_gpus": args.gpus, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": 1e3 * float(np.median(times)),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "impl": "reference",
            "config": {"workload": describe(wl, k), "l2": "n/a (host)"},
            "cpu_baseline": {"value": v, "unit": unit, "cores": cores, "kind": "oracle",
                             "sample": "per step: whole grouped GEMM calls of the workload, smallest "
                                       "token counts first, until ~4 s of host work; the rate counts "
                                       "the oracle's grouped GEMM time only (its input quantization "
                                       "is untimed)"},
            "e2e": {"value": v, "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def _tokens(args):
    return [int(t) for t in args.tokens.split(",")] if args.tokens else None


# --------------------------------------------------------------------------
# our arm
# --------------------------------------------------------------------------
# the other halves of the metric, measured after the headline step in the same run:
# the tensor-bound prefill workload and the MXFP4 decode workload
SUB_RECORDS = (("prefill", "qwen3_prefill_nf4"), ("mxfp4", "gptoss_mxfp4"))


def run_ours(args, wl):
    import torch
    import torch.distributed as dist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        torch.cuda.set_device(local)
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120))
    dev = torch.device("cuda", torch.cuda.current_device())
    line = measure_step(args, wl, dev, world, rank, headline=True)
    if wl.name == DEFAULT_WORKLOAD and not args.no_sub_records and not args.tokens and args.top_k is None:
        for key, name in SUB_RECORDS:
            sub = measure_step(args, WORKLOADS[name], dev, world, rank, headline=False)
            line[key] = {k2: sub[k2] for k2 in ("value", "unit", "ms_per_step", "dtype", "config",
                                                "roofline", "clocks", "gpu_launches")}
            torch.cuda.empty_cache()
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def measure_step(args, wl, dev, world, rank, headline=True):
    """Time the workload's step (every call, one CUDA graph a step; the per-call
    launch durations in a second pass, one graph a call) and build its
    JSON record. The headline record also carries the end-to-end figure and the CPU
    baseline; a sub-record (another half of the metric) carries neither. Every rank
    calls this the same number of times in the same order (max over ranks inside)."""
    import torch
    import torch.distributed as dist
    import bit_grouped_moe_gnf4_b200 as g

    stream = torch.cuda.current_stream()
    prefill = wl.name in PREFILL_WORKLOADS
    tokens = _tokens(args) if headline else None
    top_k = args.top_k if headline else None
    absmax = args.absmax if (headline and wl.fmt == "nf4") else "f32"
    xf16 = headline and args.x_dtype == "f16"
    xdt = torch.float16 if xf16 else torch.bfloat16

    calls, k = workload_calls(wl, args.seed, top_k, tokens)
    props = torch.cuda.get_device_properties(dev)
    l2 = getattr(props, "L2_cache_size", 126 * 2 ** 20) or 126 * 2 ** 20

    # weight stacks per projection, drawn on the device, quantized by the library
    gen = torch.Generator(device=dev)
    gen.manual_seed(args.seed + 1000 * rank)
    stacks = {}
    stack_bytes = 0
    for proj in wl.projections:
        Wl, Sl = [], []
        for e in range(wl.E):
            w = torch.randn((proj.N, proj.K), generator=gen, device=dev, dtype=torch.float32) * 0.02
            if wl.fmt == "nf4" and absmax == "bf16":
                p, s = g.quantize_nf4(w.to(torch.bfloat16).to(torch.float32))   # a bf16 source
                s = g.absmax_to_bf16(s)                                         # lossless: exact cast
            elif wl.fmt == "nf4":
                p, s = g.quantize_nf4(w)
            else:
                p, s = g.quantize_mxfp4(w)
            Wl.append(p)
            Sl.append(s)
        W = torch.stack(Wl)
        S = torch.stack(Sl)
        del Wl, Sl
        stacks[proj.name] = [(W, S)]
        stack_bytes += W.numel() + S.numel() * S.element_size()
    # copies so that two uses of one copy are > 2 x L2 apart
    step_bytes = sum(call_bytes(wl.fmt, p, b, absmax)[0] for _, p, b in calls)
    ncopies = max(1, min(8, int(np.ceil(2.0 * l2 / max(1, step_bytes))) + 1))
    free = torch.cuda.mem_get_info(dev)[0]
    while ncopies > 1 and (ncopies - 1) * stack_bytes > 0.5 * free:
        ncopies -= 1
    for proj in wl.projections:
        W, S = stacks[proj.name][0]
        for _ in range(ncopies - 1):
            stacks[proj.name].append((W.clone(), S.clone()))

    # per-call device inputs, outputs and pinned host mirrors (end-to-end leg)
    prepared = []
    for T, proj, b in calls:
        if proj.name == "gate_up":
            xb = synth.activations_bf16(args.seed, T, proj.K)
            tok, wt, dst, T_out = b.row_token, None, None, b.R
            if wl.gate_up_input == "a_cat":
                xb, tok = np.ascontiguousarray(xb[b.row_token]), None   # rows already in routed order
        else:
            xb = synth.activations_bf16(args.seed, b.R, proj.K, tag="x_down")
            tok, wt, dst, T_out = None, b.row_weight, b.row_dest, T * b.k
        if xf16:      # the same draw, rounded to fp16 instead
            xb = torch.from_numpy(xb.view(np.int16)).view(torch.bfloat16).float().to(torch.float16).numpy().view(np.uint16)
        xh = torch.from_numpy(xb.view(np.int16)).view(xdt).pin_memory()
        h = {"x": xh, "off": torch.from_numpy(b.offsets).pin_memory()}
        for nm, a in (("tok", tok), ("wt", wt), ("dst", dst)):
            h[nm] = None if a is None else torch.from_numpy(np.ascontiguousarray(a)).pin_memory()
        d = {nm: (None if t is None else t.to(dev)) for nm, t in h.items()}
        out = torch.zeros((T_out, proj.N), dtype=xdt, device=dev)
        outh = torch.empty((T_out, proj.N), dtype=xdt).pin_memory()
        nb, nn = call_bytes(wl.fmt, proj, b, absmax)
        prepared.append(dict(T=T, proj=proj, b=b, h=h, d=d, out=out, outh=outh, bytes=nb, nib=nn,
                             flop=2.0 * b.R * proj.N * proj.K))

    fn = g.grouped_gemm

    def one_call(c, copy):
        W, S = stacks[c["proj"].name][copy]
        d = c["d"]
        fn(wl.fmt, d["x"], W, S, d["off"], row_token=d["tok"], row_weight=d["wt"], row_dest=d["dst"],
           out=c["out"], R=c["b"].R, stream=torch.cuda.current_stream())

    # warm-up through the public call
    for i in range(args.warmup):
        for c in prepared:
            one_call(c, i % ncopies)
    torch.cuda.synchronize()
    g.device_status()

    # each (call, weight copy) captured once as a CUDA graph, so the timed region
    # measures device time, not the host's per-call argument checks; and each step
    # (every call, one weight copy) as one graph, as a serving loop replays a decode
    # step: the step's kernels run back to back (programmatic dependent launches), and
    # the headline is timed on these
    graphs, step_graphs = {}, {}
    cap = torch.cuda.Stream()
    for j, c in enumerate(prepared):
        for copy in range(ncopies):
            gr = torch.cuda.CUDAGraph()
            with torch.cuda.graph(gr, stream=cap, capture_error_mode="thread_local"):
                one_call(c, copy)
            graphs[(j, copy)] = gr
    for copy in range(ncopies):
        gr = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gr, stream=cap, capture_error_mode="thread_local"):
            for c in prepared:
                one_call(c, copy)
        step_graphs[copy] = gr
    torch.cuda.synchronize()
    for gr in list(graphs.values()) + list(step_graphs.values()):    # upload each graph once, untimed
        gr.replay()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()

    launches_per_step = sum(g.launches_per_call(c["b"].R) for c in prepared)
    ev_calls = [[(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                 for _ in prepared] for _ in range(args.steps)]
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(dev.index)
    clocks.start()
    time.sleep(0.3)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    # the headline: K steps, one step graph each
    torch.cuda._sleep(int(2e6))          # let the host queue the whole timed region ahead of the GPU
    t_start.record(stream)
    for i in range(args.steps):
        step_graphs[(args.warmup + i) % ncopies].replay()
    t_end.record(stream)
    torch.cuda.synchronize()
    # the per-call breakdown (launch durations of the kernel): the same K steps, each
    # call's graph between two events
    torch.cuda._sleep(int(2e6))
    for i in range(args.steps):
        copy = (args.warmup + i) % ncopies
        for j in range(len(prepared)):
            ev_calls[i][j][0].record(stream)
            graphs[(j, copy)].replay()
            ev_calls[i][j][1].record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clk = clocks.stop()
    g.device_status()
    total_ms = t_start.elapsed_time(t_end)
    call_ms = np.array([[s.elapsed_time(e) for (s, e) in row] for row in ev_calls])  # [steps, calls]
    del graphs, step_graphs

    # end-to-end: host buffers in, result back, through the same public call
    e2e_steps = max(3, min(args.steps, 10)) if headline else 1
    h2d = sum(sum(t.numel() * t.element_size() for t in c["h"].values() if t is not None) for c in prepared)
    d2h = sum(c["outh"].numel() * 2 for c in prepared)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    e0.record(stream)
    for i in range(e2e_steps):
        copy = i % ncopies
        for c in prepared:
            for nm, t in c["h"].items():
                if t is not None:
                    c["d"][nm].copy_(t, non_blocking=True)
            one_call(c, copy)
            c["outh"].copy_(c["out"], non_blocking=True)
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = e0.elapsed_time(e1) / e2e_steps

    # max over ranks
    ms_step, e2e_ms = max_over_ranks([total_ms / args.steps, e2e_ms], dev)

    work_bytes = sum(c["bytes"] for c in prepared)
    work_flop = sum(c["flop"] for c in prepared)
    if prefill:
        value = replica_rate(world, work_flop, ms_step * 1e-3) / 1e12
        e2e_v = replica_rate(world, work_flop, e2e_ms * 1e-3) / 1e12
        unit = "TFLOP/s"
    else:
        value = replica_rate(world, work_bytes, ms_step * 1e-3) / 1e9
        e2e_v = replica_rate(world, work_bytes, e2e_ms * 1e-3) / 1e9
        unit = "GB/s"

    hbm, tc_burst, tc_sust, src = measured_peaks()
    mean_call_ms = call_ms.mean(axis=0)
    if prefill:
        achieved = work_flop / (call_ms.sum(axis=1).mean() * 1e-3) / 1e12
        roof = {"bound": "tensor", "achieved": achieved, "peak": tc_sust, "unit": "TFLOP/s",
                "frac": achieved / tc_sust, "peak_source": f"{src} bf16 sustained (kernel inside a step)"}
    else:
        achieved = work_bytes / (call_ms.sum(axis=1).mean() * 1e-3) / 1e9
        roof = {"bound": "hbm", "achieved": achieved, "peak": hbm, "unit": "GB/s",
                "frac": achieved / hbm, "peak_source": f"{src} HBM copy"}
    roof["traffic"] = recorded_traffic("decode_band" if not prefill else "prefill_band", wl.name)
    roof["kernel"] = "prefill_band_kernel" if prefill else "decode_band_kernel"
    roof["per_call_ms"] = [round(float(x), 5) for x in mean_call_ms]
    roof["per_call"] = [f"T={c['T']} {c['proj'].name}" for c in prepared]
    # the same step counted on the 4-bit codes alone (no scale bytes)
    work_nib = sum(c["nib"] for c in prepared)
    roof["nibble_only_gbs"] = work_nib / (call_ms.sum(axis=1).mean() * 1e-3) / 1e9

    line = {
        "metric": METRIC, "value": value, "unit": unit, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f16" if xf16 else "bf16", "data": "synthetic",
        "config": {"workload": describe(wl, k), "format": wl.fmt, "absmax": absmax if wl.fmt == "nf4" else "e8m0",
                   "activations": "f16" if xf16 else "bf16",
                   "algorithmic_bytes_per_step": work_bytes, "nibble_bytes_per_step": work_nib,
                   "flop_per_step": work_flop,
                   "l2": f"rotating {ncopies} weight-stack copies ({ncopies * stack_bytes / 1e6:.0f} MB; "
                         f"step reads {step_bytes / 1e6:.0f} MB; L2 {l2 / 1e6:.0f} MB)",
                   "parallelism": f"replicas x{world}",
                   "timing": "value: one CUDA graph a step (the calls back to back); roofline: the "
                             "same steps again, one graph a call between events"},
        "gpu_launches": launches_per_step * args.steps,
        "e2e": {"value": e2e_v, "unit": unit, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "roofline": roof,
        "clocks": clk,
    }
    if headline and rank == 0 and world == 1 and not args.no_cpu_baseline:
        nb, nf, nc, dt, cores = oracle_sample(wl, [(c["T"], c["proj"], c["b"]) for c in prepared],
                                              budget_s=12.0, seed=args.seed)
        v = (nf / dt / 1e12) if prefill else (nb / dt / 1e9)
        line["cpu_baseline"] = {"value": v, "unit": unit, "cores": cores, "kind": "oracle",
                                "sample": f"{nc} whole grouped GEMM calls of the step (smallest token "
                                          f"counts first); {dt:.1f} s in the oracle's grouped GEMM, "
                                          f"its quantization of the inputs untimed"}
        one = oracle_one_core(wl, [(c["T"], c["proj"], c["b"]) for c in prepared], args.seed, prefill)
        if one is not None:
            line["cpu_baseline"]["value_one_core"] = one
    if not headline:
        line.pop("e2e", None)
    del stacks, prepared
    return line


# --------------------------------------------------------------------------
# the glue kernels either side of the GEMM (SwiGLU, top-k combine)
# --------------------------------------------------------------------------
def glue_problem(op, wl, k, T):
    """(input rows, input width, output rows, output width, algorithmic bytes) of one call."""
    gu, dn = wl.projections
    if op == "swiglu":
        R, I = T * k, gu.N // 2
        return R, 2 * I, R, I, R * 2 * I * 2 + R * I * 2
    H = dn.N
    return T * k, H, T, H, T * k * H * 2 + T * H * 2


def glue_oracle(op, x_bits, T, k):
    from oracle import glue as GL
    return GL.swiglu_rows(x_bits) if op == "swiglu" else GL.combine_topk(x_bits, T, k)


def glue_oracle_rate(op, wl, k, T, seed, budget_s):
    """Oracle bytes/s on whole tokens of the call, repeated until ~budget_s."""
    rin, win, rout, wout, nbytes = glue_problem(op, wl, k, T)
    x = synth.activations_bf16(seed, rin, win, tag="h" if op == "swiglu" else "y")
    try:
        from threadpoolctl import threadpool_info
        cores = max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    except Exception:
        cores = 1
    done, t0 = 0, time.perf_counter()
    while True:
        glue_oracle(op, x, T, k)
        done += 1
        if time.perf_counter() - t0 > budget_s:
            break
    dt = time.perf_counter() - t0
    return done * nbytes / dt / 1e9, cores, done, dt


def run_glue(args, wl):
    import torch
    import torch.distributed as dist
    import bit_grouped_moe_gnf4_b200 as g

    op = args.op
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    k = args.top_k if args.top_k is not None else wl.top_k[-1]
    T = max(_tokens(args) or wl.T)
    rin, win, rout, wout, nbytes = glue_problem(op, wl, k, T)
    if args.impl == "reference":
        if rank != 0:
            return
        vals = []
        for i in range(args.warmup + args.steps):
            v, cores, done, dt = glue_oracle_rate(op, wl, k, T, args.seed, 1.0)
            if i >= args.warmup:
                vals.append(v)
        v = float(np.median(vals))
        print(json.dumps({
            "metric": GLUE_OPS[op], "value": v, "unit": "GB/s", "n_gpus": args.gpus, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": nbytes / (v * 1e9) * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64" if op == "swiglu" else "f32",
            "data": "synthetic", "impl": "reference",
            "config": {"workload": f"{op} of {wl.name}: T={T}, top_k={k}, in [{rin}, {win}] -> out [{rout}, {wout}]"},
            "cpu_baseline": {"value": v, "unit": "GB/s", "cores": cores, "kind": "oracle",
                             "sample": "per step: whole calls repeated for ~1 s"},
            "e2e": {"value": v, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}), flush=True)
        return

    if world > 1:
        torch.cuda.set_device(local)
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120))
    dev = torch.device("cuda", torch.cuda.current_device())
    stream = torch.cuda.current_stream()
    props = torch.cuda.get_device_properties(dev)
    l2 = getattr(props, "L2_cache_size", 126 * 2 ** 20) or 126 * 2 ** 20

    xb = synth.activations_bf16(args.seed + rank, rin, win, tag="h" if op == "swiglu" else "y")
    xh = torch.from_numpy(xb.view(np.int16)).view(torch.bfloat16).pin_memory()
    outh = torch.empty((rout, wout), dtype=torch.bfloat16).pin_memory()
    # inputs larger than L2 between two uses of one copy, else an L2 flush between calls
    ncopies = max(1, min(8, int(np.ceil(2.0 * l2 / nbytes)) + 1))
    flush = ncopies * nbytes < 2 * l2
    if flush:
        ncopies = 1
    xs = [xh.to(dev) for _ in range(ncopies)]
    outs = [torch.empty((rout, wout), dtype=torch.bfloat16, device=dev) for _ in range(ncopies)]
    scratch = torch.empty(int(2 * l2) // 4, dtype=torch.float32, device=dev) if flush else None

    def call(j):
        # the current stream: inside graph capture that is the capturing stream
        if op == "swiglu":
            g.swiglu(xs[j], out=outs[j], stream=torch.cuda.current_stream())
        else:
            g.combine_topk(xs[j], T, k, out=outs[j], stream=torch.cuda.current_stream())

    for i in range(args.warmup):
        call(i % ncopies)
    torch.cuda.synchronize()
    g.device_status()
    graphs = []
    cap = torch.cuda.Stream()
    for j in range(ncopies):
        gr = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gr, stream=cap, capture_error_mode="thread_local"):
            call(j)
        graphs.append(gr)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    clocks = ClockSampler(dev.index)
    clocks.start()
    time.sleep(0.3)
    torch.cuda.synchronize()
    torch.cuda._sleep(int(2e6))
    for i in range(args.steps):
        if flush:
            scratch.fill_(float(i))
        evs[i][0].record(stream)
        graphs[i % ncopies].replay()
        evs[i][1].record(stream)
    torch.cuda.synchronize()
    clk = clocks.stop()
    g.device_status()
    call_ms = np.array([a.elapsed_time(b) for a, b in evs])
    del graphs

    # end to end: pinned host input in, result back, through the public call
    e2e_steps = max(3, min(args.steps, 10))
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    e0.record(stream)
    for i in range(e2e_steps):
        xs[0].copy_(xh, non_blocking=True)
        call(0)
        outh.copy_(outs[0], non_blocking=True)
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = e0.elapsed_time(e1) / e2e_steps

    ms, e2e_ms = max_over_ranks([float(call_ms.mean()), e2e_ms], dev)
    value = replica_rate(world, nbytes, ms * 1e-3) / 1e9
    hbm, _, _, src = measured_peaks()
    kernel = "swiglu_kernel" if op == "swiglu" else "combine_kernel"
    line = {
        "metric": GLUE_OPS[op], "value": value, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f32" if op == "combine" else "f32 (bf16 in/out)",
        "data": "synthetic",
        "config": {"workload": f"{op} of {wl.name}: T={T}, top_k={k}, in [{rin}, {win}] bf16 -> "
                               f"out [{rout}, {wout}] bf16",
                   "algorithmic_bytes_per_step": nbytes,
                   "l2": (f"L2 flushed ({scratch.numel() * 4 / 1e6:.0f} MB write) before each call" if flush
                          else f"rotating {ncopies} input copies ({ncopies * nbytes / 1e6:.0f} MB of traffic "
                               f"per rotation; L2 {l2 / 1e6:.0f} MB)"),
                   "parallelism": f"replicas x{world}"},
        "gpu_launches": args.steps,
        "e2e": {"value": replica_rate(world, nbytes, e2e_ms * 1e-3) / 1e9, "unit": "GB/s",
                "h2d_bytes_per_step": xh.numel() * 2, "d2h_bytes_per_step": outh.numel() * 2},
        "roofline": {"bound": "hbm", "achieved": nbytes / (ms * 1e-3) / 1e9, "peak": hbm, "unit": "GB/s",
                     "frac": nbytes / (ms * 1e-3) / 1e9 / hbm, "peak_source": f"{src} HBM copy",
                     "traffic": recorded_traffic(kernel, wl.name), "kernel": kernel},
        "clocks": clk,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        v, cores, done, dt = glue_oracle_rate(op, wl, k, T, args.seed, 10.0)
        line["cpu_baseline"] = {"value": v, "unit": "GB/s", "cores": cores, "kind": "oracle",
                                "sample": f"{done} whole calls of the oracle ({dt:.1f} s)"}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


# --------------------------------------------------------------------------
# the input gradient of the step's grouped GEMM calls
# --------------------------------------------------------------------------
def dgrad_oracle_rate(wl, calls, budget_s, seed):
    """Oracle rate (bytes/s or flop/s) of the input gradient on whole calls, smallest first."""
    from oracle import dgrad as D
    from oracle import gnf4_oracle as O
    from synth import generators as G
    q = O.quantize_nf4 if wl.fmt == "nf4" else O.quantize_mxfp4
    sdiv = 64 if wl.fmt == "nf4" else 32
    done_b = done_f = secs = 0.0
    n = 0
    t_begin = time.perf_counter()
    for T, proj, b in sorted(calls, key=lambda c: c[0]):
        Wh = np.zeros((wl.E, proj.N, proj.K // 2), np.uint8)
        Sh = np.zeros((wl.E, proj.N, proj.K // sdiv), np.float32 if wl.fmt == "nf4" else np.uint8)
        for e in b.active_experts():
            Wh[e], Sh[e] = q(G.expert_weights(seed, int(e), proj.N, proj.K))
        src, wt, gb = dgrad_call_inputs(proj, b, seed)
        t1 = time.perf_counter()
        D.dgrad(wl.fmt, gb, Wh, Sh, b.offsets, src, wt)
        secs += time.perf_counter() - t1
        done_b += call_bytes(wl.fmt, proj, b)[0]
        done_f += 2.0 * b.R * proj.N * proj.K
        n += 1
        if time.perf_counter() - t_begin > budget_s:
            break
    return done_b, done_f, n, secs


def dgrad_call_inputs(proj, b, seed):
    """(row_src, row_weight, gradient bits) of the input gradient of one forward call:
    down scattered row r to t*k + slot with weight w(r), gate_up wrote row r."""
    if proj.name == "down":
        return b.row_dest, b.row_weight, synth.activations_bf16(seed, b.T * b.k, proj.N, tag="y")
    return None, None, synth.activations_bf16(seed, b.R, proj.N, tag="y")


def run_dgrad_bench(args, wl):
    import torch
    import torch.distributed as dist
    import bit_grouped_moe_gnf4_b200 as g

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    prefill = wl.name in PREFILL_WORKLOADS
    calls, k = workload_calls(wl, args.seed, args.top_k, _tokens(args))
    unit = "TFLOP/s" if prefill else "GB/s"
    metric = ("grouped 4-bit MoE GEMM input gradient (grad_out @ dequant(W)): packed-weight GB/s "
              "(decode), TFLOP/s (prefill)")
    if args.impl == "reference":
        if rank != 0:
            return
        vals = []
        for i in range(args.warmup + args.steps):
            nb, nf, n, dt = dgrad_oracle_rate(wl, calls, 4.0, args.seed)
            if i >= args.warmup:
                vals.append(nf / dt / 1e12 if prefill else nb / dt / 1e9)
        v = float(np.median(vals))
        print(json.dumps({"metric": metric, "value": v, "unit": unit, "n_gpus": args.gpus,
                          "steps": args.steps, "warmup": args.warmup, "ms_per_step": None,
                          "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
                          "dtype": "f64", "data": "synthetic", "impl": "reference",
                          "config": {"workload": "dgrad of " + describe(wl, k)},
                          "cpu_baseline": {"value": v, "unit": unit, "cores": None, "kind": "oracle",
                                           "sample": "per step: whole calls, smallest first, ~4 s"},
                          "e2e": {"value": v, "unit": unit, "h2d_bytes_per_step": 0,
                                  "d2h_bytes_per_step": 0}}), flush=True)
        return

    if world > 1:
        torch.cuda.set_device(local)
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120))
    dev = torch.device("cuda", torch.cuda.current_device())
    stream = torch.cuda.current_stream()
    props = torch.cuda.get_device_properties(dev)
    l2 = getattr(props, "L2_cache_size", 126 * 2 ** 20) or 126 * 2 ** 20
    gen = torch.Generator(device=dev)
    gen.manual_seed(args.seed + 1000 * rank)
    stacks, stack_bytes = {}, 0
    for proj in wl.projections:
        Wl, Sl = [], []
        for e in range(wl.E):
            w = torch.randn((proj.N, proj.K), generator=gen, device=dev, dtype=torch.float32) * 0.02
            p_, s_ = g.quantize_nf4(w) if wl.fmt == "nf4" else g.quantize_mxfp4(w)
            Wl.append(p_)
            Sl.append(s_)
        stacks[proj.name] = [(torch.stack(Wl), torch.stack(Sl))]
        stack_bytes += stacks[proj.name][0][0].numel() + stacks[proj.name][0][1].numel() * \
            stacks[proj.name][0][1].element_size()
        del Wl, Sl
    step_bytes = sum(call_bytes(wl.fmt, p_, b)[0] for _, p_, b in calls)
    ncopies = max(1, min(8, int(np.ceil(2.0 * l2 / max(1, step_bytes))) + 1))
    free = torch.cuda.mem_get_info(dev)[0]
    while ncopies > 1 and (ncopies - 1) * stack_bytes > 0.5 * free:
        ncopies -= 1
    for proj in wl.projections:
        W0, S0 = stacks[proj.name][0]
        for _ in range(ncopies - 1):
            stacks[proj.name].append((W0.clone(), S0.clone()))

    prepared = []
    for T, proj, b in calls:
        src, wt, gb = dgrad_call_inputs(proj, b, args.seed)
        h = {"g": torch.from_numpy(gb.view(np.int16)).view(torch.bfloat16).pin_memory(),
             "off": torch.from_numpy(b.offsets).pin_memory(),
             "src": None if src is None else torch.from_numpy(np.ascontiguousarray(src)).pin_memory(),
             "wt": None if wt is None else torch.from_numpy(np.ascontiguousarray(wt)).pin_memory()}
        d = {nm: (None if t is None else t.to(dev)) for nm, t in h.items()}
        out = torch.empty((b.R, proj.K), dtype=torch.bfloat16, device=dev)
        outh = torch.empty((b.R, proj.K), dtype=torch.bfloat16).pin_memory()
        prepared.append(dict(T=T, proj=proj, b=b, h=h, d=d, out=out, outh=outh,
                             bytes=call_bytes(wl.fmt, proj, b)[0], flop=2.0 * b.R * proj.N * proj.K))

    def one_call(c, copy):
        W_, S_ = stacks[c["proj"].name][copy]
        d = c["d"]
        g.dgrad(wl.fmt, d["g"], W_, S_, d["off"], row_src=d["src"], row_weight=d["wt"], R=c["b"].R,
                out=c["out"], stream=torch.cuda.current_stream())

    for i in range(args.warmup):
        for c in prepared:
            one_call(c, i % ncopies)
    torch.cuda.synchronize()
    g.device_status()
    graphs = {}
    cap = torch.cuda.Stream()
    for j, c in enumerate(prepared):
        for copy in range(ncopies):
            gr = torch.cuda.CUDAGraph()
            with torch.cuda.graph(gr, stream=cap, capture_error_mode="thread_local"):
                one_call(c, copy)
            graphs[(j, copy)] = gr
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    ev = [[(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in prepared] for _ in range(args.steps)]
    clocks = ClockSampler(dev.index)
    clocks.start()
    time.sleep(0.3)
    torch.cuda.synchronize()
    torch.cuda._sleep(int(2e6))
    for i in range(args.steps):
        copy = (args.warmup + i) % ncopies
        for j in range(len(prepared)):
            ev[i][j][0].record(stream)
            graphs[(j, copy)].replay()
            ev[i][j][1].record(stream)
    torch.cuda.synchronize()
    clk = clocks.stop()
    g.device_status()
    call_ms = np.array([[a.elapsed_time(b_) for (a, b_) in row] for row in ev])
    del graphs

    e2e_steps = max(3, min(args.steps, 10))
    h2d = sum(sum(t.numel() * t.element_size() for t in c["h"].values() if t is not None) for c in prepared)
    d2h = sum(c["outh"].numel() * 2 for c in prepared)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    e0.record(stream)
    for i in range(e2e_steps):
        for c in prepared:
            for nm, t in c["h"].items():
                if t is not None:
                    c["d"][nm].copy_(t, non_blocking=True)
            one_call(c, i % ncopies)
            c["outh"].copy_(c["out"], non_blocking=True)
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = e0.elapsed_time(e1) / e2e_steps

    ms_step, e2e_ms = max_over_ranks([float(call_ms.sum(axis=1).mean()), e2e_ms], dev)
    work_b = sum(c["bytes"] for c in prepared)
    work_f = sum(c["flop"] for c in prepared)
    work = work_f / 1e12 if prefill else work_b / 1e9
    hbm, tc_burst, tc_sust, src_ = measured_peaks()
    achieved = work / (ms_step * 1e-3)
    if prefill:
        roof = {"bound": "tensor", "achieved": achieved, "peak": tc_sust, "unit": unit,
                "frac": achieved / tc_sust, "peak_source": f"{src_} bf16 sustained (kernel inside a step)"}
    else:
        roof = {"bound": "hbm", "achieved": achieved, "peak": hbm, "unit": unit, "frac": achieved / hbm,
                "peak_source": f"{src_} HBM copy"}
    roof["traffic"] = recorded_traffic("dgrad_kernel", wl.name)
    roof["kernel"] = "dgrad_kernel"
    roof["per_call_ms"] = [round(float(x), 5) for x in call_ms.mean(axis=0)]
    roof["per_call"] = [f"T={c['T']} {c['proj'].name}" for c in prepared]
    line = {"metric": metric, "value": replica_rate(world, work, ms_step * 1e-3), "unit": unit,
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic",
            "config": {"workload": "dgrad of " + describe(wl, k), "format": wl.fmt,
                       "algorithmic_bytes_per_step": work_b, "flop_per_step": work_f,
                       "l2": f"rotating {ncopies} weight-stack copies", "parallelism": f"replicas x{world}"},
            "gpu_launches": len(prepared) * args.steps,
            "e2e": {"value": replica_rate(world, work, e2e_ms * 1e-3), "unit": unit,
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
            "roofline": roof, "clocks": clk}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        nb, nf, n, dt = dgrad_oracle_rate(wl, calls, 10.0, args.seed)
        try:
            from threadpoolctl import threadpool_info
            cores = max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
        except Exception:
            cores = 1
        line["cpu_baseline"] = {"value": (nf / dt / 1e12) if prefill else (nb / dt / 1e9), "unit": unit,
                                "cores": cores, "kind": "oracle",
                                "sample": f"{n} whole calls of the step, smallest first ({dt:.1f} s of oracle "
                                          f"dgrad; its input quantization untimed)"}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


# --------------------------------------------------------------------------
# one whole MoE layer per token count, captured as one CUDA graph
# --------------------------------------------------------------------------
def run_layer_bench(args, wl):
    import torch
    import bit_grouped_moe_gnf4_b200 as g

    if args.impl == "reference" or int(os.environ.get("WORLD_SIZE", "1")) > 1:
        if int(os.environ.get("RANK", "0")) == 0:
            print(json.dumps({"impl": args.impl, "unavailable": "--op layer is a 1-GPU measurement of "
                              "this library's layer; the oracle's layer is timed by --op gemm/swiglu/combine"}))
        return
    dev = torch.device("cuda", torch.cuda.current_device())
    stream = torch.cuda.current_stream()
    k = args.top_k if args.top_k is not None else wl.top_k[-1]
    Ts = _tokens(args) or list(wl.T)
    gu, dn = wl.projections
    H, I2 = gu.K, gu.N
    gen = torch.Generator(device=dev)
    gen.manual_seed(args.seed)

    def stack(proj):
        Wl, Sl = [], []
        for e in range(wl.E):
            w = torch.randn((proj.N, proj.K), generator=gen, device=dev, dtype=torch.float32) * 0.02
            p_, s_ = g.quantize_nf4(w) if wl.fmt == "nf4" else g.quantize_mxfp4(w)
            Wl.append(p_)
            Sl.append(s_)
        return torch.stack(Wl), torch.stack(Sl)

    Wg, Sg = stack(gu)
    Wd, Sd = stack(dn)
    scratch = torch.empty(64 * 2 ** 20, dtype=torch.float32, device=dev)     # 256 MB: flushes L2
    layers = []
    for T in Ts:
        ids, w = (G_route(wl))(args.seed, T, wl.E, k)
        b = synth.make_routed_batch(args.seed, T, wl.E, k, routing=wl.routing)
        R = T * k
        d = {"ids": torch.from_numpy(ids.astype(np.int32)).to(dev), "w": torch.from_numpy(w).to(dev),
             "x": torch.from_numpy(synth.activations_bf16(args.seed, T, H).view(np.int16)).to(dev).view(torch.bfloat16),
             "h": torch.empty((R, I2), dtype=torch.bfloat16, device=dev),
             "a": torch.empty((R, I2 // 2), dtype=torch.bfloat16, device=dev),
             "y": torch.empty((R, dn.N), dtype=torch.bfloat16, device=dev),
             "out": torch.empty((T, dn.N), dtype=torch.bfloat16, device=dev)}
        nbytes = call_bytes(wl.fmt, gu, b)[0] + call_bytes(wl.fmt, dn, b)[0]
        layers.append((T, d, nbytes, b))

    fused = not args.unfused_swiglu

    def layer(d, T):
        st = torch.cuda.current_stream()
        off, tok, wt, dst = g.routing_metadata(d["ids"], d["w"], wl.E, stream=st)
        if fused:       # gate_up with the SwiGLU in its epilogue: no [R, 2I] round trip
            g.grouped_gemm_swiglu(wl.fmt, d["x"], Wg, Sg, off, row_token=tok, out=d["a"], R=T * k, stream=st)
        else:
            g.grouped_gemm(wl.fmt, d["x"], Wg, Sg, off, row_token=tok, out=d["h"], R=T * k, stream=st)
            g.swiglu(d["h"], out=d["a"], stream=st)
        g.grouped_gemm(wl.fmt, d["a"], Wd, Sd, off, row_weight=wt, row_dest=dst, out=d["y"], R=T * k, stream=st)
        g.combine_topk(d["y"], T, k, out=d["out"], stream=st)

    for _ in range(args.warmup):
        for T, d, _, _ in layers:
            layer(d, T)
    torch.cuda.synchronize()
    g.device_status()
    graphs = []
    cap = torch.cuda.Stream()
    for T, d, _, _ in layers:
        gr = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gr, stream=cap, capture_error_mode="thread_local"):
            layer(d, T)
        graphs.append(gr)
    torch.cuda.synchronize()
    ev = [[(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in layers]
          for _ in range(args.steps)]
    clocks = ClockSampler(dev.index)
    clocks.start()
    time.sleep(0.3)
    torch.cuda.synchronize()
    for i in range(args.steps):
        for j in range(len(layers)):
            scratch.fill_(float(i))                      # L2 flushed before each layer
            ev[i][j][0].record(stream)
            graphs[j].replay()
            ev[i][j][1].record(stream)
    torch.cuda.synchronize()
    clk = clocks.stop()
    g.device_status()
    ms = np.array([[a.elapsed_time(b_) for a, b_ in row] for row in ev]).mean(axis=0)
    tokens = sum(T for T, _, _, _ in layers)
    wbytes = sum(nb for _, _, nb, _ in layers)
    hbm, _, _, src = measured_peaks()
    achieved = wbytes / (ms.sum() * 1e-3) / 1e9
    line = {"metric": "MoE layer (device routing, gate_up, SwiGLU, down, combine): tokens/s",
            "value": tokens / (ms.sum() * 1e-3), "unit": "tokens/s", "n_gpus": 1, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": float(ms.sum()), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": "layer of " + describe(wl, k), "l2": "flushed (256 MB write) before each layer",
                       "swiglu": "fused into the gate_up epilogue" if fused else "separate kernel",
                       "layers": [f"T={T}" for T, _, _, _ in layers]},
            "gpu_launches": (4 if fused else 5) * len(layers) * args.steps,
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": hbm, "unit": "GB/s", "frac": achieved / hbm,
                         "peak_source": f"{src} HBM copy", "traffic": None,
                         "note": "packed-weight bytes of both projections over the whole layer's time",
                         "per_layer_ms": [round(float(x), 5) for x in ms]},
            "clocks": clk}
    print(json.dumps(line), flush=True)


def G_route(wl):
    from synth import generators as G
    return G.route_softmax_topk if wl.routing == "softmax" else G.route_zipf_topk


def main():
    args = parse()
    wl = WORKLOADS[args.workload]
    if args.op == "layer":
        run_layer_bench(args, wl)
        return
    if args.op == "dgrad":
        run_dgrad_bench(args, wl)
        return
    if args.op in GLUE_OPS:
        run_glue(args, wl)
        return
    if args.impl == "reference":
        run_reference(args, wl)
    else:
        run_ours(args, wl)


if __name__ == "__main__":
    main()
