#!/usr/bin/env python
"""Throughput of the block-sparse attention hot path on B200.

One step = the whole hot path over one workload (default: the causal
sliding-window workload, B=1, H=16, Sq=Skv=8192, D=128, window 512, bf16
N(0,1), seed 2):
  a1+a6  block map + rank-sorted column lists      (bsa_plan_build)
  a2     fixed-m bound and per-head gate            (bsa_fixed_m_bound; beside a1)
  a3     forward, fixed-m gated, O residual kept    (bsa_attn_fwd)
  a4     Delta, fp16 copies of Q and dO, semaphores (bsa_bwd_preprocess)
  a5     deterministic backward, descending order   (bsa_bwd_main)
  a7     dQ convert                                 (bsa_bwd_convert)
(the forward-only workloads, varlen and video: a1, a2, a3).
Metric: useful TFLOP/s = (non-empty 128x128 tiles x per-tile flops) / time, with
per-tile flops 4*128*128*D forward and 2.5x that backward.  L2 is flushed
before every step, outside the step's events (class L2Flush).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME] [--softmax fixed_m|online] [--bound norm|smoothed|block]
                    [--order desc|asc|outside_in|greedy] [--nondet] [--o-residual auto|drop]

With N > 1 it runs under torch.distributed.run, one rank per GPU, every rank
running the same workload (replicas: the (b, h) units are independent and
the path has no exchange step); value = work of all ranks / max rank time.
"""

from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

WORKLOAD_NAME = "window"
WORKLOADS = {
    "tiny": "tiny dense: B=1, H=2, Sq=Skv=256, D=64, bf16 N(0,1) seed 0, no mask",
    "packed": "packed segments: B=2, H=8, S=4096, D=128, bf16 N(0,1) seed 1, segment runs of "
              "uniform{256..2048} tokens (block-diagonal)",
    "packed_const": "packed segments with one constant id per batch row (equal to no mask): B=2, H=8, "
                    "S=4096, D=128, bf16 N(0,1) seed 1",
    "window": "causal sliding window 512: B=1, H=16, Sq=Skv=8192, D=128, bf16 N(0,1) seed 2",
    "window_rect": "causal sliding window 512, bottom-right: B=1, H=16, Sq=4096, Skv=8192, D=128, "
                   "bf16 N(0,1) seed 2",
    "varlen": "varlen with alignment padding: H=24, D=128, T=33024, cu_seqlens=[0,33002,33024] "
              "(22 alignment rows), non-causal, bf16 N(0,1) seed 3; forward only",
    "video": "video-DiT: B=1, H=40, Sq=75600 (21x45x80), Skv=75776 (KV padded to a multiple of 2048, "
             "padding masked), D=128, q,k ~ N(0,0.5) + 3-axis RoPE, head 0 with 8 sink keys x20, seed 4; "
             "forward only",
    "prefix_lm": "prefix-LM (causal + bidirectional prefix of 2048): B=1, H=16, Sq=Skv=8192, "
                 "D=128, bf16 N(0,1) seed 2",
    "dilated": "dilated causal window (span 1024, dilation 2): B=1, H=16, Sq=Skv=8192, D=128, "
               "bf16 N(0,1) seed 2",
    "document": "document-causal (runs of 256..2048 tokens): B=1, H=16, Sq=Skv=8192, D=128, "
                "bf16 N(0,1) seed 2",
    "gqa": "grouped-query causal sliding window 512: B=1, H=16 over H_kv=4, Sq=Skv=8192, D=128, "
           "bf16 N(0,1) seed 5",
}
# forward-only workloads (the configs state no backward for them)
FORWARD_ONLY = ("varlen", "video")
# dense bf16 tcgen05 rate per SM and clock (flop), for the spec peak = SMs x max SM clock x rate
BF16_FLOP_PER_CLK_SM = 8192
DATASHEET_BF16_TFLOPS = 2250.0


def workload_text(args):
    fwd = args.softmax + (" gated" if args.softmax == "fixed_m" else "")
    if args.softmax == "fixed_m" and args.bound == "smoothed":
        fwd += ", k-smoothed bound"
    if args.softmax == "fixed_m" and args.bound == "block":
        fwd += " per row, per q-block bound"
    if args.workload in FORWARD_ONLY:
        return f"{WORKLOADS[args.workload]}; forward {fwd}"
    bwd = "atomic (non-deterministic)" if args.nondet else f"deterministic ({args.order} kv-column order)"
    resid = "" if args.o_residual == "auto" else ", no O residual"
    return f"{WORKLOADS[args.workload]}; forward {fwd} + {bwd} backward{resid}"
METRIC = "attention TFLOP/s (non-empty tiles) fwd+bwd on 1 B200; % of bf16 tensor peak"


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--softmax", default="fixed_m", choices=["fixed_m", "online"])
    ap.add_argument("--bound", default="norm", choices=["norm", "smoothed", "block"],
                    help="fixed-m reference: Cauchy-Schwarz on ||k|| (per-head gate), on the centred keys, "
                         "or per q-block over the key blocks it reaches (per-row gate)")
    ap.add_argument("--order", default="desc", choices=["asc", "desc", "outside_in", "greedy"])
    ap.add_argument("--nondet", action="store_true", help="atomic (non-deterministic) dQ backward")
    ap.add_argument("--o-residual", default="auto", choices=["auto", "drop"],
                    help="auto (the library default): the forward keeps O's bf16 rounding residual and "
                         "Delta is exact to the fp32 O; drop: Delta from the bf16 O")
    ap.add_argument("--no-orders", action="store_true",
                    help="skip timing the backward main kernel under every kv-column order and atomically")
    ap.add_argument("--workload", default=WORKLOAD_NAME, choices=sorted(WORKLOADS))
    ap.add_argument("--small", action="store_true",
                    help="small shape of the same workload (for profiler captures)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-graph", action="store_true",
                    help="time the step as eager library calls instead of CUDA-graph replays")
    return ap.parse_args()


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "bf16_tflops_sustained": float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                "source": "measured"}
    except Exception:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                "source": "fallback"}


class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons during the timed region."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        self.lines = []
        if self.proc is not None:
            time.sleep(0.2)
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [l for l in out.splitlines() if l.strip()]
        return False

    def summary(self):
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in getattr(self, "lines", []):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 7:
                continue
            try:
                sm.append(float(parts[0]))
                mx.append(float(parts[1]))
            except ValueError:
                continue
            for n, v in zip(names, parts[3:7]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        loaded = [s for s in sm if s > 0.5 * max(sm)] or sm
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": max(mx),
                "reasons": sorted(reasons), "samples": len(sm)}


def dist_setup(args, backend: str = "nccl"):
    """(world, rank, local rank) from the torchrun environment; with more than
    one rank, joins the process group (NCCL on the GPUs; the CPU tests pass
    gloo) with a short timeout, so that a rank that never arrives ends the
    others' next collective with an error."""
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if torch.cuda.is_available():
        torch.cuda.set_device(local)
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return world, rank, local


def max_over_ranks(x: float, world: int) -> float:
    """The maximum of x over all ranks (every rank takes part and gets it)."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world: int):
    """All ranks meet, and this rank's device work has finished."""
    import torch
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    if torch.cuda.is_available():
        torch.cuda.synchronize()


def window_pairs(wl):
    """Allowed (query, key) pairs of a plain causal-window mask (no other
    predicate), summed over batches and query heads, in closed form: row i sees
    keys (i + o - W, i + o] within [0, Skv) with o = Skv - Sq (all keys up to
    i + o when W = 0).  None for any other mask."""
    import numpy as np
    if set(wl.mask) != {"window"}:
        return None
    W, o = int(wl.mask["window"]), wl.Skv - wl.Sq
    i = np.arange(wl.Sq, dtype=np.int64)
    hi = np.minimum(i + o, wl.Skv - 1)
    lo = np.maximum(i + o - W + 1, 0) if W > 0 else np.zeros_like(i)
    return int(np.maximum(hi - lo + 1, 0).sum()) * wl.B * wl.H


def whole_job_tflops(world: int, steps: int, flops_per_step: float, max_total_ms: float) -> float:
    """value: the work of all ranks (each runs `steps` steps of the same
    workload) over the slowest rank's time for them."""
    return world * steps * flops_per_step / (max_total_ms * 1e-3) / 1e12


def tiles_of(ws):
    ptr, _ = ws.row_lists()
    return int(ptr[-1])


def source_tag(*files) -> str:
    """sha256 prefix of the kernel sources, so that a committed DRAM-traffic
    figure is used only for the kernel build it was measured on."""
    import hashlib
    h = hashlib.sha256()
    for f in files:
        with open(os.path.join(ROOT, "block_sparse_attention_map_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def profiled_traffic(kernel: str, workload: str, src: str):
    """dram bytes per launch of `kernel` on `workload` from the committed ncu
    summary (a line `traffic <kernel> <workload> <bytes> <source tag>`), when it
    was taken on the current kernel source; else None."""
    path = os.path.join(ROOT, "profiles", "traffic.txt")
    try:
        for line in open(path):
            parts = line.split()
            if (len(parts) == 5 and parts[0] == "traffic" and parts[1] == kernel and parts[2] == workload
                    and parts[4] == src):
                return float(parts[3])
    except OSError:
        pass
    return None


# ------------------------------------------------------------------ CPU oracle leg

def oracle_sample(wl, n_rows: int, head: int = 0):
    """Time the fp64 oracle (forward, and backward where the workload has one)
    on query rows and keys [0, n_rows) of one head under the same mask
    predicates; returns (seconds, useful flops credited, threads)."""
    import numpy as np
    import oracle
    try:
        from threadpoolctl import threadpool_info
        threads = max([i.get("num_threads", 1) for i in threadpool_info()] or [os.cpu_count()])
    except Exception:
        threads = os.cpu_count()
    f = lambda t: t.detach().float().cpu().numpy().astype(np.float64)
    hk = head // (wl.H // wl.k.shape[2])
    q = f(wl.q[:, :n_rows, head:head + 1])
    k, v = f(wl.k[:, :n_rows, hk:hk + 1]), f(wl.v[:, :n_rows, hk:hk + 1])
    # the sample treats rows and keys [0, n_rows) as a square problem with the
    # same mask predicates (segment ids and cu_seqlens cut to the sample)
    desc = wl.mask_numpy()
    for key in ("seg_q", "seg_kv"):
        if key in desc:
            desc[key] = desc[key][:, :n_rows]
    if "cu_seqlens" in desc:
        cu = np.minimum(np.asarray(desc["cu_seqlens"]), n_rows)
        desc["cu_seqlens"] = np.unique(cu)
        desc["n_align_tail"] = 0 if cu[-1 - desc["n_align_tail"]] >= n_rows else desc["n_align_tail"]
    if "kv_valid_len" in desc:
        desc["kv_valid_len"] = np.minimum(desc["kv_valid_len"], n_rows)
    sub = oracle.MaskDesc(**desc)
    cls = oracle.tile_classes(sub, 1, n_rows, n_rows)
    t0 = time.perf_counter()
    oracle.attention_forward(q, k, v, sub, wl.scale)
    if wl.backward:
        do = f(wl.dO[:, :n_rows, head:head + 1])
        oracle.attention_backward(q, k, v, do, sub, wl.scale)
    dt = time.perf_counter() - t0
    nnz = int((cls != oracle.EMPTY).sum())
    flops = oracle.useful_flops(nnz, wl.D) * (3.5 if wl.backward else 1.0)
    return dt, flops, threads


def run_reference(args, world, rank):
    """The reference arm: the fp64 oracle, as it stands, on the host cores."""
    import torch
    from block_sparse_attention_map_b200.workloads import make_workload
    if rank != 0:
        return
    wl = make_workload(args.workload, device="cpu", small=args.small)
    n_rows = min(1024, wl.Sq)
    for _ in range(args.warmup):
        oracle_sample(wl, n_rows)
    total_t, total_f, threads = 0.0, 0.0, 1
    for _ in range(args.steps):
        dt, fl, threads = oracle_sample(wl, n_rows)
        total_t += dt
        total_f += fl
    value = total_f / total_t / 1e12
    what = "forward + backward" if wl.backward else "forward"
    sample = (f"rows and keys 0..{n_rows - 1} of head 0 of {wl.H} under the same mask, "
              f"{what} in fp64, per step")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * total_t / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": workload_text(args), "global_batch": wl.B, "seq_len": wl.Sq,
                   "heads": wl.H, "head_dim": wl.D, "mask": wl.mask_text()},
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------ GPU arm

class L2Flush:
    """Empties L2 between timed steps: a 256 MiB write (more than the 126 MB
    L2), then a 256 MiB read of a second buffer.  The write alone leaves L2
    full of dirty lines whose write-back the next step's first kernel would pay
    for; after the read, L2 holds clean lines of the flush buffer only."""

    def __init__(self, dev):
        import torch
        self.w = torch.empty(256 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)
        self.r = torch.zeros(256 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)
        self.acc = torch.zeros((), dtype=torch.float32, device=dev)

    def __call__(self):
        self.w.zero_()
        self.acc.copy_(self.r.sum())


def _median_event_ms(fn, before, n, stream):
    """Median CUDA-event time of fn() over n runs, before() (untimed: an L2 flush,
    a stage the timed one depends on) ahead of each."""
    import torch
    times = []
    for _ in range(n):
        before()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        fn()
        b.record(stream)
        torch.cuda.synchronize()
        times.append(a.elapsed_time(b))
    return statistics.median(times)


def order_table(args, wl, flush, stream, n=10):
    """backward_main (a5) under every kv-column order and the atomic variant,
    measured in this run on this workload: median of n launches, L2 flushed and
    Delta / the semaphores (or the zeroed accumulator) prepared before each."""
    import block_sparse_attention_map_b200 as bsa
    out = {}
    for name in ("asc", "desc", "outside_in", "greedy", "atomic"):
        st = bsa.Stages(wl.q, wl.k, wl.v, wl.mask, softmax_mode=args.softmax,
                        order="desc" if name == "atomic" else name, deterministic=name != "atomic",
                        bound_mode=args.bound, o_residual=args.o_residual)
        st.plan_and_bound()
        st.forward()

        def before():
            flush()
            st.preprocess(wl.dO)

        out[name] = _median_event_ms(lambda: st.backward_main(wl.dO), before, n, stream)
        if st.ws.status() != 0:
            raise RuntimeError(f"device status {st.ws.status()} timing the {name} backward")
        del st
    return out


def softmax_table(args, wl, flush, stream, n=10):
    """The forward (a3) under online and fixed-m softmax, measured in this run:
    median of n launches, L2 flushed before each (plan and bound built once)."""
    import block_sparse_attention_map_b200 as bsa
    out, gates = {}, None
    for mode in ("online", "fixed_m"):
        st = bsa.Stages(wl.q, wl.k, wl.v, wl.mask, softmax_mode=mode, bound_mode=args.bound,
                        o_residual=args.o_residual)
        st.plan_and_bound()
        st.forward()
        fixed_rows = st.ws.fixed_rows()  # one forward since the plan build
        out[mode] = _median_event_ms(st.forward, flush, n, stream)
        if st.ws.status() != 0:
            raise RuntimeError(f"device status {st.ws.status()} timing the {mode} forward")
        if mode == "fixed_m":
            gates = {"fixed_m_rows": fixed_rows, "rows": wl.B * wl.H * wl.Sq}
            if args.bound != "block":
                g = st.ws.gate().cpu()
                gates.update({"fixed_m_heads": int(g.sum()), "online_heads": int(g.numel() - g.sum())})
        del st
    return out, gates


def run_ours(args, world, rank, local):
    import torch
    import block_sparse_attention_map_b200 as bsa
    from block_sparse_attention_map_b200.workloads import make_workload

    dev = torch.device("cuda", local)
    wl = make_workload(args.workload, device=dev, small=args.small)
    has_bwd = wl.backward
    st = bsa.Stages(wl.q, wl.k, wl.v, wl.mask, softmax_mode=args.softmax, order=args.order,
                    deterministic=not args.nondet, bound_mode=args.bound, o_residual=args.o_residual)
    dO = wl.dO
    flush = L2Flush(dev)
    stream = torch.cuda.current_stream()
    # the planner runs beside the bound's pass over Q and K (one library call,
    # the plan on the library's side stream), then the rest in order
    names = ["plan_and_bound", "forward"] + (["preprocess", "backward_main", "convert"] if has_bwd else [])
    calls = {"plan_and_bound": st.plan_and_bound, "forward": st.forward,
             "preprocess": lambda: st.preprocess(dO), "backward_main": lambda: st.backward_main(dO),
             "convert": st.convert}

    def step(ev=None):
        for i, n in enumerate(names):
            if ev is not None:
                ev[i].record(stream)
            calls[n]()
        if ev is not None:
            ev[len(names)].record(stream)

    for _ in range(args.warmup):
        flush()
        step()
    torch.cuda.synchronize()
    status = st.ws.status()
    if status != 0:
        raise RuntimeError(f"device status {status} after warm-up")
    n_tiles = tiles_of(st.ws) * wl.H  # non-empty tiles over all (b, h)
    f_fwd = 4.0 * 128 * 128 * wl.D * n_tiles
    f_bwd = 2.5 * f_fwd if has_bwd else 0.0

    # eager pass: one library call per stage, an event between stages (the
    # per-stage split; every call's host work sits between the launches)
    events = [[torch.cuda.Event(enable_timing=True) for _ in range(len(names) + 1)] for _ in range(args.steps)]
    launches0 = bsa.launch_count()
    barrier(world)
    for s in range(args.steps):
        flush()
        step(events[s])
    torch.cuda.synchronize()
    barrier(world)
    eager_launches = bsa.launch_count() - launches0
    status = st.ws.status()
    if status != 0:
        raise RuntimeError(f"device status {status} after the eager steps")
    stage_ms = {n: 0.0 for n in names}
    eager_step_ms = []
    for ev in events:
        for i, n in enumerate(names):
            stage_ms[n] += ev[i].elapsed_time(ev[i + 1])
        eager_step_ms.append(ev[0].elapsed_time(ev[len(names)]))
    eager_ms = max_over_ranks(sum(eager_step_ms), world) / args.steps
    avg = {n: stage_ms[n] / args.steps for n in names}

    # timed pass: the same step captured once into a CUDA graph and replayed, so
    # the host's per-call work (argument checks, tensor-map encoding, launches)
    # is off the device's path; every replay runs every stage
    graph, graph_note, launches_per_step = None, None, None
    if not args.no_graph:
        try:
            g = torch.cuda.CUDAGraph()
            l0 = bsa.launch_count()
            with torch.cuda.graph(g, capture_error_mode="thread_local"):
                step()
            launches_per_step = bsa.launch_count() - l0
            for _ in range(args.warmup):
                flush()
                g.replay()
            torch.cuda.synchronize()
            if st.ws.status() != 0:
                raise RuntimeError(f"device status {st.ws.status()} after graph warm-up")
            graph = g
        except Exception as ex:  # capture not possible here: time the eager step instead
            graph_note = f"graph capture failed ({type(ex).__name__}: {ex}); eager timing"
            torch.cuda.synchronize()
    barrier(world)
    with ClockSampler(local) as clk:
        t_wall = time.perf_counter()
        if graph is not None:
            ev_g = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                    for _ in range(args.steps)]
            for s in range(args.steps):
                flush()
                ev_g[s][0].record(stream)
                graph.replay()
                ev_g[s][1].record(stream)
        else:
            ev_e = [[torch.cuda.Event(enable_timing=True) for _ in range(len(names) + 1)] for _ in range(args.steps)]
            l0 = bsa.launch_count()
            for s in range(args.steps):
                flush()
                step(ev_e[s])
        torch.cuda.synchronize()
        t_wall = time.perf_counter() - t_wall
    barrier(world)
    status = st.ws.status()
    if status != 0:
        raise RuntimeError(f"device status {status} after the timed steps")
    if graph is not None:
        step_ms = [a.elapsed_time(b) for a, b in ev_g]
        launches = launches_per_step * args.steps
    else:
        step_ms = [ev[0].elapsed_time(ev[len(names)]) for ev in ev_e]
        launches = bsa.launch_count() - l0
    total_ms = max_over_ranks(sum(step_ms), world)
    ms_step = total_ms / args.steps
    value = whole_job_tflops(world, args.steps, f_fwd + f_bwd, total_ms)
    # the same time over the flops of the allowed entries alone (4 D per pair
    # forward, 2.5x that backward), where the mask has a closed form
    pairs = window_pairs(wl)
    exact_value = (whole_job_tflops(world, args.steps, (3.5 if has_bwd else 1.0) * 4.0 * wl.D * pairs, total_ms)
                   if pairs is not None else None)

    peaks = load_peaks()
    peak = peaks["bf16_tflops"]
    clocks = clk.summary()
    n_sm = torch.cuda.get_device_properties(dev).multi_processor_count
    max_mhz = clocks.get("sm_max_mhz") or 1965.0
    spec_peak = n_sm * max_mhz * 1e6 * BF16_FLOP_PER_CLK_SM / 1e12
    fwd_tf = f_fwd / (avg["forward"] * 1e-3) / 1e12
    main_tf = f_bwd / (avg["backward_main"] * 1e-3) / 1e12 if has_bwd else None
    tag = f"{args.workload}{wl.Sq}" if not args.small else None
    src_fwd, src_bwd = source_tag("fwd.cu", "ptx.cuh"), source_tag("bwd.cu", "ptx.cuh")
    roof_fwd = {"kernel": "k_attn_fwd (a3)", "bound": "tensor", "achieved": fwd_tf, "peak": peak,
                "unit": "TFLOP/s", "frac": fwd_tf / peak, "traffic": profiled_traffic("k_attn_fwd", tag, src_fwd),
                "peak_source": peaks["source"] + " bf16 burst",
                "frac_of_spec_peak": fwd_tf / spec_peak}
    if has_bwd:
        roof = {"kernel": "k_attn_bwd (a5)", "bound": "tensor", "achieved": main_tf, "peak": peak,
                "unit": "TFLOP/s", "frac": main_tf / peak,
                "traffic": profiled_traffic("k_attn_bwd", tag, src_bwd) if not args.nondet else None,
                "peak_source": peaks["source"] + " bf16 burst", "frac_of_spec_peak": main_tf / spec_peak}
    else:
        roof = roof_fwd

    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": workload_text(args) + (" [small shape]" if args.small else ""),
                   "global_batch": wl.B * world, "seq_len": wl.Sq, "kv_len": wl.Skv, "heads": wl.H,
                   "kv_heads": wl.k.shape[2], "head_dim": wl.D, "mask": wl.mask_text(),
                   "nonempty_tiles": n_tiles, "softmax": args.softmax, "bound": args.bound,
                   "passes": "forward + backward" if has_bwd else "forward only",
                   "o_residual": args.o_residual if has_bwd else None,
                   "bwd_order": ("nondeterministic" if args.nondet else args.order) if has_bwd else None,
                   "l2": "flushed before every step, outside the timed events: a 256 MiB write, then a 256 MiB "
                         "read that writes the dirty lines back, so the step starts on a clean L2",
                   "parallelism": f"replicas x{world}"},
        "pct_of_bf16_peak": 100.0 * value / peak,
        "pct_of_spec_peak": 100.0 * value / spec_peak,
        "spec_peak_tflops": spec_peak,
        "spec_peak_note": f"{n_sm} SMs x {max_mhz:.0f} MHz (max SM clock) x {BF16_FLOP_PER_CLK_SM} dense bf16 "
                          f"flop/clk/SM; datasheet {DATASHEET_BF16_TFLOPS:.0f} TFLOP/s",
        "exact_mask_tflops": exact_value,
        "exact_mask_pairs": pairs,
        "stages_ms": avg,
        "timing": ("CUDA-graph replay of the whole step (captured once after warm-up)" if graph is not None
                   else (graph_note or "eager library calls (--no-graph)")),
        "eager_ms_per_step": eager_ms,
        "eager_gpu_launches_per_step": eager_launches / args.steps,
        "forward_tflops": fwd_tf,
        "forward_pct_of_peak": 100.0 * fwd_tf / peak,
        "forward_pct_of_spec_peak": 100.0 * fwd_tf / spec_peak,
    }
    if has_bwd:
        bwd_ms = avg["preprocess"] + avg["backward_main"] + avg["convert"]
        line.update({
            "backward_tflops": f_bwd / (bwd_ms * 1e-3) / 1e12,
            "backward_pct_of_peak": 100.0 * f_bwd / (bwd_ms * 1e-3) / 1e12 / peak,
            "backward_main_tflops": main_tf,
            "backward_main_pct_of_peak": 100.0 * main_tf / peak,
            "backward_main_pct_of_spec_peak": 100.0 * main_tf / spec_peak,
        })
    line["roofline"] = roof
    if has_bwd:
        line["roofline_forward"] = roof_fwd
    line.update({"gpu_launches": launches, "wall_s_timed_loop": t_wall, "clocks": clocks})

    # the plan and the bound each alone, beside their overlapped call, each
    # captured into its own CUDA graph (no host gaps) and replayed: median of
    # 10, L2 flushed before each, outside the events
    if args.softmax == "fixed_m" and graph is not None:
        iso = {}
        for nm, fn in (("plan", st.plan), ("bound", st.bound), ("plan_and_bound", st.plan_and_bound)):
            gi = torch.cuda.CUDAGraph()
            with torch.cuda.graph(gi, capture_error_mode="thread_local"):
                fn()
            iso[nm] = _median_event_ms(gi.replay, flush, 10, stream)
            del gi
        if st.ws.status() != 0:
            raise RuntimeError(f"device status {st.ws.status()} timing the plan and the bound")
        line["plan_bound_isolated_ms"] = iso
    if has_bwd and not args.no_orders:
        ords = order_table(args, wl, flush, stream)
        line["backward_main_ms_by_order"] = ords
        line["backward_main_tflops_by_order"] = {k: f_bwd / (v * 1e-3) / 1e12 for k, v in ords.items()}
    if not has_bwd:
        fm, gates = softmax_table(args, wl, flush, stream)
        line["forward_ms_by_softmax"] = fm
        line["forward_tflops_by_softmax"] = {k: f_fwd / (v * 1e-3) / 1e12 for k, v in fm.items()}
        line["fixed_m_gate"] = gates
    if not args.no_e2e:
        line["e2e"] = e2e_leg(args, wl, dev, f_fwd + f_bwd, world)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        n_rows = min(1024, wl.Sq)
        dt, fl, threads = oracle_sample(wl, n_rows)
        what = "forward + backward" if has_bwd else "forward"
        line["cpu_baseline"] = {
            "value": fl / dt / 1e12, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
            "sample": f"rows and keys 0..{n_rows - 1} of head 0 under the same mask, {what}, fp64"}
    if rank == 0:
        print(json.dumps(line), flush=True)


def e2e_leg(args, wl, dev, flops, world):
    """The same step through the public API with host buffers: every step copies
    its own inputs (q, k, v and, with a backward, dO) from pinned host memory to
    the device, runs the full path and copies its results (O, LSE and dQ, dK,
    dV) back to pinned host memory, all inside the timed region.  Steps are
    pipelined as a training loop would run them: two buffer sets, the uploads,
    the compute and the downloads on three streams (PCIe carries both directions
    at once), each set reused only after its previous compute and download are
    done."""
    import torch
    import block_sparse_attention_map_b200 as bsa

    has_bwd = wl.backward
    names_in = ("q", "k", "v", "dO") if has_bwd else ("q", "k", "v")
    host = {n: getattr(wl, n).cpu().pin_memory() for n in names_in}
    out_spec = [("o", wl.q.shape, torch.bfloat16), ("lse", (wl.B, wl.H, wl.Sq), torch.float32)]
    if has_bwd:
        out_spec += [("dq", wl.q.shape, torch.bfloat16), ("dk", wl.k.shape, torch.bfloat16),
                     ("dv", wl.v.shape, torch.bfloat16)]
    slots = []
    for _ in range(2):
        dev_in = {n: torch.empty_like(getattr(wl, n)) for n in names_in}
        st = bsa.Stages(dev_in["q"], dev_in["k"], dev_in["v"], wl.mask, softmax_mode=args.softmax,
                        order=args.order, deterministic=not args.nondet, bound_mode=args.bound,
                        o_residual=args.o_residual)
        out_h = {n: torch.empty(shape, dtype=dt).pin_memory() for n, shape, dt in out_spec}
        ev = {k: torch.cuda.Event() for k in ("in", "comp", "out")}
        slots.append({"in": dev_in, "st": st, "out_h": out_h, "ev": ev, "used": False})
    s_up, s_comp, s_down = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
    main = torch.cuda.current_stream()

    def step(i):
        sl = slots[i % 2]
        ev, st, dev_in = sl["ev"], sl["st"], sl["in"]
        with torch.cuda.stream(s_up):
            if sl["used"]:
                s_up.wait_event(ev["comp"])  # the set's inputs are free once its last compute ran
            for n in names_in:
                dev_in[n].copy_(host[n], non_blocking=True)
            ev["in"].record(s_up)
        with torch.cuda.stream(s_comp):
            s_comp.wait_event(ev["in"])
            if sl["used"]:
                s_comp.wait_event(ev["out"])  # its outputs were read back
            st.plan_and_bound()
            st.forward()
            if has_bwd:
                st.preprocess(dev_in["dO"])
                st.backward_main(dev_in["dO"])
                st.convert()
            ev["comp"].record(s_comp)
        with torch.cuda.stream(s_down):
            s_down.wait_event(ev["comp"])
            srcs = {"o": st.out, "lse": st.lse, "dq": st.dq, "dk": st.dk, "dv": st.dv}
            for n, _, _ in out_spec:
                sl["out_h"][n].copy_(srcs[n], non_blocking=True)
            ev["out"].record(s_down)
        sl["used"] = True

    for i in range(max(2, args.warmup)):
        step(i)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    e0.record(main)
    for s_ in (s_up, s_comp, s_down):
        s_.wait_event(e0)
    for i in range(args.steps):
        step(i)
    for s_ in (s_up, s_comp, s_down):
        main.wait_stream(s_)
    e1.record(main)
    torch.cuda.synchronize()
    for sl in slots:
        if sl["st"].ws.status() != 0:
            raise RuntimeError(f"device status {sl['st'].ws.status()} in the end-to-end leg")
    ms = max_over_ranks(e0.elapsed_time(e1), world)
    h2d = sum(t.numel() * t.element_size() for t in host.values())
    d2h = sum(t.numel() * t.element_size() for t in slots[0]["out_h"].values())
    return {"value": whole_job_tflops(world, args.steps, flops, ms), "unit": "TFLOP/s",
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "ms_per_step": ms / args.steps,
            "pipeline": "two buffer sets; uploads, compute and downloads on three streams"}


def main():
    args = parse()
    if args.impl == "reference":
        world = int(os.environ.get("WORLD_SIZE", "1"))
        rank = int(os.environ.get("RANK", "0"))
        run_reference(args, world, rank)
        return
    world, rank, local = dist_setup(args)
    try:
        run_ours(args, world, rank, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
