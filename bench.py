"""Benchmark of the NF4 hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--m 16]

Workload (the decode configuration): the 224 linears of a Llama-7B-shaped
decoder stack (32 layers x {q,k,v,o 4096x4096; gate,up 11008x4096; down
4096x11008}), bf16 weights ~N(0, 0.02^2) quantized to NF4 + double quantization
(3.34 GB), and bf16 activations ~N(0, 1) with M tokens.  One step = one decode
pass: nf4_linear on every one of the 224 weights (fused dequant-GEMV), replayed
from a CUDA graph.  The weights read per step are 26x the 126 MB L2, so every
step streams from HBM.

Printed: one JSON line.  ``value`` = whole-job HBM GB/s of algorithmic bytes
(NF4 weight + metadata + X + Y) over the timed steps; extra legs in the same
run report M = 1 and 4, the dequant-GEMM TFLOP/s at M = 4096 (K = 4096,
N = 11008), quantize + double-quant and dequantize GB/s over the stack, the
end-to-end rate through the C ABI with host buffers, the roofline of the GEMV
kernel and the CPU oracle's rate on a bounded sample.

``--impl reference`` times the CPU oracle (the reference arm) on a bounded
sample of the same workload and prints the same metric.
"""
from __future__ import annotations

import argparse
import csv
import hashlib
import io
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "NF4 dequant-GEMV HBM GB/s (% peak); dequant-GEMM TFLOP/s at M=4096"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
WORKLOAD = "llama7b-shaped decode: 224 NF4+DQ linears (32 x q,k,v,o 4096x4096; gate,up 11008x4096; down 4096x11008)"


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def linear_bytes(n: int, k: int, m: int, y_bytes: int) -> int:
    """Algorithmic bytes of one fused linear: packed codes, absmax codes, DQ
    scales and mean, X read once, Y written once."""
    nb = n * k // 64
    return n * k // 2 + nb + 4 * ((nb + 255) // 256) + 4 + 2 * m * k + y_bytes * m * n


def quant_bytes(n: int, k: int) -> int:
    """Algorithmic bytes of quantize + double quant from bf16: read W, write
    codes, absmax codes, scales and mean."""
    nb = n * k // 64
    return 2 * n * k + n * k // 2 + nb + 4 * ((nb + 255) // 256) + 4


def merge_bytes(n: int, k: int, r: int) -> int:
    """Merge + requantize: codes and double-quantized absmax in, codes and fp32
    absmax out, the two bf16 LoRA matrices read once."""
    p = n * k
    return p // 2 + p // 64 + 4 * ((p // 64 + 255) // 256) + 4 + p // 2 + 4 * (p // 64) + 2 * r * (n + k)


def dequant_bytes(n: int, k: int) -> int:
    nb = n * k // 64
    return n * k // 2 + nb + 4 * ((nb + 255) // 256) + 4 + 2 * n * k


# ---------------------------------------------------------------------------
# clocks during the timed region
# ---------------------------------------------------------------------------
class ClockSampler:
    """nvidia-smi sampled every 100 ms from before the warm-up until after the
    timed region; summary() keeps the samples that fall inside the timed region
    (widened by 150 ms on each side when the region is shorter than the
    sampling interval)."""
    FIELDS = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.out = ""
        self.t0 = self.t1 = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), "--query-gpu=" + self.FIELDS,
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, ValueError):
            self.proc = None
        time.sleep(0.3)

    def mark_start(self):
        self.t0 = time.time()

    def mark_end(self):
        self.t1 = time.time()

    def stop(self):
        if self.proc is not None:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                self.out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                self.out, _ = self.proc.communicate()

    def summary(self):
        import datetime
        rows = []
        for r in csv.reader(io.StringIO(self.out or "")):
            if len(r) < 10:
                continue
            try:
                t = datetime.datetime.strptime(r[0].strip(), "%Y/%m/%d %H:%M:%S.%f").timestamp()
            except ValueError:
                continue
            rows.append((t, [x.strip() for x in r[1:]]))
        if not rows or self.t0 is None or self.t1 is None:
            return None
        inside = [f for t, f in rows if self.t0 <= t <= self.t1]
        if not inside:
            inside = [f for t, f in rows if self.t0 - 0.15 <= t <= self.t1 + 0.15]
        if not inside:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}

        def num(v):
            try:
                return float(v)
            except ValueError:
                return None
        sm = [num(f[1]) for f in inside if num(f[1]) is not None]
        mx = [num(f[2]) for f in inside if num(f[2]) is not None]
        pw = [num(f[3]) for f in inside if num(f[3]) is not None]
        reasons = set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for f in inside:
            for name, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(name)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None,
                "power_w_median": statistics.median(pw) if pw else None,
                "reasons": sorted(reasons), "samples": len(inside)}


# ---------------------------------------------------------------------------
# distributed plumbing (weak scaling: every rank runs its own copy of the
# workload; no collective on the data path)
# ---------------------------------------------------------------------------
def dist_setup():
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if torch.cuda.is_available():
        torch.cuda.set_device(local)
    if world > 1:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return rank, world, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, world: int) -> float:
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device="cuda" if torch.cuda.is_available() else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(x: float, world: int) -> float:
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device="cuda" if torch.cuda.is_available() else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


# ---------------------------------------------------------------------------
# CPU oracle on a bounded sample (reference arm and cpu_baseline)
# ---------------------------------------------------------------------------
def host_threads() -> int:
    """Host cores this process may run on (at most 64)."""
    try:
        n = len(os.sched_getaffinity(0))
    except AttributeError:
        n = os.cpu_count() or 1
    return max(1, min(64, n))


def _oracle_slabs(m: int, count: int):
    """`count` independent 512 x 4096 bf16 slabs of a q_proj-shaped weight (as
    bit patterns) and an M-token activation."""
    import numpy as np
    import torch

    from quantized_linear_layers_nf4_b200 import synth
    rows, k = 512, 4096
    slabs = []
    for i in range(count):
        w = synth.weight_normal(rows, k, seed=synth.seed_for(4, i), dtype=torch.bfloat16)
        slabs.append(w.view(torch.int16).numpy().view(np.uint16).reshape(-1))
    x = synth.activations(m, k, seed=synth.seed_for(2, 100 + m))
    xb = x.view(torch.int16).numpy().view(np.uint16)
    return slabs, xb, rows, k


def _timed_threads(work, threads: int, budget_s: float):
    """Runs work(i) repeatedly in `threads` threads for about budget_s seconds;
    returns (total repetitions, elapsed seconds).  The oracle's C routines run
    without the interpreter lock, so the threads run in parallel."""
    import threading
    counts = [0] * threads
    t0 = time.perf_counter()

    def loop(i):
        while time.perf_counter() - t0 < budget_s:
            work(i)
            counts[i] += 1
    ts = [threading.Thread(target=loop, args=(i,)) for i in range(threads)]
    for t in ts:
        t.start()
    for t in ts:
        t.join()
    return sum(counts), time.perf_counter() - t0


class OracleBench:
    """The oracle (test infrastructure, as it stands) on bounded samples of the
    decode workload, with `threads` host threads on independent 512 x 4096
    slabs (quantized once, in parallel, untimed): dequant-GEMV (dequantize rows
    -> bf16 -> fp64 dot products with M tokens), quantize + double quant from
    bf16, and dequantize to bf16.  Rates are GB/s of algorithmic bytes."""

    def __init__(self, m: int, threads: int):
        from concurrent.futures import ThreadPoolExecutor

        import oracle as O
        self.O, self.m, self.threads = O, m, threads
        self.slabs, self.xb, self.rows, self.k = _oracle_slabs(m, threads)

        def prep(w):
            wq, am = O.quantize(w)
            q, s_, mu = O.double_quant(am)
            return wq, q, s_, mu
        with ThreadPoolExecutor(threads) as ex:
            self.states = list(ex.map(prep, self.slabs))

    def gemv(self, budget_s: float):
        O, rows, k = self.O, self.rows, self.k

        def work(i):
            wq, q, s_, mu = self.states[i]
            d = O.dequantize_range(wq, q, s_, mu, 0, rows * k)
            O.linear_bf16(self.xb, O.f32_to_bf16(d).reshape(rows, k))
        n, t = _timed_threads(work, self.threads, budget_s)
        return n * linear_bytes(rows, k, self.m, 2) / t / 1e9, n, t

    def quantize_dq(self, budget_s: float):
        O = self.O

        def work(i):
            wq, am = O.quantize(self.slabs[i])
            O.double_quant(am)
        n, t = _timed_threads(work, self.threads, budget_s)
        return n * quant_bytes(self.rows, self.k) / t / 1e9

    def dequantize(self, budget_s: float):
        O, rows, k = self.O, self.rows, self.k

        def work(i):
            wq, q, s_, mu = self.states[i]
            O.f32_to_bf16(O.dequantize_range(wq, q, s_, mu, 0, rows * k))
        n, t = _timed_threads(work, self.threads, budget_s)
        return n * dequant_bytes(rows, k) / t / 1e9

    def describe(self, n_gemv: int, t_gemv: float) -> str:
        return ("oracle on %d host thread(s), one 512x4096 NF4+DQ slab each: dequant-GEMV (dequantize, bf16 "
                "round, fp64 dot products) at M=%d, %d repetitions in %.1f s; quantize + double quant from bf16; "
                "dequantize to bf16" % (self.threads, self.m, n_gemv, t_gemv))


def oracle_rates(m: int, budget_s: float, threads: int):
    """All three oracle rates with `threads` host threads; returns ({leg: GB/s},
    description)."""
    ob = OracleBench(m, threads)
    g, n, t = ob.gemv(budget_s)
    return ({"gemv_gbs": g, "quantize_dq_gbs": ob.quantize_dq(budget_s / 2),
             "dequantize_bf16_gbs": ob.dequantize(budget_s / 2)}, ob.describe(n, t))


def run_reference(args, rank, world):
    if rank != 0:
        return
    t_all = time.perf_counter()
    per_step = []
    desc = ""
    threads = host_threads()
    ob = OracleBench(args.m, threads)
    for i in range(args.warmup + args.steps):
        gbs, n, el = ob.gemv(max(1.0, 6.0 / max(1, args.steps)))
        desc = ob.describe(n, el)
        if i >= args.warmup:
            per_step.append((gbs, el))
    value = statistics.mean(g for g, _ in per_step)
    ms = 1000.0 * statistics.mean(e for _, e in per_step)
    line = {
        "impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": "GB/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": {"workload": WORKLOAD, "m": args.m, "sample": "512x4096 slab"},
        "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": threads, "kind": "oracle",
                         "sample": desc},
        "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
        "wall_s": round(time.perf_counter() - t_all, 1),
    }
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------
# GPU legs
# ---------------------------------------------------------------------------
def _events_time(fn, reps, stream):
    import torch
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    start.record(stream)
    for _ in range(reps):
        fn()
    end.record(stream)
    end.synchronize()
    return start.elapsed_time(end) / 1000.0 / reps


def gemv_traffic(kernel_src: str):
    """DRAM bytes per launch of the GEMV kernel from the committed ncu summary,
    or None when the kernel source changed since the counters were taken."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    ent = d.get("gemv")
    if not ent:
        return None
    sha = hashlib.sha256(open(kernel_src, "rb").read()).hexdigest()[:16]
    if ent.get("source_sha") != sha:
        return None
    return ent.get("dram_bytes_per_launch_scaled")


def run_ours(args, rank, world, local):
    import torch

    import quantized_linear_layers_nf4_b200 as nf4
    from quantized_linear_layers_nf4_b200 import synth
    from quantized_linear_layers_nf4_b200.build import build

    if rank == 0:
        build()
    barrier(world)
    nf4._lib.lib()
    pk, pk_kind = peaks()
    dev = torch.device("cuda", local)
    stream = torch.cuda.current_stream()

    # ---- weights: 224 NF4 tensors (quantized on device from seeded bf16) ----
    stack = synth.llama7b_stack(args.layers)
    weights = []
    for idx, (_, _, n, k) in enumerate(stack):
        W = synth.weight_normal(n, k, seed=synth.seed_for(4, idx), dtype=torch.bfloat16, device=dev)
        weights.append(nf4.quantize_weight(W))
        del W
    torch.cuda.synchronize()
    shapes = sorted(set((w.n, w.k) for w in weights))

    early = not args.no_weights_early
    # launch groups of the step: per layer q/k/v (one X), o, gate/up (one X), down
    groups = []
    for li in range(args.layers):
        lw = weights[7 * li: 7 * li + 7]
        groups += ([[w] for w in lw] if args.no_group else [lw[0:3], [lw[3]], lw[4:6], [lw[6]]])

    def decode_setup(m):
        xs = {k: synth.activations(m, k, seed=synth.seed_for(2, 100 + m) + k, device=dev)
              for k in set(k for _, k in shapes)}
        # outputs: one buffer per (n, position in the launch group)
        ys = {}
        for grp in groups:
            for i, w in enumerate(grp):
                ys.setdefault((w.n, i), torch.empty((m, w.n), dtype=torch.bfloat16, device=dev))
        # one split-k workspace serves every linear of the step (they run one after another)
        ws = None if args.no_workspace else nf4.linear_workspace(shapes, m=m, device=dev)

        def step():
            for grp in groups:
                nf4.nf4_linear_group(xs[grp[0].k], grp, torch.bfloat16,
                                     outs=[ys[(w.n, i)] for i, w in enumerate(grp)],
                                     weights_early=early, workspace=ws)
        step()
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            step()
        torch.cuda.synchronize()
        nbytes = sum(linear_bytes(w.n, w.k, m, 2) for w in weights)
        return g, xs, ys, nbytes

    # ---- main leg: decode pass at M = args.m ----
    g, xs, ys, step_bytes = decode_setup(args.m)
    clk = ClockSampler(local)
    clk.start()
    for _ in range(args.warmup):
        g.replay()
    torch.cuda.synchronize()
    barrier(world)
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    clk.mark_start()
    start.record(stream)
    for _ in range(args.steps):
        g.replay()
    end.record(stream)
    end.synchronize()
    clk.mark_end()
    clk.stop()
    barrier(world)
    t_step = start.elapsed_time(end) / 1000.0 / args.steps
    t_step_max = max_over_ranks(t_step, world)
    total_bytes = sum_over_ranks(float(step_bytes), world)
    value = total_bytes / t_step_max / 1e9
    # nf4_linear_group makes one launch for a group it runs together, else one per weight
    launches_per_step = sum(nf4.nf4_linear_group_launches(args.m, [w.n for w in grp], grp[0].k) for grp in groups)
    avg_launch_s = t_step / launches_per_step
    bytes_per_launch = step_bytes / launches_per_step

    # ---- e2e: host buffers through the C ABI, copies inside the timed region ----
    xh = {k: x.cpu().pin_memory() for k, x in xs.items()}
    yh = {key: torch.empty(y.shape, dtype=y.dtype).pin_memory() for key, y in ys.items()}
    h2d = sum(x.numel() * x.element_size() for x in xh.values())
    d2h = sum(y.numel() * y.element_size() for y in yh.values())

    def e2e_step():
        for k, x in xh.items():
            xs[k].copy_(x, non_blocking=True)
        g.replay()
        for key, y in ys.items():
            yh[key].copy_(y, non_blocking=True)
    for _ in range(args.warmup):
        e2e_step()
    barrier(world)
    t_e2e = max_over_ranks(_events_time(e2e_step, args.steps, stream), world)
    e2e_value = total_bytes / t_e2e / 1e9
    del g

    # ---- extra legs (rank-local, reported for rank 0) ----
    by_m = {args.m: round(step_bytes / t_step / 1e9, 1)}
    for m in (1, 4, 16):
        if m == args.m:
            continue
        gm, _, _, bm = decode_setup(m)
        for _ in range(2):
            gm.replay()
        by_m[m] = round(bm / _events_time(gm.replay, max(2, args.steps // 2), stream) / 1e9, 1)
        del gm

    # one weight shape alone: back-to-back launches on rotating copies of the
    # weight (about 300 MB, beyond L2), graph-captured, m = 16
    single = {}
    for tag, w0 in (("4096x4096", weights[0]), ("11008x4096", weights[4]), ("4096x11008", weights[6])):
        ncopy = max(2, int(300e6 // linear_bytes(w0.n, w0.k, 16, 2)) + 1)
        copies = [w0] + [nf4.NF4Weight(w0.n, w0.k, w0.wq.clone(), w0.absmax_q.clone(), w0.absmax_scale.clone(),
                                       w0.absmax_offset.clone(), w0.quant_type) for _ in range(ncopy - 1)]
        Xs1 = synth.activations(16, w0.k, seed=synth.seed_for(2, 300), device=dev)
        Ys1 = torch.empty((16, w0.n), dtype=torch.bfloat16, device=dev)
        ws1 = nf4.linear_workspace([(w0.n, w0.k)], m=16)

        def f_single():
            for wc in copies:
                nf4.nf4_linear(Xs1, wc, torch.bfloat16, out=Ys1, workspace=ws1, weights_early=early)
        f_single()
        g1 = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g1):
            f_single()
        for _ in range(3):
            g1.replay()
        t1 = _events_time(g1.replay, 20, stream) / len(copies)
        single[tag] = {"gbs": round(linear_bytes(w0.n, w0.k, 16, 2) / t1 / 1e9, 1),
                       "us_per_launch": round(t1 * 1e6, 2), "copies": len(copies)}
        del g1, copies
    single_note = "back-to-back nf4_linear_ws launches (m = 16) over rotating copies beyond L2, graph-captured"

    # dequant-GEMM at M = 4096, K = 4096, N = 11008
    gemm = None
    if not args.skip_gemm:
        Wg = synth.weight_normal(11008, 4096, seed=synth.seed_for(3, 0), dtype=torch.bfloat16, device=dev)
        wg = nf4.quantize_weight(Wg)
        del Wg
        Xg = synth.activations(4096, 4096, seed=synth.seed_for(3, 1), device=dev)
        Yg = torch.empty((4096, 11008), dtype=torch.bfloat16, device=dev)
        fn = lambda: nf4.nf4_linear(Xg, wg, torch.bfloat16, out=Yg)
        for _ in range(3):
            fn()
        t_g = _events_time(fn, 20, stream)
        tflops = 2.0 * 4096 * 4096 * 11008 / t_g / 1e12
        gemm = {"m": 4096, "k": 4096, "n": 11008, "tflops": round(tflops, 2),
                "ms": round(t_g * 1e3, 3), "peak_tflops": pk["bf16_tflops"],
                "frac": round(tflops / pk["bf16_tflops"], 4), "peak_kind": pk_kind + " burst bf16"}
        # the same weight over a sweep of token counts (m <= 16 runs the GEMV)
        sweep = {}
        for mm in (16, 128, 256, 512, 1024, 2048, 8192):
            Xs = synth.activations(mm, 4096, seed=synth.seed_for(3, 2) + mm, device=dev)
            Ys = torch.empty((mm, 11008), dtype=torch.bfloat16, device=dev)
            fs = lambda: nf4.nf4_linear(Xs, wg, torch.bfloat16, out=Ys)
            for _ in range(3):
                fs()
            ts = _events_time(fs, 20, stream)
            sweep[mm] = round(2.0 * mm * 4096 * 11008 / ts / 1e12, 1)
            del Xs, Ys
        sweep[4096] = gemm["tflops"]
        gemm["tflops_by_m"] = dict(sorted(sweep.items()))
        # backward through the frozen base on the same weight: dX [4096, 4096] = dY [4096, 11008] * What
        dYg = synth.activations(4096, 11008, seed=synth.seed_for(3, 7), device=dev)
        dXg = torch.empty((4096, 4096), dtype=torch.bfloat16, device=dev)
        fdx = lambda: nf4.nf4_linear_dx(dYg, wg, torch.bfloat16, out=dXg)
        for _ in range(3):
            fdx()
        t_dx = _events_time(fdx, 20, stream)
        gemm["dx"] = {"m": 4096, "n": 11008, "k": 4096, "tflops": round(2.0 * 4096 * 11008 * 4096 / t_dx / 1e12, 2),
                      "ms": round(t_dx * 1e3, 3), "frac": round(2.0 * 4096 * 11008 * 4096 / t_dx / 1e12 / pk["bf16_tflops"], 4)}
        del dYg, dXg
        # the QLoRA layer (r = 16, scale = lora_alpha / r = 32 / 16) against the plain linear:
        # decode on a q_proj-shaped weight at m = 16, prefill on this weight at m = 4096
        rl = 16
        lora = {"r": rl, "scale": 2.0}
        for tag, wl, ml in (("decode_4096x4096_m16", weights[0], 16), ("prefill_11008x4096_m4096", wg, 4096)):
            Xl = synth.activations(ml, wl.k, seed=synth.seed_for(3, 8) + ml, device=dev)
            Yl = torch.empty((ml, wl.n), dtype=torch.bfloat16, device=dev)
            dl = (synth.activations(rl, wl.k, seed=synth.seed_for(3, 9), device=dev).float() * 0.02).to(torch.bfloat16)
            ul = (synth.activations(wl.n, rl, seed=synth.seed_for(3, 10), device=dev).float() * 0.02).to(torch.bfloat16)
            wsl = nf4.lora_workspace(ml, [(wl.n, wl.k)], rl, device=dev)
            wsp = nf4.linear_workspace([(wl.n, wl.k)], m=ml, device=dev)
            early_l = ml <= 16   # the decode path runs with programmatic dependent launch
            if ml <= 16:
                # decode: graph-captured launches over rotating copies of the weight
                # (beyond L2), as in the decode step; both arms the same way
                ncopy = max(2, int(300e6 // linear_bytes(wl.n, wl.k, ml, 2)) + 1)
                copies = [wl] + [nf4.NF4Weight(wl.n, wl.k, wl.wq.clone(), wl.absmax_q.clone(),
                                               wl.absmax_scale.clone(), wl.absmax_offset.clone(), wl.quant_type)
                                 for _ in range(ncopy - 1)]

                def run_l():
                    for wc in copies:
                        nf4.nf4_linear_lora(Xl, wc, dl, ul, 2.0, wsl, out=Yl, weights_early=True)

                def run_p():
                    for wc in copies:
                        nf4.nf4_linear(Xl, wc, torch.bfloat16, out=Yl, workspace=wsp, weights_early=True)
                graphs = []
                for fn in (run_l, run_p):
                    fn()
                    torch.cuda.synchronize()
                    g = torch.cuda.CUDAGraph()
                    with torch.cuda.graph(g):
                        fn()
                    for _ in range(3):
                        g.replay()
                    graphs.append(g)
                t_l = _events_time(graphs[0].replay, 10, stream) / ncopy
                t_p = _events_time(graphs[1].replay, 10, stream) / ncopy
                del graphs, copies
                how = "CUDA graph of %d launches over rotating copies beyond L2, programmatic dependent launch" % ncopy
            else:
                f_l = lambda: nf4.nf4_linear_lora(Xl, wl, dl, ul, 2.0, wsl, out=Yl, weights_early=early_l)
                f_p = lambda: nf4.nf4_linear(Xl, wl, torch.bfloat16, out=Yl, workspace=wsp, weights_early=early_l)
                f_l(); f_p()
                t_l = _events_time(f_l, 20, stream)
                t_p = _events_time(f_p, 20, stream)
                how = "back-to-back calls"
            lora[tag] = {"us_lora": round(t_l * 1e6, 2), "us_plain": round(t_p * 1e6, 2),
                         "overhead": round(t_l / t_p - 1.0, 4), "timing": how}
            del Xl, Yl, dl, ul, wsl, wsp
        gemm["lora"] = lora
        # the FP4 codebook on the same kernels and the same 11008 x 4096 weight:
        # GEMM at m = 4096 and the decode GEMV at m = 16, NF4 timed alongside
        Wf = synth.weight_normal(11008, 4096, seed=synth.seed_for(3, 0), dtype=torch.bfloat16, device=dev)
        wf = nf4.quantize_weight(Wf, quant_type="fp4")
        del Wf
        fp4 = {}
        f_f = lambda: nf4.nf4_linear(Xg, wf, torch.bfloat16, out=Yg)
        for _ in range(3):
            f_f()
        fp4["gemm_tflops_m4096"] = round(2.0 * 4096 * 4096 * 11008 / _events_time(f_f, 20, stream) / 1e12, 1)
        X16 = synth.activations(16, 4096, seed=synth.seed_for(3, 11), device=dev)
        Y16 = torch.empty((16, 11008), dtype=torch.bfloat16, device=dev)
        ws16 = nf4.linear_workspace([(11008, 4096)], m=16, device=dev)
        # eight copies of each weight per timed rep (190 MB > L2), so every launch reads HBM
        for tag, wt in (("fp4", wf), ("nf4", wg)):
            copies = [nf4.NF4Weight(wt.n, wt.k, wt.wq.clone(), wt.absmax_q.clone(), wt.absmax_scale.clone(),
                                    wt.absmax_offset.clone(), wt.quant_type) for _ in range(8)]

            def f_v():
                for wc in copies:
                    nf4.nf4_linear(X16, wc, torch.bfloat16, out=Y16, workspace=ws16)
            f_v()
            t_v = _events_time(f_v, 10, stream) / len(copies)
            fp4["gemv_gbs_m16_" + tag] = round(linear_bytes(11008, 4096, 16, 2) / t_v / 1e9, 1)
            del copies
        gemm["fp4"] = fp4
        del Xg, Yg, wg, wf, X16, Y16, ws16

    # 70B-shaped stress layer: 28672 x 8192 Student-t(4) weight with outlier input
    # columns, as GEMV (m = 1, 16) and GEMM (m = 512, 4096)
    stress = None
    if not args.skip_gemm:
        n5, k5 = 28672, 8192
        W5 = synth.weight_student_t(n5, k5, seed=synth.seed_for(5, 0), dtype=torch.bfloat16, device=dev)
        w5 = nf4.quantize_weight(W5)
        del W5
        stress = {"n": n5, "k": k5, "gemv_gbs": {}, "gemm_tflops": {}}
        for mm in (1, 16, 512, 4096):
            X5 = synth.activations(mm, k5, seed=synth.seed_for(5, 1) + mm, device=dev)
            Y5 = torch.empty((mm, n5), dtype=torch.bfloat16, device=dev)
            ws5 = nf4.linear_workspace([(n5, k5)], m=mm)
            f5 = lambda: nf4.nf4_linear(X5, w5, torch.bfloat16, out=Y5, workspace=ws5)
            for _ in range(3):
                f5()
            t5 = _events_time(f5, 20, stream)
            if mm <= 16:
                stress["gemv_gbs"][mm] = round(linear_bytes(n5, k5, mm, 2) / t5 / 1e9, 1)
            else:
                stress["gemm_tflops"][mm] = round(2.0 * mm * n5 * k5 / t5 / 1e12, 1)
            del X5, Y5
        del w5

    # quantize + double quant, and dequantize, over the stack
    qd = None
    if not args.skip_quant:
        sub = weights[:7]
        # every tensor has its own input and output buffers (0.4 GB of bf16 weights
        # in, as much out: one rep's working set is several times L2), and each leg
        # runs as a CUDA graph of its 7 (or 14) launches, so host launch overhead is
        # not in the timed region
        Wbs = [torch.empty((w.n, w.k), dtype=torch.bfloat16, device=dev).normal_(0.0, 0.02) for w in sub]
        outs = [torch.empty((w.n, w.k), dtype=torch.bfloat16, device=dev) for w in sub]
        qbufs = [(torch.empty(w.n * w.k // 2, dtype=torch.uint8, device=dev),
                  torch.empty(w.n * w.k // 64, dtype=torch.float32, device=dev),
                  torch.empty(w.n * w.k // 64, dtype=torch.int8, device=dev),
                  torch.empty(w.n * w.k // 64 // 256 + 1, dtype=torch.float32, device=dev),
                  torch.empty(1, dtype=torch.float32, device=dev),
                  torch.empty(w.n * w.k // 64 // 256 + 2, dtype=torch.float64, device=dev)) for w in sub]

        def qstep():
            for w, v, (wq, am, aq, sc, mu, ws) in zip(sub, Wbs, qbufs):
                nf4.nf4_quantize(v, wq, am)
                nf4.nf4_double_quant(am, aq, sc, mu, ws)

        def dstep():
            # the layer's 7 weights in one launch
            nf4.nf4_dequantize_batch(sub, torch.bfloat16, outs=outs)

        def dstep_each():
            for w, o in zip(sub, outs):
                nf4.nf4_dequantize(w, torch.bfloat16, out=o)
        # merge a rank-16 LoRA update into every tensor of the layer and requantize
        # (codes + fp32 absmax out, the merged bf16 weight not written)
        rm = 16
        lora_mats = [((synth.activations(rm, w.k, seed=synth.seed_for(6, i), device=dev).float() * 0.02)
                      .to(torch.bfloat16),
                      (synth.activations(w.n, rm, seed=synth.seed_for(6, 100 + i), device=dev).float() * 0.02)
                      .to(torch.bfloat16)) for i, w in enumerate(sub)]

        def mstep():
            for w, (dm, um), (wq, am, _, _, _, _) in zip(sub, lora_mats, qbufs):
                nf4.nf4_merge_lora(w, dm, um, 2.0, wq=wq, absmax=am)
        graphs = {}
        for name, fn in (("q", qstep), ("d", dstep), ("d1", dstep_each), ("m", mstep)):
            fn()
            torch.cuda.synchronize()
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                fn()
            for _ in range(3):
                g.replay()
            graphs[name] = g
        tq = _events_time(graphs["q"].replay, 10, stream)
        td = _events_time(graphs["d"].replay, 10, stream)
        td1 = _events_time(graphs["d1"].replay, 10, stream)
        tm = _events_time(graphs["m"].replay, 10, stream)
        del graphs
        qb = sum(quant_bytes(w.n, w.k) for w in sub)
        db = sum(dequant_bytes(w.n, w.k) for w in sub)
        mb = sum(merge_bytes(w.n, w.k, rm) for w in sub)
        qd = {"quantize_dq_gbs": round(qb / tq / 1e9, 1), "dequantize_bf16_gbs": round(db / td / 1e9, 1),
              "dequantize_bf16_gbs_one_call_per_weight": round(db / td1 / 1e9, 1),
              "merge_lora_gbs": round(mb / tm / 1e9, 1), "merge_lora_ms_per_layer": round(tm * 1e3, 3),
              "merge_lora_r": rm,
              "sample": "one decoder layer (7 tensors, 202M params) per rep, bf16 in/out, distinct buffers per "
                        "tensor, each leg a CUDA graph; dequantize as one nf4_dequantize_batch launch (and as one "
                        "call per weight)"}
        del lora_mats, Wbs, outs, qbufs

    clocks = clk.summary()
    result = None
    if rank == 0:
        traffic = gemv_traffic(os.path.join(ROOT, "quantized_linear_layers_nf4_b200", "csrc", "nf4_gemv.cu"))
        achieved = bytes_per_launch / avg_launch_s / 1e9
        result = {
            "metric": METRIC, "value": round(value, 1), "unit": "GB/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(t_step_max * 1e3, 4),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic",
            "config": {"workload": WORKLOAD, "m": args.m, "layers": args.layers,
                       "weights_gb_per_step": round(step_bytes / 1e9, 3),
                       "l2": "inputs larger than L2 (%.2f GB of NF4 weights per step vs 126 MB)"
                             % (sum(w.nbytes() for w in weights) / 1e9),
                       "y_dtype": "bf16", "parallelism": "replicas (weak scaling)",
                       "launch": ("CUDA graph of %d launches per step (%s)%s"
                                  % (launches_per_step, "nf4_linear_ws per weight" if args.no_group else
                                     "per layer: nf4_linear_group q/k/v, o, nf4_linear_group gate/up, down; "
                                     "a group runs as one launch when that is predicted faster",
                                     ", NF4_LINEAR_WEIGHTS_EARLY: programmatic dependent launches, weight loads "
                                     "overlap the previous launch" if early else "")),
                       "split_k": "thread-block clusters, partial sums through distributed shared memory"
                                  if args.no_workspace
                                  else "global workspace, last CTA of a tile adds the partial sums"},
            "frac_of_peak": round(value / world / pk["hbm_gbs"], 4),
            "decode_gbs_by_m": by_m,
            "decode_single_shape": {"note": single_note, **single},
            "gemm": gemm,
            "stress_70b_layer": stress,
            "quant": qd,
            "roofline": {"bound": "hbm", "kernel": "k_nf4_gemv", "achieved": round(achieved, 1),
                         "peak": pk["hbm_gbs"], "unit": "GB/s", "frac": round(achieved / pk["hbm_gbs"], 4),
                         "traffic": traffic, "peak_kind": pk_kind,
                         "algorithmic_bytes_per_launch": int(bytes_per_launch)},
            "e2e": {"value": round(e2e_value, 1), "unit": "GB/s", "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h},
            "gpu_launches": launches_per_step * args.steps,
            "clocks": clocks,
        }
    return result


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--m", type=int, default=16, help="tokens per decode step (1..16)")
    ap.add_argument("--layers", type=int, default=32)
    ap.add_argument("--no-workspace", action="store_true",
                    help="split k through thread-block clusters instead of a global workspace")
    ap.add_argument("--no-group", action="store_true",
                    help="one launch per weight instead of grouping q/k/v and gate/up")
    ap.add_argument("--no-weights-early", action="store_true",
                    help="launch each linear without programmatic dependent launch")
    ap.add_argument("--skip-gemm", action="store_true")
    ap.add_argument("--skip-quant", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    rank, world, local = dist_setup()
    try:
        if args.impl == "reference":
            run_reference(args, rank, world)
            return
        result = run_ours(args, rank, world, local)
        if rank == 0:
            if world == 1 and not args.no_cpu_baseline:
                threads = host_threads()
                one, desc1 = oracle_rates(args.m, 6.0, 1)
                allc, desc = oracle_rates(args.m, 6.0, threads)
                result["cpu_baseline"] = {
                    "value": round(allc["gemv_gbs"], 4), "unit": "GB/s", "cores": threads, "kind": "oracle",
                    "sample": desc,
                    "quantize_dq_gbs": round(allc["quantize_dq_gbs"], 4),
                    "dequantize_bf16_gbs": round(allc["dequantize_bf16_gbs"], 4),
                    "one_thread": {k2: round(v2, 4) for k2, v2 in one.items()}}
            else:
                result["cpu_baseline"] = None
            print(json.dumps(result), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
