"""Benchmark of the FP8 attention forward with P-cast scale S and KV order.

Workload (one step): the causal GQA prefill of the P-cast study's LLM shape,
B=1, H=32 query heads over H_kv=8 KV heads, N=32768, d=128, E4M3 Q/K/V from
the seeded sink construction (n_sink=4, Delta=8), S=256, reverse KV order,
O in BF16, collapse counter on: one launch of the library's tcgen05 kernel.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Prints one JSON line (rank 0).  value = algorithmic TFLOP/s of the whole job
(2*B*H*N^2*d per causal step, all ranks' work / the slowest rank's time);
e2e = the same metric through the public API with pinned host buffers,
host<->device copies inside the timed region; roofline = the kernel's
achieved TFLOP/s against the FP8 dense peak (measured BF16 GEMM x 2);
cpu_baseline = the CPU oracle on a bounded sample of the same rows.
Multi-GPU (torchrun): every rank runs its own independent prefill (weak
scaling); no collective is on the data path.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

CFG = dict(B=1, H=32, H_kv=8, N=32768, d=128, causal=1, S=256.0, kv_order=1, n_sink=4,
           delta=8.0, block_n=128)
WORKLOAD = ("causal GQA prefill B=1 H=32/H_kv=8 N=32768 d=128 E4M3, sink construction "
            "n_sink=4 Delta=8, S=256, reverse KV order, O bf16, collapse counter on")
# --shard heads: the long-context problem split by kv heads over the ranks
CFG_LONG = dict(B=1, H=32, H_kv=8, N=131072, d=128, causal=1, S=256.0, kv_order=1, n_sink=4,
                delta=10.0, block_n=128)
WORKLOAD_LONG = ("long-context causal GQA B=1 H=32/H_kv=8 N=131072 d=128 E4M3, sink "
                 "construction n_sink=4 Delta=10, S=256, reverse KV order, O bf16, collapse "
                 "counter on; kv heads split over the ranks")
METRIC = "FP8 attn fwd TFLOPS & % of B200 FP8 peak; P-collapse rate vs F(Δ,S)"
CLOCK_FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
                "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
                "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")


def algorithmic_flops(B, H, N, d, causal):
    return (2 if causal else 4) * B * H * N * N * d


def rank_seed(rank):
    """Each rank runs its own independent prefill: distinct seeded inputs."""
    import workload
    return workload.CONFIG_SEED_BASE + 3 + 1000 * rank


def reduce_max(x, world, device):
    """Max over ranks (the slowest rank's time defines the job's time)."""
    if world == 1:
        return float(x)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def reduce_sum(values, world, device):
    """Element-wise integer sum over ranks (collapse counts)."""
    if world == 1:
        return [int(v) for v in values]
    import torch
    import torch.distributed as dist
    t = torch.tensor([int(v) for v in values], dtype=torch.int64, device=device)
    dist.all_reduce(t)
    return [int(v) for v in t.tolist()]


def job_tflops(flops_per_rank, world, max_ms_per_step):
    """Whole-job throughput: all ranks' algorithmic work / the slowest rank's time."""
    return world * flops_per_rank / (max_ms_per_step * 1e-3) / 1e12


def peak_tflops():
    """FP8 dense peak: the measured BF16 GEMM burst peak x 2 (nominal fp8/bf16
    ratio), else the machine's fallback figure."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            pk = json.load(f)
        return 2.0 * float(pk["bf16_tflops"]), "measured bf16 burst x 2 (MEASURED_PEAKS.json)"
    except Exception:
        return 2.0 * 1590.0, "fallback 1.59 PFLOP/s bf16 x 2"


# E[max of k independent standard normals], for k sink keys (1/sqrt(pi) at k = 2)
EXPECTED_MAX_NORMAL = {1: 0.0, 2: 0.5641895835, 3: 0.8462843753, 4: 1.0293753730}


def closed_form_F(delta, S, k=4):
    """The P-cast paper's closed form for the forward-order fraction of non-sink
    probabilities that the E4M3 cast flushes to zero (Methodology, theoretical
    framework): F(Delta, S) = Phi(Delta + delta_k - 10 ln 2 - ln S).  A reported
    reference value beside the measured fraction."""
    x = delta + EXPECTED_MAX_NORMAL[k] - 10.0 * math.log(2.0) - math.log(S)
    return 0.5 * math.erfc(-x / math.sqrt(2.0))


def fp8_gemm_peak(dev, n=8192, reps=10):
    """This GPU's dense FP8 GEMM rate in TFLOP/s: torch._scaled_mm (cuBLASLt) on
    E4M3 n x n x n with unit scales, BF16 out, best of `reps` CUDA-event timings.
    A context denominator beside the roofline's peak; None where unsupported."""
    import torch
    try:
        g = torch.Generator(device=dev).manual_seed(7)
        a = torch.randn(n, n, device=dev, generator=g).to(torch.float8_e4m3fn)
        bt = torch.randn(n, n, device=dev, generator=g).to(torch.float8_e4m3fn).t()
        one = torch.ones((), device=dev)
        run = lambda: torch._scaled_mm(a, bt, scale_a=one, scale_b=one, out_dtype=torch.bfloat16)
        for _ in range(3):
            run()
        torch.cuda.synchronize()
        best = float("inf")
        for _ in range(reps):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            run()
            e1.record()
            torch.cuda.synchronize()
            best = min(best, e0.elapsed_time(e1))
        del a, bt
        return 2.0 * n ** 3 / (best * 1e-3) / 1e12
    except Exception:
        return None


KERNEL_SOURCES = ["online_softmax_tcgen05_b200/csrc/fp8_attn_fwd.cu",
                  "online_softmax_tcgen05_b200/csrc/fp8_attn_fwd_pair.cu",
                  "online_softmax_tcgen05_b200/csrc/attn_kernel.cuh",
                  "online_softmax_tcgen05_b200/csrc/sm100.cuh",
                  "online_softmax_tcgen05_b200/csrc/exp2_poly.cuh",
                  "online_softmax_tcgen05_b200/csrc/row_max.cuh",
                  "online_softmax_tcgen05_b200/csrc/softmax_block.cuh"]
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "attn_fwd_prefill_N32768.json")


def kernel_sources_sha256():
    import hashlib
    h = hashlib.sha256()
    for rel in KERNEL_SOURCES:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def measured_traffic(prefill=True):
    """DRAM bytes per launch (dram__bytes_read.sum + dram__bytes_write.sum) from
    the committed ncu capture of the prefill workload; None for another workload
    or when the kernel sources changed since that capture."""
    if not prefill:
        return None
    try:
        with open(TRAFFIC_FILE) as f:
            rec = json.load(f)
        if rec.get("kernel_sources_sha256") != kernel_sources_sha256():
            return None
        return int(rec["dram_bytes_read"]) + int(rec["dram_bytes_write"])
    except Exception:
        return None


def smi_index(local_rank):
    """nvidia-smi index of this process's GPU (CUDA_VISIBLE_DEVICES aware)."""
    vis = os.environ.get("CUDA_VISIBLE_DEVICES", "")
    ids = [x.strip() for x in vis.split(",") if x.strip()]
    if local_rank < len(ids) and ids[local_rank].isdigit():
        return int(ids[local_rank])
    return local_rank


class ClockSampler:
    """nvidia-smi sampling (200 ms) during the timed region."""

    def __init__(self, index):
        self.index = smi_index(index)
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), "--query-gpu=" + CLOCK_FIELDS,
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except Exception:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *a):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for nm, val in zip(names, parts[5:9]):
                if val.lower().startswith("active"):
                    reasons.add(nm)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(sm)}


def make_inputs(seed, dev, cfg=CFG, kv_heads=None):
    import torch
    import workload
    from online_softmax_tcgen05_b200 import e4m3_cast
    W = workload.make_sink_workload(cfg["B"], cfg["H"], cfg["H_kv"], cfg["N"], cfg["d"],
                                    cfg["n_sink"], cfg["delta"], seed=seed, kv_heads=kv_heads)
    qkv = [e4m3_cast(torch.from_numpy(x).to(dev)) for x in (W.q, W.k, W.v)]
    return W, qkv


def head_shard(rank, world, Hkv):
    """kv heads [g0, g1) of this rank when a problem is split by kv heads."""
    if Hkv % world:
        raise ValueError("H_kv = %d does not split over %d ranks" % (Hkv, world))
    per = Hkv // world
    return rank * per, (rank + 1) * per


def run_ours(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist
    import online_softmax_tcgen05_b200 as fa
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    fa.load_library()
    fa.set_schedule(fa.SCHEDULE_TWO_TILES if args.schedule == "two-tiles" else fa.SCHEDULE_ONE_TILE)
    import workload
    strong = args.shard == "heads"
    cfg = CFG_LONG if strong else CFG
    if strong:
        g0, g1 = head_shard(rank, world, cfg["H_kv"])
        W, (q, k, v) = make_inputs(workload.CONFIG_SEED_BASE + 5, dev, cfg, kv_heads=(g0, g1))
    else:
        W, (q, k, v) = make_inputs(rank_seed(rank), dev)
    B, H, Hkv, N, d = W.B, W.H, W.Hkv, W.N, W.d
    scale = 1.0 / math.sqrt(d)
    O = torch.empty((B, H, N, d), dtype=torch.bfloat16, device=dev)
    ctr = torch.zeros(2, dtype=torch.int64, device=dev)
    stream = torch.cuda.current_stream()

    def step(count=True):
        fa.fp8_attn_fwd_ex(q, k, v, O, B=B, H=H, H_kv=Hkv, N=N, d=d, causal=True, scale=scale,
                           S=cfg["S"], kv_order=cfg["kv_order"], n_sink=cfg["n_sink"],
                           o_dtype=fa.O_BF16, block_n=cfg["block_n"],
                           collapse_ctr=ctr[0:1] if count else None,
                           collapse_sink_ctr=ctr[1:2] if count else None, stream=stream)

    def barrier():
        if world > 1:
            dist.barrier()

    def timed(fn, steps):
        barrier()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(steps):
            fn()
        e1.record(stream)
        torch.cuda.synchronize()
        barrier()
        return reduce_max(e0.elapsed_time(e1), world, dev)

    for _ in range(args.warmup):
        step(True)
        step(False)
    torch.cuda.synchronize()
    ctr.zero_()
    with ClockSampler(local_rank) as clk:
        ms_on = timed(lambda: step(True), args.steps)
    collapse_total, collapse_sink = (int(x) for x in ctr.cpu().tolist())
    ms_off = timed(lambda: step(False), args.steps)

    flops = algorithmic_flops(B, H, N, d, True)          # this rank's work
    step_ms = ms_on / args.steps
    # weak: every rank runs a whole problem; strong: the ranks share one problem
    value = job_tflops(flops, world, step_ms)
    kernel_tflops = flops / (step_ms * 1e-3) / 1e12
    peak, peak_src = peak_tflops()

    if args.mode == "kernel":
        if rank != 0:
            return None
        return {"metric": METRIC, "value": round(value, 2), "unit": "TFLOP/s", "n_gpus": world,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(step_ms, 4),
                "mode": "kernel only",
                "value_counter_off": round(job_tflops(flops, world, ms_off / args.steps), 2)}

    # end to end through the public API: pinned host E4M3 inputs -> device ->
    # kernel -> BF16 output back to pinned host memory, every step
    qh, kh, vh = (t.cpu().pin_memory() for t in (q, k, v))
    oh = torch.empty((B, H, N, d), dtype=torch.bfloat16, pin_memory=True)

    def e2e_step():
        fa.attention(qh, kh, vh, causal=True, scale=scale, S=cfg["S"], kv_order=cfg["kv_order"],
                     n_sink=cfg["n_sink"], block_n=cfg["block_n"], count_collapse=True, out=oh)

    for _ in range(max(1, args.warmup // 2)):
        e2e_step()
    e2e_steps = max(2, args.steps // 2)
    ms_e2e = timed(e2e_step, e2e_steps)
    e2e_value = job_tflops(flops, world, ms_e2e / e2e_steps)
    h2d = sum(t.numel() * t.element_size() for t in (qh, kh, vh))
    d2h = oh.numel() * oh.element_size() + 16

    collapse_total, collapse_sink = reduce_sum([collapse_total, collapse_sink], world, dev)

    if rank != 0:
        return None
    fp8_gemm = fp8_gemm_peak(dev)   # after every timed region
    pairs = world * B * H * (N - cfg["n_sink"]) * (N - cfg["n_sink"] + 1) // 2
    frac = collapse_total / args.steps / pairs
    line = {
        "metric": METRIC, "value": round(value, 2), "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(step_ms, 4),
        "higher_is_better": True, "scaling": "strong" if strong else "weak",
        "vs_baseline": None, "dtype": "e4m3", "data": "synthetic",
        "config": ({"workload": WORKLOAD_LONG, **cfg, "per_rank": "kv heads split over the "
                    "ranks; collapse counts all-reduced", "l2": "inputs 805 MB > 126 MB L2"}
                   if strong else
                   {"workload": WORKLOAD, **CFG, "per_rank": "independent prefill per GPU",
                    "l2": "inputs 201 MB > 126 MB L2, no flush"}),
        "value_counter_off": round(job_tflops(flops, world, ms_off / args.steps), 2),
        "pct_of_fp8_peak": {"measured": round(kernel_tflops / peak, 4),
                            "nominal_4500": round(kernel_tflops / 4500.0, 4),
                            "fp8_gemm_this_gpu": (None if fp8_gemm is None else
                                                  {"tflops": round(fp8_gemm, 1),
                                                   "frac": round(kernel_tflops / fp8_gemm, 4),
                                                   "how": "torch._scaled_mm E4M3 8192^3, "
                                                          "best of 10"})},
        "roofline": {"bound": "tensor", "achieved": round(kernel_tflops, 2),
                     "peak": round(peak, 1), "unit": "TFLOP/s",
                     "frac": round(kernel_tflops / peak, 4), "traffic": measured_traffic(prefill=not strong),
                     "peak_source": peak_src + " (of measured)" if "measured" in peak_src
                     else peak_src},
        "collapse": {"fraction": frac, "count_per_step": collapse_total // args.steps // world,
                     "in_sink_block": collapse_sink // args.steps // world,
                     "closed_form_forward_F": closed_form_F(cfg["delta"], cfg["S"], cfg["n_sink"])},
        "e2e": {"value": round(e2e_value, 2), "unit": "TFLOP/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "ms_per_step": round(ms_e2e / e2e_steps, 3)},
        "gpu_launches": args.steps,
        "clocks": clk.summary(),
        "kernel_schedule": args.schedule,
    }
    if world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(W, cfg, n_rows=8192 if strong else 65536)
    return line


def sample_rows(n_rows, seed=7, cfg=CFG):
    import numpy as np
    rng = np.random.default_rng(seed)
    total = cfg["B"] * cfg["H"] * cfg["N"]
    return np.sort(rng.choice(total, n_rows, replace=False)).astype(np.int64)


def oracle_sample(W, rows, Q8=None, K8=None, V8=None, cfg=CFG):
    """Time the oracle's FP8 emulation on the given rows of the workload;
    returns (seconds, algorithmic FLOPs of those rows)."""
    import oracle
    N, d = W.N, W.d
    if Q8 is None:
        Q8, K8, V8 = (oracle.e4m3_encode(x) for x in (W.q, W.k, W.v))
    t0 = time.perf_counter()
    oracle.attn_emulate(Q8, K8, V8, W.B, W.H, W.Hkv, N, d, 1,
                        1.0 / math.sqrt(d), cfg["S"], cfg["kv_order"], cfg["block_n"],
                        cfg["n_sink"], o_bf16=True, rows=rows)
    dt = time.perf_counter() - t0
    flops = float(sum(4 * d * ((int(r) % N) + 1) for r in rows))
    return dt, flops, (Q8, K8, V8)


def cpu_baseline(W, cfg=CFG, n_rows=65536):
    total = W.B * W.H * W.N
    rows = sample_rows(n_rows, cfg=dict(cfg, H=W.H))
    dt, flops, _ = oracle_sample(W, rows, cfg=cfg)
    return {"value": flops / dt / 1e12, "unit": "TFLOP/s", "cores": os.cpu_count(),
            "kind": "oracle",
            "sample": "%d seeded random query rows of the %d (all heads and positions), "
                      "FP8 pipeline emulation, %.1f s" % (n_rows, total, dt)}


def run_reference(args, rank, world):
    """The oracle as the reference arm, on rank 0 only."""
    if rank != 0:
        return None
    import workload
    W = workload.make_sink_workload(CFG["B"], CFG["H"], CFG["H_kv"], CFG["N"], CFG["d"],
                                    CFG["n_sink"], CFG["delta"],
                                    seed=workload.CONFIG_SEED_BASE + 3)
    rows_per_step = 1024
    enc = None
    for i in range(args.warmup):
        _, _, enc = oracle_sample(W, sample_rows(rows_per_step, seed=100 + i),
                                  *(enc or (None, None, None)))
    tot_t, tot_f = 0.0, 0.0
    for i in range(args.steps):
        dt, fl, enc = oracle_sample(W, sample_rows(rows_per_step, seed=200 + i),
                                    *(enc or (None, None, None)))
        tot_t += dt
        tot_f += fl
    value = tot_f / tot_t / 1e12
    sample = ("%d seeded random query rows per step of the %d, FP8 pipeline emulation"
              % (rows_per_step, CFG["B"] * CFG["H"] * CFG["N"]))
    return {"metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * tot_t / max(args.steps, 1), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "e4m3", "data": "synthetic",
            "config": {"workload": WORKLOAD, **CFG}, "impl": "reference",
            "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": os.cpu_count(),
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


# ------------------------------------------------------------------ reports --
# `--report collapse` and `--report configs` (one GPU): one JSON line per run,
# for the record of the method's evaluation; the default bench line above is
# unaffected.
class _ReportLaunch:
    """One configuration on device inputs, with its buffers allocated once:
    launch() only enqueues the kernel (for timing); counts() zeroes the
    counters, runs once and returns (collapse total, in sink-holding blocks)."""

    def __init__(self, fa, ins, shape, causal, S, order, n_sink, count=True):
        import torch
        self.fa, (self.q, self.k, self.v) = fa, ins
        self.shape, self.causal, self.S, self.order, self.ns = shape, causal, S, order, n_sink
        B, H, Hkv, N, d = shape
        self.O = torch.empty((B, H, N, d), dtype=torch.bfloat16, device=self.q.device)
        self.ctr = torch.zeros(2, dtype=torch.int64, device=self.q.device) if count else None

    def launch(self):
        B, H, Hkv, N, d = self.shape
        c = self.ctr
        self.fa.fp8_attn_fwd_ex(self.q, self.k, self.v, self.O, B=B, H=H, H_kv=Hkv, N=N, d=d,
                                causal=bool(self.causal), scale=1.0 / math.sqrt(d), S=self.S,
                                kv_order=self.order, n_sink=self.ns, o_dtype=self.fa.O_BF16,
                                block_n=128, collapse_ctr=None if c is None else c[0:1],
                                collapse_sink_ctr=None if c is None else c[1:2])

    def counts(self):
        import torch
        self.ctr.zero_()
        self.launch()
        torch.cuda.synchronize()
        c = self.ctr.cpu().tolist()
        return int(c[0]), int(c[1])


def _median_ms(fn, reps, warmup):
    import torch
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    times = []
    for _ in range(reps):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        fn()
        e1.record()
        torch.cuda.synchronize()
        times.append(e0.elapsed_time(e1))
    return statistics.median(times)


def _visible_pairs(B, H, N, n_sink, causal):
    """Non-sink (query, key) pairs the collapse fraction is taken over."""
    m = N - n_sink
    return B * H * (m * (m + 1) // 2 if causal else N * m)


def report_collapse(dev):
    """Delta/S sweep (B1 H8 N4096 d128, non-causal, 4 sink keys): the measured
    collapse fraction in forward order beside the closed form F(Delta, S), and the
    fraction outside the sink-holding KV block in reverse order."""
    import torch
    import workload
    import online_softmax_tcgen05_b200 as fa
    B, H, N, d, ns = 1, 8, 4096, 128, 4
    pairs = _visible_pairs(B, H, N, ns, 0)
    for delta in range(0, 13):
        W = workload.make_sink_workload(B, H, H, N, d, ns, float(delta),
                                        seed=workload.CONFIG_SEED_BASE + 2)
        ins = [fa.e4m3_cast(torch.from_numpy(x).to(dev)) for x in (W.q, W.k, W.v)]
        for S in (1.0, 16.0, 256.0, 448.0):
            line = {"report": "collapse", "workload": "sweep B1 H8 N4096 d128 non-causal, "
                    "4 sink keys", "delta": delta, "S": S,
                    "closed_form_F": round(closed_form_F(delta, S, ns), 6)}
            for order, name in ((fa.KV_FORWARD, "forward"), (fa.KV_REVERSE, "reverse")):
                tot, sink = _ReportLaunch(fa, ins, (B, H, H, N, d), 0, S, order, ns).counts()
                line[name] = {"fraction": round(tot / pairs, 6),
                              "outside_sink_block": round((tot - sink) / pairs, 8)}
            print(json.dumps(line), flush=True)
        del ins


def report_configs(dev):
    """The timing protocols of the evaluation's larger configurations (median of
    CUDA-event timings), with the collapse fraction of each run: the causal GQA
    prefill with the counter on and off; batched non-causal with forward and
    reverse order alternating; the long-context causal GQA grid Delta x S x order."""
    import torch
    import workload
    import online_softmax_tcgen05_b200 as fa

    def gen(B, H, Hkv, N, d, ns, delta, seed):
        W = workload.make_sink_workload(B, H, Hkv, N, d, ns, delta, seed=seed)
        return [fa.e4m3_cast(torch.from_numpy(x).to(dev)) for x in (W.q, W.k, W.v)]

    def launch(ins, shape, causal, S, order, ns, count):
        return _ReportLaunch(fa, ins, shape, causal, S, order, ns, count)

    # prefill: B1 H32/8 N32768, causal, Delta 8, S 256, reverse; 10 warm-up, median of 50
    shape = (1, 32, 8, 32768, 128)
    ins = gen(*shape, 4, 8.0, workload.CONFIG_SEED_BASE + 3)
    flops = algorithmic_flops(1, 32, 32768, 128, True)
    for count in (True, False):
        ms = _median_ms(launch(ins, shape, 1, 256.0, fa.KV_REVERSE, 4, count).launch, 50, 10)
        print(json.dumps({"report": "configs", "workload": "prefill B1 H32/8 N32768 d128 causal",
                          "S": 256.0, "order": "reverse", "counter": count,
                          "median_ms": round(ms, 4), "TFLOP/s": round(flops / ms / 1e9, 1)}),
              flush=True)
    del ins
    # batched: B4 H32 N8192, non-causal, Delta 10, S 256; forward and reverse alternating
    shape = (4, 32, 32, 8192, 128)
    ins = gen(*shape, 4, 10.0, workload.CONFIG_SEED_BASE + 4)
    flops = algorithmic_flops(4, 32, 8192, 128, False)
    runs = {fa.KV_FORWARD: launch(ins, shape, 0, 256.0, fa.KV_FORWARD, 4, True),
            fa.KV_REVERSE: launch(ins, shape, 0, 256.0, fa.KV_REVERSE, 4, True)}
    times = {fa.KV_FORWARD: [], fa.KV_REVERSE: []}
    for _ in range(5):
        for o in runs:
            runs[o].launch()
    torch.cuda.synchronize()
    for _ in range(50):
        for o in runs:
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            runs[o].launch()
            e1.record()
            torch.cuda.synchronize()
            times[o].append(e0.elapsed_time(e1))
    for o, name in ((fa.KV_FORWARD, "forward"), (fa.KV_REVERSE, "reverse")):
        tot, sink = runs[o].counts()
        ms = statistics.median(times[o])
        print(json.dumps({"report": "configs", "workload": "batched B4 H32 N8192 d128 non-causal",
                          "S": 256.0, "delta": 10.0, "order": name, "counter": True,
                          "median_ms": round(ms, 4), "TFLOP/s": round(flops / ms / 1e9, 1),
                          "collapse_fraction": tot / _visible_pairs(4, 32, 8192, 4, 0)}),
              flush=True)
    del ins, runs
    # long context: B1 H32/8 N131072, causal, counter on; Delta {6, 10} x S {1, 256} x order
    shape = (1, 32, 8, 131072, 128)
    flops = algorithmic_flops(1, 32, 131072, 128, True)
    pairs = _visible_pairs(1, 32, 131072, 4, 1)
    for delta in (6.0, 10.0):
        ins = gen(*shape, 4, delta, workload.CONFIG_SEED_BASE + 5)
        for S in (1.0, 256.0):
            for o, name in ((fa.KV_REVERSE, "reverse"), (fa.KV_FORWARD, "forward")):
                run = launch(ins, shape, 1, S, o, 4, True)
                ms = _median_ms(run.launch, 3, 1)
                tot, sink = run.counts()
                print(json.dumps({"report": "configs",
                                  "workload": "long B1 H32/8 N131072 d128 causal",
                                  "delta": delta, "S": S, "order": name, "counter": True,
                                  "median_ms": round(ms, 3), "TFLOP/s": round(flops / ms / 1e9, 1),
                                  "collapse_fraction": tot / pairs,
                                  "outside_sink_block": (tot - sink) / pairs,
                                  "closed_form_F": round(closed_form_F(delta, S, 4), 8)}),
                      flush=True)
        del ins


def report_batched_orders(dev):
    """Batched non-causal configuration (B4 H32 N8192 d128, Delta 10, S 256, counter
    on): forward and reverse KV order, 3 warm-up pairs then 50 alternating timed
    pairs, median of each (launches 7 and 8 are the first timed forward and
    reverse ones, for a profiler capture)."""
    import torch
    import workload
    import online_softmax_tcgen05_b200 as fa
    shape = (4, 32, 32, 8192, 128)
    W = workload.make_sink_workload(*shape, 4, 10.0, seed=workload.CONFIG_SEED_BASE + 4)
    ins = [fa.e4m3_cast(torch.from_numpy(x).to(dev)) for x in (W.q, W.k, W.v)]
    runs = [(name, _ReportLaunch(fa, ins, shape, 0, 256.0, o, 4, True))
            for name, o in (("forward", fa.KV_FORWARD), ("reverse", fa.KV_REVERSE))]
    for _ in range(3):
        for _, r in runs:
            r.launch()
    torch.cuda.synchronize()
    times = {name: [] for name, _ in runs}
    for _ in range(50):
        for name, r in runs:
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            r.launch()
            e1.record()
            torch.cuda.synchronize()
            times[name].append(e0.elapsed_time(e1))
    flops = algorithmic_flops(4, 32, 8192, 128, False)
    for name, _ in runs:
        ms = statistics.median(times[name])
        print(json.dumps({"report": "batched-orders", "order": name, "median_ms": round(ms, 4),
                          "TFLOP/s": round(flops / ms / 1e9, 1)}), flush=True)


def report_schedules(dev, pairs=30):
    """The two kernel schedules side by side in one process (fp8attn_set_schedule):
    one query tile per CTA (default) and two query tiles per CTA with the softmax
    warps taking turns on the exponential unit.  Prefill (causal GQA, reverse),
    batched non-causal forward and reverse; counter on and off; 3 warm-up rounds
    then `pairs` alternating timed launches of each schedule, median of each.
    Both schedules' outputs and counters are compared bit for bit first."""
    import torch
    import workload
    import online_softmax_tcgen05_b200 as fa
    cases = [("prefill", (1, 32, 8, 32768, 128), 1, fa.KV_REVERSE, 8.0, 3),
             ("batched forward", (4, 32, 32, 8192, 128), 0, fa.KV_FORWARD, 10.0, 4),
             ("batched reverse", (4, 32, 32, 8192, 128), 0, fa.KV_REVERSE, 10.0, 4)]
    scheds = [("one tile", fa.SCHEDULE_ONE_TILE), ("two tiles", fa.SCHEDULE_TWO_TILES)]
    try:
        for name, shape, causal, order, delta, cfg in cases:
            W = workload.make_sink_workload(*shape, 4, delta, seed=workload.CONFIG_SEED_BASE + cfg)
            ins = [fa.e4m3_cast(torch.from_numpy(x).to(dev)) for x in (W.q, W.k, W.v)]
            del W
            B, H, _, N, d = shape
            flops = algorithmic_flops(B, H, N, d, bool(causal))
            for count in (True, False):
                runs = [(sn, sv, _ReportLaunch(fa, ins, shape, causal, 256.0, order, 4, count))
                        for sn, sv in scheds]
                if count:
                    got = []
                    for _, sv, r in runs:
                        fa.set_schedule(sv)
                        got.append((r.counts(), r.O.clone()))
                    same = got[0][0] == got[1][0] and torch.equal(got[0][1], got[1][1])
                times = {sn: [] for sn, _, _ in runs}
                for i in range(3 + pairs):
                    for sn, sv, r in runs:
                        fa.set_schedule(sv)
                        e0 = torch.cuda.Event(enable_timing=True)
                        e1 = torch.cuda.Event(enable_timing=True)
                        e0.record()
                        r.launch()
                        e1.record()
                        torch.cuda.synchronize()
                        if i >= 3:
                            times[sn].append(e0.elapsed_time(e1))
                for sn, _, _ in runs:
                    ms = statistics.median(times[sn])
                    print(json.dumps({"report": "schedules", "workload": name, "schedule": sn,
                                      "counter": count, "median_ms": round(ms, 4),
                                      "TFLOP/s": round(flops / ms / 1e9, 1),
                                      "outputs_equal": same}), flush=True)
            del ins
    finally:
        fa.set_schedule(fa.SCHEDULE_ONE_TILE)


def report_e2e_timeline(dev, steps=2, warmup=4):
    """The prefill end to end through the host-buffer entry, profiled with CUPTI
    (torch.profiler) for diagnosis: per step, the time from the step's first
    device operation to its first kernel, the span from the first kernel's start
    to the last kernel's end, the download tail after the last kernel, and the
    bytes and busy time of the copies in each direction.  Times taken under a
    profiler; never a bench value."""
    import json as _json
    import tempfile

    import torch
    from torch.profiler import ProfilerActivity, profile
    import online_softmax_tcgen05_b200 as fa
    cfg = CFG
    W, (q, k, v) = make_inputs(rank_seed(0), dev)
    B, H, N, d = W.B, W.H, W.N, W.d
    qh, kh, vh = (t.cpu().pin_memory() for t in (q, k, v))
    oh = torch.empty((B, H, N, d), dtype=torch.bfloat16, pin_memory=True)

    def step():
        fa.attention(qh, kh, vh, causal=True, scale=1.0 / math.sqrt(d), S=cfg["S"],
                     kv_order=cfg["kv_order"], n_sink=cfg["n_sink"], block_n=cfg["block_n"],
                     count_collapse=True, out=oh)

    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    with profile(activities=[ProfilerActivity.CUDA]) as prof:
        for _ in range(steps):
            torch.cuda.synchronize()
            step()
        torch.cuda.synchronize()
    with tempfile.NamedTemporaryFile(suffix=".json") as f:
        prof.export_chrome_trace(f.name)
        events = _json.load(open(f.name))["traceEvents"]
    ev = sorted((e for e in events if e.get("ph") == "X" and e.get("cat") in
                 ("kernel", "gpu_memcpy", "gpu_memset")), key=lambda e: e["ts"])
    # each call starts by zeroing its collapse counters (a fill kernel): split there
    starts = [i for i, e in enumerate(ev) if e["cat"] == "kernel" and "attn_fwd" not in e["name"]]
    bounds = starts[:steps] + [len(ev)]
    for sidx in range(len(bounds) - 1):
        part = ev[bounds[sidx]:bounds[sidx + 1]]
        kern = [e for e in part if e["cat"] == "kernel" and "attn_fwd" in e["name"]]
        h2d = [e for e in part if e["cat"] == "gpu_memcpy" and "HtoD" in e["name"]]
        d2h = [e for e in part if e["cat"] == "gpu_memcpy" and "DtoH" in e["name"]]
        t0 = part[0]["ts"]
        end = max(e["ts"] + e["dur"] for e in part)
        k0 = min(e["ts"] for e in kern)
        k1 = max(e["ts"] + e["dur"] for e in kern)
        nbytes = lambda es: sum(int(e.get("args", {}).get("bytes", 0)) for e in es)
        busy = lambda es: sum(e["dur"] for e in es) / 1e3
        print(json.dumps({"report": "e2e-timeline", "step": sidx,
                          "total_ms": round((end - t0) / 1e3, 3),
                          "to_first_kernel_ms": round((k0 - t0) / 1e3, 3),
                          "kernel_span_ms": round((k1 - k0) / 1e3, 3),
                          "tail_after_last_kernel_ms": round((end - k1) / 1e3, 3),
                          "kernels": len(kern),
                          "h2d": {"copies": len(h2d), "MB": round(nbytes(h2d) / 1e6, 1),
                                  "busy_ms": round(busy(h2d), 3)},
                          "d2h": {"copies": len(d2h), "MB": round(nbytes(d2h) / 1e6, 1),
                                  "busy_ms": round(busy(d2h), 3)}}), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--shard", choices=["replica", "heads"], default="replica",
                    help="replica: one independent prefill per rank (weak scaling); heads: "
                         "the long-context problem split by kv heads (strong scaling)")
    ap.add_argument("--schedule", choices=["one-tile", "two-tiles"], default="one-tile",
                    help="kernel schedule (fp8attn_set_schedule): one query tile per CTA "
                         "(default) or two per CTA with turns on the exponential unit")
    ap.add_argument("--mode", choices=["full", "kernel"], default="full",
                    help="kernel: only the device-timed kernel loop (for profiling)")
    ap.add_argument("--report", choices=["collapse", "configs", "batched-orders", "e2e-timeline",
                                         "schedules"],
                    default=None,
                    help="one GPU: JSON lines for the Delta/S collapse sweep against the closed "
                         "form, or the timing protocols of the larger configurations")
    args = ap.parse_args()
    if args.report is not None:
        import torch
        dev = torch.device("cuda", 0)
        torch.cuda.set_device(dev)
        {"collapse": report_collapse, "configs": report_configs,
         "batched-orders": report_batched_orders,
         "e2e-timeline": report_e2e_timeline, "schedules": report_schedules}[args.report](dev)
        return
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        if world == 1 and args.gpus > 1:
            sys.exit("run multi-GPU through torchrun: --nproc-per-node %d" % args.gpus)
    if args.impl == "reference":
        line = run_reference(args, rank, world)
        if line is not None:
            print(json.dumps(line), flush=True)
        return
    pg = False
    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local_rank))
        pg = True
    try:
        line = run_ours(args, rank, world, local_rank)
        if line is not None:
            print(json.dumps(line), flush=True)
    finally:
        if pg:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
