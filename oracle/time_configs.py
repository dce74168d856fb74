"""Timing of the oracle, the CPU reference of the FP8 attention forward, on the
host cores.  Test and measurement infrastructure: nothing on the GPU path uses it.

    python oracle/time_configs.py

Prints one JSON line per measurement (algorithmic FLOPs of the rows computed
divided by the measured seconds):
  - the tiny configuration (B1 H1 N1024 d64, non-causal) in full: the FP8
    pipeline emulation on all cores and on one thread, and the float64 exact
    pass on all cores;
  - one run of the Delta/S sweep configuration (B1 H8 N4096 d128, non-causal)
    in full;
  - 4096 seeded sampled query rows of the batched configuration (B4 H32 N8192
    d128, non-causal).
The causal prefill and long-context configurations are timed on sampled rows by
bench.py (its cpu_baseline and --impl reference).
"""
import json
import math
import os
import sys
import time

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

import oracle  # noqa: E402
import workload  # noqa: E402


def _timed(fn):
    t0 = time.perf_counter()
    fn()
    return time.perf_counter() - t0


def _line(config, what, threads, seconds, flops):
    print(json.dumps({"config": config, "pass": what, "threads": threads,
                      "seconds": round(seconds, 4),
                      "TFLOP/s": round(flops / seconds / 1e12, 5)}), flush=True)


def main():
    cores = os.cpu_count()
    # tiny: block_n 64, S = 256, reverse order, 4 sink keys, Delta = 8
    B, H, N, d = 1, 1, 1024, 64
    W = workload.make_sink_workload(B, H, H, N, d, 4, 8.0, seed=workload.CONFIG_SEED_BASE + 1)
    Q8, K8, V8 = (oracle.e4m3_encode(x) for x in (W.q, W.k, W.v))
    flops = 4.0 * B * H * N * N * d
    name = "tiny B1 H1 N1024 d64 non-causal"
    for nt in (0, 1):
        dt = _timed(lambda: oracle.attn_emulate(Q8, K8, V8, B, H, H, N, d, 0, 1.0 / math.sqrt(d),
                                                256.0, 1, 64, 4, nthreads=nt))
        _line(name, "FP8 emulation", nt or cores, dt, flops)
    dt = _timed(lambda: oracle.attn_exact(Q8, K8, V8, B, H, H, N, d, 0, 1.0 / math.sqrt(d)))
    _line(name, "float64 exact", cores, dt, flops)

    # one run of the sweep: block_n 128, S = 256, reverse order, Delta = 8
    B, H, N, d = 1, 8, 4096, 128
    W = workload.make_sink_workload(B, H, H, N, d, 4, 8.0, seed=workload.CONFIG_SEED_BASE + 2)
    Q8, K8, V8 = (oracle.e4m3_encode(x) for x in (W.q, W.k, W.v))
    dt = _timed(lambda: oracle.attn_emulate(Q8, K8, V8, B, H, H, N, d, 0, 1.0 / math.sqrt(d),
                                            256.0, 1, 128, 4))
    _line("sweep run B1 H8 N4096 d128 non-causal", "FP8 emulation", cores, dt,
          4.0 * B * H * N * N * d)

    # batched: 4096 seeded sampled rows, S = 256, forward order, Delta = 10
    B, H, N, d = 4, 32, 8192, 128
    W = workload.make_sink_workload(B, H, H, N, d, 4, 10.0, seed=workload.CONFIG_SEED_BASE + 4)
    Q8, K8, V8 = (oracle.e4m3_encode(x) for x in (W.q, W.k, W.v))
    rows = np.sort(np.random.default_rng(workload.CONFIG_SEED_BASE + 4)
                   .choice(B * H * N, 4096, replace=False)).astype(np.int64)
    dt = _timed(lambda: oracle.attn_emulate(Q8, K8, V8, B, H, H, N, d, 0, 1.0 / math.sqrt(d),
                                            256.0, 0, 128, 4, rows=rows))
    _line("batched B4 H32 N8192 d128 non-causal, 4096 sampled rows", "FP8 emulation", cores, dt,
          4.0 * len(rows) * N * d)


if __name__ == "__main__":
    main()
