"""GPU parity of the tcgen05 FP8 attention forward against the oracle's FP8
pipeline emulation, through the C ABI (ctypes binding).

Tolerances of the attention forward: max |dO| <= 2e-2 and relative RMS <= 5e-3
against the emulation (the MMA accumulates in another order).  Collapse counts:
at most 2 keys apart per query row, and totals within max(2, 1e-4 of the
oracle's): they may differ only where an FP32 rounding difference moves S*p
across 2^-10 (tests/helpers.py states the rule).

Workloads: the sink construction of workload/ (Q = g + 8u, sink keys
z + beta u, beta = Delta sqrt(d) / 8) at the paper-derived configurations:
tiny (B1 H1 N1024 d64), the Delta/S sweep (B1 H8 N4096 d128), the GQA causal
prefill (B1 H32/8 N32768 d128), batched non-causal (B4 H32 N8192) and long
context (N131072), plus small shapes with ragged tails and the edge cases.
"""
import math

import numpy as np
import pytest

from helpers import (assert_counts_close, assert_o_close, coverage_rows, gpu_inputs, gpu_inputs_bf16,
                     oracle, sample_rows, total_tol, workload)

pytestmark = pytest.mark.gpu


def run_gpu(ins, B, H, Hkv, N, d, causal, S, order, block_n, n_sink, f32=True, scale=None,
            count=True, denominator=0):
    import torch
    from online_softmax_tcgen05_b200 import O_BF16, O_F32, QK_BF16, QK_E4M3, fp8_attn_fwd_ex
    (Qg, _), (Kg, _), (Vg, _) = ins
    dev = Qg.device
    O = torch.full((B, H, N, d), float("nan"), dtype=torch.float32 if f32 else torch.bfloat16,
                   device=dev)
    ctr = torch.zeros(2, dtype=torch.int64, device=dev)
    rows = torch.zeros(max(B * H * N, 1), dtype=torch.int32, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    fp8_attn_fwd_ex(Qg, Kg, Vg, O, B=B, H=H, H_kv=Hkv, N=N, d=d, causal=causal,
                    scale=scale if scale is not None else 1.0 / math.sqrt(d), S=S,
                    kv_order=order, n_sink=n_sink, o_dtype=O_F32 if f32 else O_BF16,
                    block_n=block_n, denominator=denominator,
                    qk_dtype=QK_BF16 if Qg.dtype == torch.bfloat16 else QK_E4M3,
                    collapse_ctr=ctr[0:1] if count else None,
                    collapse_sink_ctr=ctr[1:2] if count else None,
                    collapse_rows=rows if count else None, status_word=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0, hex(int(status.item()))
    Of = O.float().cpu().numpy().reshape(-1, d)
    c = ctr.cpu().numpy()
    return Of, int(c[0]), int(c[1]), rows.cpu().numpy()[:B * H * N].astype(np.int64)


def check_case(W, ins, causal, S, order, block_n, f32=True, rows=None, what=""):
    B, H, Hkv, N, d, ns = W.B, W.H, W.Hkv, W.N, W.d, W.n_sink
    (_, Q8), (_, K8), (_, V8) = ins
    Og, tot, sink_tot, crow = run_gpu(ins, B, H, Hkv, N, d, causal, S, order, block_n, ns, f32)
    Oe, cr, ctot, slack = oracle.attn_emulate(Q8, K8, V8, B, H, Hkv, N, d, causal, W.scale, S,
                                              order, block_n, ns, o_bf16=not f32, rows=rows,
                                              flip_slack=True)
    if rows is None:
        Og_s, crow_s = Og, crow
    else:
        Og_s, crow_s = Og[rows], crow[rows]
    assert np.isfinite(Og_s).all(), what
    assert_o_close(Og_s, Oe, what, slack)
    # collapse: per-row counts, and the (sampled or whole-problem) totals
    assert_counts_close(crow_s, cr, what)
    if rows is None:
        assert tot == crow.sum()
        assert abs(int(ctot.sum()) - tot) <= total_tol(ctot.sum()), (what, ctot, tot)
        assert abs(int(ctot[0]) - sink_tot) <= total_tol(ctot[0]), (what, ctot, sink_tot)
    return Og, tot, sink_tot, crow


# ------------------------------------------------------------------ tiny -----
@pytest.mark.parametrize("S", [1.0, 256.0])
@pytest.mark.parametrize("order", [0, 1])
def test_tiny_sink_config(S, order):
    W = workload.make_sink_workload(1, 1, 1, 1024, 64, 4, 8.0, seed=workload.CONFIG_SEED_BASE + 1)
    ins = gpu_inputs(W)
    Og, tot, sink_tot, crow = check_case(W, ins, 0, S, order, 64, what=("tiny", S, order))
    frac = tot / (1024 * 1020)
    if order == 1 and S == 256.0:
        assert tot - sink_tot == 0                   # nothing outside the sink block
    if order == 0 and S == 1.0:
        assert frac > 0.9                            # F(8, 1) ~ 0.98
    # the counting and the plain kernel variants compute the same O
    Og2, *_ = run_gpu(ins, 1, 1, 1, 1024, 64, 0, S, order, 64, 4, count=False)
    assert np.array_equal(Og, Og2)


# ------------------------------------------------------- shapes and tails ----
CASES = [
    # B, H, Hkv, N, d, block_n, causal
    (1, 2, 1, 384, 128, 128, 0),
    (1, 2, 1, 384, 128, 128, 1),
    (1, 2, 2, 1000, 128, 128, 1),
    (1, 2, 2, 1000, 128, 64, 1),
    (2, 2, 1, 520, 64, 64, 0),
    (1, 4, 2, 700, 64, 128, 1),
    (1, 1, 1, 333, 64, 64, 1),
    (1, 1, 1, 256, 128, 64, 0),
    (2, 4, 2, 700, 64, 128, 1),   # causal CTA order across two batch elements
]


@pytest.mark.parametrize("B,H,Hkv,N,d,block_n,causal", CASES)
def test_parity_shapes(B, H, Hkv, N, d, block_n, causal):
    W = workload.make_sink_workload(B, H, Hkv, N, d, 4, 9.0, seed=N + d + block_n)
    ins = gpu_inputs(W)
    for S in (1.0, 256.0, 448.0):
        for order in (0, 1):
            check_case(W, ins, causal, S, order, block_n, f32=(S != 448.0),
                       what=(B, H, Hkv, N, d, block_n, causal, S, order))


@pytest.mark.parametrize("case", range(40))
def test_random_shapes(case):
    """Seeded random problems: batch, GQA group, ragged N, d, block_n, causal or not,
    order, S (powers of two and not), sink count, Delta and O dtype, all against
    the oracle on every row."""
    rng = np.random.default_rng(1000 + case)
    Hkv = int(rng.integers(1, 4))
    group = int(rng.choice([1, 2, 4, 5]))
    B = int(rng.integers(1, 4))
    while B * Hkv * group > 16:
        B -= 1
    if B == 0:
        B, group = 1, 1
    H = Hkv * group
    N = int(rng.integers(1, 1501))
    d = int(rng.choice([64, 128]))
    block_n = int(rng.choice([64, 128]))
    causal = int(rng.integers(0, 2))
    order = int(rng.integers(0, 2))
    S = float(rng.choice([0.5, 1.0, 16.0, 256.0, 300.0, 448.0]))
    n_sink = int(rng.integers(0, min(N, 8) + 1))
    delta = float(rng.uniform(0.0, 12.0))
    f32 = bool(rng.integers(0, 2))
    qk_bf16 = bool(rng.random() < 0.3)      # kernel-faithful mode: BF16 Q and K
    cast_denominator = bool(rng.random() < 0.3)
    what = dict(B=B, H=H, Hkv=Hkv, N=N, d=d, block_n=block_n, causal=causal, order=order, S=S,
                n_sink=n_sink, delta=delta, f32=f32, qk_bf16=qk_bf16,
                cast_denominator=cast_denominator)
    W = workload.make_sink_workload(B, H, Hkv, N, d, n_sink, delta, seed=5000 + case)
    ins = gpu_inputs_bf16(W) if qk_bf16 else gpu_inputs(W)
    if not cast_denominator:
        check_case(W, ins, causal, S, order, block_n, f32=f32, what=what)
        return
    (_, Q8), (_, K8), (_, V8) = ins
    Og, _, _, crow = run_gpu(ins, B, H, Hkv, N, d, causal, S, order, block_n, n_sink, f32,
                             denominator=1)
    Oe, cr, _, slack = oracle.attn_emulate(Q8, K8, V8, B, H, Hkv, N, d, causal, W.scale, S, order,
                                           block_n, n_sink, o_bf16=not f32, denom_mode=1,
                                           flip_slack=True)
    assert np.isfinite(Og).all(), what
    assert_o_close(Og, Oe, what, slack)
    assert_counts_close(crow, cr, what)


@pytest.mark.parametrize("N", [1, 2, 63, 127, 128, 129, 255])
@pytest.mark.parametrize("causal", [0, 1])
def test_edge_lengths(N, causal):
    W = workload.make_sink_workload(1, 2, 1, N, 64, min(4, N), 8.0, seed=1000 + N)
    ins = gpu_inputs(W)
    for order in (0, 1):
        check_case(W, ins, causal, 256.0, order, 64, what=("edge", N, causal, order))
        check_case(W, ins, causal, 1.0, order, 128, what=("edge", N, causal, order))


@pytest.mark.parametrize("n_sink", [0, 128, 256])
def test_sink_counts_extremes(n_sink):
    W = workload.make_sink_workload(1, 1, 1, 256, 128, n_sink, 10.0, seed=77)
    ins = gpu_inputs(W)
    _, tot, sink_tot, _ = check_case(W, ins, 0, 1.0, 0, 128, what=("n_sink", n_sink))
    if n_sink == 256:
        assert tot == 0                               # every key is a sink
    if n_sink == 128:
        assert sink_tot == 0                          # block 0 holds only sinks


def test_short_form_matches_full_form():
    import torch
    from online_softmax_tcgen05_b200 import fp8_attn_fwd
    B, H, N, d = 1, 2, 512, 128
    W = workload.make_sink_workload(B, H, H, N, d, 4, 8.0, seed=5)
    ins = gpu_inputs(W)
    (Qg, _), (Kg, _), (Vg, _) = ins
    O = torch.empty((B, H, N, d), dtype=torch.bfloat16, device="cuda")
    ctr = torch.zeros(1, dtype=torch.int64, device="cuda")
    fp8_attn_fwd(Qg, Kg, Vg, O, B, H, N, d, 1, 1 / math.sqrt(d), 256.0, 1, 4, ctr)
    torch.cuda.synchronize()
    Og, tot, _, _ = run_gpu(ins, B, H, H, N, d, 1, 256.0, 1, 128, 4, f32=False)
    assert np.array_equal(O.float().cpu().numpy().reshape(-1, d), Og)
    assert int(ctr.item()) == tot


def test_host_tensors_end_to_end():
    import torch
    from online_softmax_tcgen05_b200 import attention
    B, H, N, d = 1, 2, 640, 128
    W = workload.make_sink_workload(B, H, 1, N, d, 4, 8.0, seed=6)
    ins = gpu_inputs(W)
    (Qg, Q8), (Kg, K8), (Vg, V8) = ins
    Oh, st_h = attention(torch.from_numpy(Q8), torch.from_numpy(K8), torch.from_numpy(V8),
                         causal=True, S=256.0, kv_order=1, n_sink=4, count_collapse=True)
    Od, st_d = attention(Qg, Kg, Vg, causal=True, S=256.0, kv_order=1, n_sink=4,
                         count_collapse=True)
    torch.cuda.synchronize()
    assert not Oh.is_cuda and Od.is_cuda
    assert torch.equal(Oh, Od.cpu()) and st_h.collapse == st_d.collapse


@pytest.mark.parametrize("chunks", [3, 8])
def test_host_tensors_many_chunks(chunks):
    """The host path with more pieces than staging sets: sets are reused, kernels
    alternate between two compute streams, and pieces cross a batch boundary.
    The result must equal the device path bit for bit, per-row counts included."""
    import torch
    from online_softmax_tcgen05_b200 import attention
    B, H, Hkv, N, d = 2, 8, 4, 1000, 64
    W = workload.make_sink_workload(B, H, Hkv, N, d, 4, 8.0, seed=17)
    ins = gpu_inputs(W)
    (Qg, Q8), (Kg, K8), (Vg, V8) = ins
    kw = dict(causal=True, S=256.0, kv_order=0, n_sink=4, count_collapse=True, per_row=True,
              out_dtype=torch.float32)
    for _ in range(2):   # the second call reuses the cached staging buffers
        Oh, st_h = attention(torch.from_numpy(Q8), torch.from_numpy(K8), torch.from_numpy(V8),
                             host_chunks=chunks, **kw)
    Od, st_d = attention(Qg, Kg, Vg, **kw)
    torch.cuda.synchronize()
    assert torch.equal(Oh, Od.cpu())
    assert st_h.collapse == st_d.collapse and st_h.collapse_sink_block == st_d.collapse_sink_block
    assert torch.equal(st_h.collapse_rows.cpu(), st_d.collapse_rows.cpu())


@pytest.mark.parametrize("qk_bf16,o_f32,pinned,causal", [(False, False, True, 1),
                                                         (True, True, False, 1),
                                                         (False, True, True, 0)])
def test_host_entry_direct(qk_bf16, o_f32, pinned, causal):
    """fp8_attn_fwd_host called directly on a side stream, twice with one plan and
    workspace (the second call reuses every staging set): O, the counters and the
    per-row counts equal the device entry's bit for bit, with pinned or pageable
    host memory, E4M3 or BF16 Q/K, BF16 or FP32 O."""
    import torch
    from online_softmax_tcgen05_b200 import (O_BF16, O_F32, QK_BF16, QK_E4M3, HostPlan,
                                             fp8_attn_fwd_ex, fp8_attn_fwd_host,
                                             host_workspace_bytes)
    B, H, Hkv, N, d = 2, 6, 3, 700, 128
    W = workload.make_sink_workload(B, H, Hkv, N, d, 4, 8.0, seed=31)
    if qk_bf16:
        ins = gpu_inputs_bf16(W)
    else:
        ins = gpu_inputs(W)
    (Qg, _), (Kg, _), (Vg, _) = ins
    o_dt = torch.float32 if o_f32 else torch.bfloat16
    kw = dict(B=B, H=H, H_kv=Hkv, N=N, d=d, causal=causal, S=256.0, kv_order=1, n_sink=4,
              o_dtype=O_F32 if o_f32 else O_BF16, qk_dtype=QK_BF16 if qk_bf16 else QK_E4M3)
    dev = Qg.device
    Od = torch.empty((B, H, N, d), dtype=o_dt, device=dev)
    ctr_d = torch.zeros(2, dtype=torch.int64, device=dev)
    rows_d = torch.zeros((B, H, N), dtype=torch.int32, device=dev)
    fp8_attn_fwd_ex(Qg, Kg, Vg, Od, collapse_ctr=ctr_d[0:1], collapse_sink_ctr=ctr_d[1:2],
                    collapse_rows=rows_d, **kw)
    torch.cuda.synchronize()
    host = [t.cpu() for t in (Qg, Kg, Vg)]
    if pinned:
        host = [t.pin_memory() for t in host]
    plan = HostPlan()
    for chunks in (4, 5):   # pieces of one or two kv heads; first pieces split per head
        ws = torch.empty(host_workspace_bytes(host_chunks=chunks, **{k: kw[k] for k in
                         ("B", "H", "H_kv", "N", "d")}, qk_dtype=kw["qk_dtype"],
                         o_dtype=kw["o_dtype"]), dtype=torch.uint8, device=dev)
        side = torch.cuda.Stream()
        for _ in range(2):
            Oh = torch.full((B, H, N, d), float("nan"), dtype=o_dt)
            if pinned:
                Oh = Oh.pin_memory()
            ctr = torch.zeros(2, dtype=torch.int64, device=dev)
            rows = torch.full((B, H, N), -1, dtype=torch.int32, device=dev)
            side.wait_stream(torch.cuda.current_stream())
            fp8_attn_fwd_host(*host, Oh, plan=plan, workspace=ws, host_chunks=chunks,
                              stream=side, collapse_ctr=ctr[0:1], collapse_sink_ctr=ctr[1:2],
                              collapse_rows=rows, **kw)
            side.synchronize()
            assert torch.equal(Oh, Od.cpu())
            assert torch.equal(ctr.cpu(), ctr_d.cpu())
            assert torch.equal(rows.cpu(), rows_d.cpu())
    plan.close()


def test_empty_problems_are_a_no_op():
    """B, H or N of zero: the call succeeds, launches nothing and leaves the
    counters alone; attention() returns an empty O for device and host inputs."""
    import torch
    from online_softmax_tcgen05_b200 import attention, fp8_attn_fwd_ex
    for B, H, Hkv, N in ((0, 2, 1, 128), (1, 0, 0, 128), (1, 2, 1, 0)):
        q = torch.zeros((B, H, N, 64), dtype=torch.uint8, device="cuda")
        kv = torch.zeros((B, Hkv, N, 64), dtype=torch.uint8, device="cuda")
        O = torch.zeros((B, H, N, 64), dtype=torch.bfloat16, device="cuda")
        ctr = torch.full((2,), 7, dtype=torch.int64, device="cuda")
        fp8_attn_fwd_ex(q, kv, kv, O, B=B, H=H, H_kv=Hkv, N=N, d=64, causal=1,
                        collapse_ctr=ctr[0:1], collapse_sink_ctr=ctr[1:2])
        torch.cuda.synchronize()
        assert ctr.tolist() == [7, 7]
        if H > 0:
            for dev in ("cuda", "cpu"):
                o, st = attention(q.to(dev), kv.to(dev), kv.to(dev), causal=True,
                                  count_collapse=True, per_row=True)
                assert tuple(o.shape) == (B, H, N, 64) and st.collapse == 0
                assert tuple(st.collapse_rows.shape) == (B, H, N)


def test_max_planes_grid():
    """B * H = 65535 (the largest grid the library accepts) with GQA, a ragged
    N and 64-key blocks, causal: sampled rows against the oracle, per-row
    collapse counts exact, first and last planes included."""
    B, H, Hkv, N, d = 3, 21845, 4369, 65, 64
    W = workload.make_sink_workload(B, H, Hkv, N, d, 4, 8.0, seed=29)
    ins = gpu_inputs(W)
    total = B * H * N
    rows = sample_rows(B, H, N, 512, seed=3,
                       include=(0, N - 1, total - N, total - 1, (H - 1) * N + 64))
    check_case(W, ins, 1, 256.0, 1, 64, rows=rows, what="65535 planes")


@pytest.mark.parametrize("causal", [0, 1])
def test_query_row_ranges_compose(causal):
    """Launches over disjoint query-row ranges (q_begin, q_end), in any order,
    reproduce one launch over all rows bit for bit, leave the rows outside their
    range untouched, and their collapse counts add up to the full launch's."""
    import torch
    from online_softmax_tcgen05_b200 import O_F32, fp8_attn_fwd_ex
    B, H, Hkv, N, d = 2, 4, 2, 1000, 128
    W = workload.make_sink_workload(B, H, Hkv, N, d, 4, 8.0, seed=23)
    ins = gpu_inputs(W)
    (Qg, _), (Kg, _), (Vg, _) = ins
    full, tot, sink_tot, crow = run_gpu(ins, B, H, Hkv, N, d, causal, 256.0, 1, 128, 4)
    full = full.reshape(B, H, N, d)
    crow = crow.reshape(B, H, N)
    dev = Qg.device
    O = torch.full((B, H, N, d), float("nan"), dtype=torch.float32, device=dev)
    ctr = torch.zeros(2, dtype=torch.int64, device=dev)
    rows = torch.full((B, H, N), -1, dtype=torch.int32, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    done = np.zeros(N, dtype=bool)
    for lo, hi in ((384, 640), (896, N), (0, 128), (640, 896), (128, 384)):
        fp8_attn_fwd_ex(Qg, Kg, Vg, O, B=B, H=H, H_kv=Hkv, N=N, d=d, causal=causal,
                        scale=1.0 / math.sqrt(d), S=256.0, kv_order=1, n_sink=4, o_dtype=O_F32,
                        collapse_ctr=ctr[0:1], collapse_sink_ctr=ctr[1:2], collapse_rows=rows,
                        status_word=status, q_begin=lo, q_end=hi)
        torch.cuda.synchronize()
        assert int(status.item()) == 0, hex(int(status.item()))
        done[lo:hi] = True
        Oc, rc = O.cpu().numpy(), rows.cpu().numpy()
        assert np.array_equal(Oc[:, :, done], full[:, :, done])
        assert np.isnan(Oc[:, :, ~done]).all()
        assert np.array_equal(rc[:, :, done], crow[:, :, done])
        assert (rc[:, :, ~done] == -1).all()
    c = ctr.cpu().numpy()
    assert int(c[0]) == tot and int(c[1]) == sink_tot


# ------------------------------------------------------------ sweep (cfg 2) --
@pytest.fixture(scope="module")
def sweep_inputs():
    out = {}
    for delta in range(0, 13):
        W = workload.make_sink_workload(1, 8, 8, 4096, 128, 4, float(delta),
                                        seed=workload.CONFIG_SEED_BASE + 2)
        out[delta] = (W, gpu_inputs(W))
    return out


def test_sweep_collapse_and_closed_form(sweep_inputs):
    rows = sample_rows(1, 8, 4096, 512, seed=2)
    full_frac = {}
    for delta in range(0, 13):
        W, ins = sweep_inputs[delta]
        for S in (1.0, 16.0, 256.0, 448.0):
            for order in ((0, 1) if delta in (0, 6, 8, 12) else (0,)):
                _, tot, sink_tot, _ = check_case(W, ins, 0, S, order, 128, rows=rows,
                                                 what=("sweep", delta, S, order))
                full_frac[(delta, S, order)] = tot / (8 * 4096 * 4092)
                if order == 1 and S == 256.0:
                    assert tot == sink_tot
    for S in (1.0, 16.0, 256.0, 448.0):
        F = [full_frac[(dl, S, 0)] for dl in range(13)]
        assert all(b >= a - 1e-4 for a, b in zip(F, F[1:])), (S, F)     # monotone in Delta
        dc = oracle.delta_c(S)
        if F[-1] > 0.5:
            cross = next(i for i, f in enumerate(F) if f >= 0.5)
            lo = cross - 1 + (0.5 - F[cross - 1]) / (F[cross] - F[cross - 1])
            assert abs(lo - dc) <= 1.0, (S, lo, dc, F)
        else:
            assert dc > 11.0                                            # S = 256, 448


# Full-problem collapse totals (every row, every pair) at points of the sweep
# that span the regimes: forward S = 1 across the collapse onset, S = 16 at its
# threshold, S = 256 / 448 where forward order starts to collapse, and reverse
# order (collapse confined to the sink block).
SWEEP_FULL_POINTS = [(6, 1.0, 0), (8, 1.0, 0), (8, 16.0, 0), (10, 16.0, 0), (10, 256.0, 0),
                     (12, 448.0, 0), (12, 256.0, 1), (7, 1.0, 1)]


def test_sweep_full_problem_totals(sweep_inputs):
    """All 32768 rows of the sweep configuration at eight (Delta, S, order)
    points: O within tolerance, per-row counts within 2 keys, the total and the
    sink-block sub-count within max(2, 1e-4) of the oracle's."""
    for delta, S, order in SWEEP_FULL_POINTS:
        W, ins = sweep_inputs[delta]
        _, tot, sink_tot, crow = check_case(W, ins, 0, S, order, 128,
                                            what=("sweep full", delta, S, order))
        print("sweep full Delta=%d S=%g order=%d: collapse %d (sink block %d)"
              % (delta, S, order, tot, sink_tot))


def _mse_table(ins, W, configs, rows):
    """MSE against float64 attention of the kernel's outputs and of the oracle's
    emulation, per (order, S), on the given sampled rows."""
    (_, Q8), (_, K8), (_, V8) = ins
    H, N, d = W.H, W.N, W.d
    ref = oracle.attn_exact(Q8, K8, V8, 1, H, H, N, d, 0, W.scale, rows=rows)
    gpu, emu = {}, {}
    for order, S in configs:
        Og, *_ = run_gpu(ins, 1, H, H, N, d, 0, S, order, 128, 4)
        Oe, _, _ = oracle.attn_emulate(Q8, K8, V8, 1, H, H, N, d, 0, W.scale, S, order, 128, 4,
                                       rows=rows)
        gpu[(order, S)] = float(np.mean((Og[rows] - ref) ** 2))
        emu[(order, S)] = float(np.mean((Oe - ref) ** 2))
    return gpu, emu


def test_sweep_mse_orderings(sweep_inputs):
    """The MSE comparisons of the pages (Experimental results) on the kernel's
    outputs for the sink-construction sweep at Delta = 7: the kernel's MSE
    against float64 attention equals the oracle emulation's within 2% for every
    configuration; forward S = 1 is the worst configuration and reverse + 256
    matches forward + 256.  The magnitudes (pages: 3-10x, S = 256 10-15% below
    448) are pinned on the pages' own logit model in the oracle tests; this
    construction gives smaller ones (its sink logits carry extra variance) and
    they are printed, not gated."""
    W, ins = sweep_inputs[7]
    rows = sample_rows(1, 8, 4096, 2048, seed=5)
    configs = [(0, 1.0), (0, 256.0), (0, 448.0), (1, 256.0), (1, 1.0)]
    gpu, emu = _mse_table(ins, W, configs, rows)
    for c in configs:
        assert abs(gpu[c] / emu[c] - 1) < 0.02, (c, gpu, emu)
    base = gpu[(0, 1.0)]
    best = min(gpu[(0, 256.0)], gpu[(1, 256.0)], gpu[(1, 1.0)])
    assert base == max(gpu.values()) and base / best > 1.5, gpu
    assert abs(gpu[(1, 256.0)] / gpu[(0, 256.0)] - 1) < 0.1, gpu
    print("sweep Delta=7 MSE: forward S=1 / best %.3f, S256 / S448 %.3f, reverse256 / "
          "forward256 %.3f" % (base / best, gpu[(0, 256.0)] / gpu[(0, 448.0)],
                                gpu[(1, 256.0)] / gpu[(0, 256.0)]))


# --------------------------------------------------------- full-size cases ---
# Sampled rows: 4096 per configuration, spread over every (batch, head) plane
# (so over every causal scheduling group), with each plane's first and last
# row, a row of its last query tile and last rows of tiles (their diagonal KV
# block holds the most visible keys).


def test_prefill_gqa_causal_full_size():
    B, H, Hkv, N, d = 1, 32, 8, 32768, 128
    W = workload.make_sink_workload(B, H, Hkv, N, d, 4, 8.0, seed=workload.CONFIG_SEED_BASE + 3)
    ins = gpu_inputs(W)
    rows = coverage_rows(B, H, N, 128, seed=3)
    assert rows.size == 4096
    _, tot, sink_tot, _ = check_case(W, ins, 1, 256.0, 1, 128, f32=False, rows=rows,
                                     what="prefill")
    assert tot == sink_tot                                 # reverse + 256: none outside
    check_case(W, ins, 1, 1.0, 0, 128, f32=False, rows=rows, what="prefill fwd S1")


def test_batched_noncausal_full_size():
    B, H, N, d = 4, 32, 8192, 128
    W = workload.make_sink_workload(B, H, H, N, d, 4, 10.0, seed=workload.CONFIG_SEED_BASE + 4)
    ins = gpu_inputs(W)
    rows = coverage_rows(B, H, N, 32, seed=4)
    assert rows.size == 4096
    for order in (0, 1):
        check_case(W, ins, 0, 256.0, order, 128, f32=False, rows=rows, what=("batched", order))


def test_long_context_full_size():
    B, H, Hkv, N, d = 1, 32, 8, 131072, 128
    W = workload.make_sink_workload(B, H, Hkv, N, d, 4, 10.0, seed=workload.CONFIG_SEED_BASE + 5)
    ins = gpu_inputs(W)
    rows = coverage_rows(B, H, N, 128, seed=5)
    assert rows.size == 4096
    _, tot, sink_tot, _ = check_case(W, ins, 1, 256.0, 1, 128, f32=False, rows=rows,
                                     what="long rev 256")
    # Reverse + 256 leaves (almost) nothing outside the sink block.  The paper's
    # < 1e-12 bound is for unit-variance logits; here the per-row logit spread
    # varies with |g_i|, so at N = 131072 a few far-tail entries can underflow.
    # With n_sink = block_n only entries outside the sink block are counted (the
    # arithmetic is unchanged): the rows holding them must agree with the oracle.
    pairs = H * N * (N + 1) // 2
    assert (tot - sink_tot) / pairs < 1e-9
    _, out_tot, _, out_rows = run_gpu(ins, B, H, Hkv, N, d, 1, 256.0, 1, 128, 128, f32=False)
    assert out_tot == tot - sink_tot
    hit = np.flatnonzero(out_rows)
    if hit.size:
        (_, Q8), (_, K8), (_, V8) = ins
        _, cr, _ = oracle.attn_emulate(Q8, K8, V8, B, H, Hkv, N, d, 1, W.scale, 256.0, 1, 128,
                                       128, o_bf16=True, rows=hit)
        assert np.abs(cr.astype(np.int64) - out_rows[hit]).sum() <= 1, (hit, cr, out_rows[hit])
    check_case(W, ins, 1, 1.0, 0, 128, f32=False, rows=rows, what="long fwd 1")


def test_mse_gain_grows_with_sequence_length_on_gpu():
    """The paper's sequence-length claim on the kernel's own outputs: the MSE
    (against float64 attention on the same E4M3 inputs) of forward S = 1 over
    reverse S = 256 grows with N, from 1k to 128k keys."""
    gains = []
    for N in (1024, 4096, 16384, 65536, 131072):
        B, H, d = 1, 2, 128
        W = workload.make_sink_workload(B, H, H, N, d, 4, 7.0, seed=workload.CONFIG_SEED_BASE + 6)
        ins = gpu_inputs(W)
        (_, Q8), (_, K8), (_, V8) = ins
        rows = sample_rows(B, H, N, 128, seed=9)
        ref = oracle.attn_exact(Q8, K8, V8, B, H, H, N, d, 0, W.scale, rows=rows)
        mse = {}
        for order, S in ((0, 1.0), (1, 256.0)):
            Og, *_ = run_gpu(ins, B, H, H, N, d, 0, S, order, 128, 4)
            mse[(order, S)] = float(np.mean((Og[rows] - ref) ** 2))
        gains.append(mse[(0, 1.0)] / mse[(1, 256.0)])
    assert all(a < b for a, b in zip(gains, gains[1:])), gains
    assert gains[-1] > 4 * gains[0], gains



@pytest.mark.parametrize("B,H,Hkv,N,d,block_n,causal", [(1, 2, 1, 700, 128, 128, 1),
                                                        (1, 2, 2, 520, 64, 64, 0)])
def test_cast_denominator_parity(B, H, Hkv, N, d, block_n, causal):
    """Row sum from the cast values (FP8ATTN_DENOM_CAST_P) against the oracle."""
    W = workload.make_sink_workload(B, H, Hkv, N, d, 4, 9.0, seed=60 + N)
    ins = gpu_inputs(W)
    (_, Q8), (_, K8), (_, V8) = ins
    for S in (1.0, 256.0, 448.0):
        for order in (0, 1):
            Og, *_ = run_gpu(ins, B, H, Hkv, N, d, causal, S, order, block_n, 4, denominator=1)
            Oe, _, _, slack = oracle.attn_emulate(Q8, K8, V8, B, H, Hkv, N, d, causal, W.scale, S,
                                                  order, block_n, 4, denom_mode=1, flip_slack=True)
            assert_o_close(Og, Oe, ("cast denominator", S, order), slack)



@pytest.mark.parametrize("B,H,Hkv,N,d,block_n,causal", [(1, 2, 1, 384, 128, 128, 1),
                                                        (1, 2, 2, 1000, 128, 64, 1),
                                                        (2, 2, 1, 520, 64, 128, 0),
                                                        (1, 1, 1, 333, 64, 64, 1)])
def test_bf16_qk_parity(B, H, Hkv, N, d, block_n, causal):
    """Kernel-faithful mode: QK^T on BF16 Q and K (tcgen05 kind::f16), P~ and V
    E4M3, against the oracle in the same mode."""
    W = workload.make_sink_workload(B, H, Hkv, N, d, 4, 9.0, seed=70 + N + d)
    ins = gpu_inputs_bf16(W)
    for S in (1.0, 256.0, 448.0):
        for order in (0, 1):
            check_case(W, ins, causal, S, order, block_n, f32=(S != 448.0),
                       what=("bf16 qk", B, H, Hkv, N, d, block_n, causal, S, order))


def test_bf16_qk_mse_orderings_on_gpu():
    """The same MSE comparisons with unquantised (BF16) Q and K, the pages'
    kernel-faithful setting for Q and K: kernel MSE = oracle MSE within 2% per
    configuration, forward S = 1 the worst, reverse + 256 = forward + 256."""
    W = workload.make_sink_workload(1, 8, 8, 4096, 128, 4, 7.0, seed=workload.CONFIG_SEED_BASE + 2)
    ins = gpu_inputs_bf16(W)
    rows = sample_rows(1, 8, 4096, 2048, seed=5)
    configs = [(0, 1.0), (0, 256.0), (0, 448.0), (1, 256.0)]
    gpu, emu = _mse_table(ins, W, configs, rows)
    for c in configs:
        assert abs(gpu[c] / emu[c] - 1) < 0.02, (c, gpu, emu)
    base = gpu[(0, 1.0)]
    assert base == max(gpu.values()) and base / min(gpu[(0, 256.0)], gpu[(1, 256.0)]) > 1.5, gpu
    assert abs(gpu[(1, 256.0)] / gpu[(0, 256.0)] - 1) < 0.1, gpu
    print("bf16 Q/K Delta=7 MSE: forward S=1 / best %.3f, S256 / S448 %.3f"
          % (base / min(gpu[(0, 256.0)], gpu[(1, 256.0)]), gpu[(0, 256.0)] / gpu[(0, 448.0)]))


# ------------------------------------------------- S not a power of two ------
@pytest.mark.parametrize("S", [300.0, 448.0])
def test_non_power_of_two_S_matches_oracle(S):
    """For S not a power of two the kernel forms fl(S * p) with an FP32 multiply
    and divides by fl(S * l), the steps the pages give (Optimality of S=256,
    condition 1: a non-power-of-two S rounds in the scaling).  Sweep-shaped
    problem at the sink strengths where forward order starts to collapse for
    these S (Delta_c = 11.6 and 12.0): every row against the oracle, per-row
    counts within 2 keys; the observed disagreement is printed."""
    B, H, N, d = 1, 4, 4096, 128
    for delta, causal in ((12.0, 0), (10.0, 1)):
        W = workload.make_sink_workload(B, H, H, N, d, 4, delta,
                                        seed=workload.CONFIG_SEED_BASE + 2)
        ins = gpu_inputs(W)
        (_, Q8), (_, K8), (_, V8) = ins
        for order in (0, 1):
            Og, tot, _, crow = run_gpu(ins, B, H, H, N, d, causal, S, order, 128, 4)
            Oe, cr, _, slack = oracle.attn_emulate(Q8, K8, V8, B, H, H, N, d, causal, W.scale, S,
                                                   order, 128, 4, flip_slack=True)
            what = ("S", S, "delta", delta, "causal", causal, "order", order)
            assert_o_close(Og, Oe, what, slack)
            worst, dtot = assert_counts_close(crow, cr, what)
            diff_rows = int(np.count_nonzero(crow != cr.astype(np.int64)))
            print("S=%g Delta=%g causal=%d order=%d: collapse gpu %d oracle %d, rows differing "
                  "%d of %d, worst row %d" % (S, delta, causal, order, tot, int(cr.sum()),
                                              diff_rows, crow.size, worst))


# ----------------------------------------- head-sharded long context (NEXT) --
def test_kv_head_shards_equal_the_full_launch():
    """The multi-GPU split of the long-context problem (each rank owns whole kv
    heads and their query heads) on one GPU: the problem at N = 16384 as 2 and
    then 4 kv-head shards, each generated on its own with
    make_sink_workload(kv_heads=...) as a rank does, launched one after
    another.  Each shard's inputs equal the full problem's slice byte for byte,
    its O equals the full launch's heads bit for bit, its per-row counts equal,
    and the shards' collapse counters add up to the full launch's exactly."""
    import torch
    B, H, Hkv, N, d = 1, 32, 8, 16384, 128
    seed = workload.CONFIG_SEED_BASE + 5
    group = H // Hkv
    W = workload.make_sink_workload(B, H, Hkv, N, d, 4, 10.0, seed=seed)
    ins = gpu_inputs(W)
    (Qg, _), (Kg, _), (Vg, _) = ins
    for S, order in ((256.0, 1), (1.0, 0)):
        full, tot, sink_tot, crow = run_gpu(ins, B, H, Hkv, N, d, 1, S, order, 128, 4, f32=False)
        full = full.reshape(B, H, N, d)
        crow = crow.reshape(B, H, N)
        for shards in (2, 4):
            per = Hkv // shards
            s_tot = s_sink = 0
            for r in range(shards):
                g0, g1 = r * per, (r + 1) * per
                Ws = workload.make_sink_workload(B, H, Hkv, N, d, 4, 10.0, seed=seed,
                                                 kv_heads=(g0, g1))
                ins_s = gpu_inputs(Ws)
                (Qs, _), (Ks, _), (Vs, _) = ins_s
                assert torch.equal(Qs, Qg[:, g0 * group:g1 * group])
                assert torch.equal(Ks, Kg[:, g0:g1]) and torch.equal(Vs, Vg[:, g0:g1])
                Os, t, st, rs = run_gpu(ins_s, B, Ws.H, Ws.Hkv, N, d, 1, S, order, 128, 4,
                                        f32=False)
                assert np.array_equal(Os.reshape(B, Ws.H, N, d),
                                      full[:, g0 * group:g1 * group]), (S, order, shards, r)
                assert np.array_equal(rs.reshape(B, Ws.H, N), crow[:, g0 * group:g1 * group])
                s_tot += t
                s_sink += st
            assert (s_tot, s_sink) == (tot, sink_tot), (S, order, shards, s_tot, tot)


# ------------------------------------------------ attention() on a stream ----
def test_attention_on_a_side_stream_counts():
    """attention() on device tensors with stream= a side stream: the counters are
    zeroed before the kernel runs and read after it, and O and the counts equal
    the oracle's (O within tolerance, counts within the collapse rule)."""
    import torch
    from online_softmax_tcgen05_b200 import attention
    B, H, Hkv, N, d = 1, 4, 2, 2048, 128
    W = workload.make_sink_workload(B, H, Hkv, N, d, 4, 9.0, seed=81)
    ins = gpu_inputs(W)
    (Qg, Q8), (Kg, K8), (Vg, V8) = ins
    side = torch.cuda.Stream()
    Oe, cr, ctot, slack = oracle.attn_emulate(Q8, K8, V8, B, H, Hkv, N, d, 1, W.scale, 1.0, 0, 128,
                                              4, flip_slack=True)
    for _ in range(3):
        O, st = attention(Qg, Kg, Vg, causal=True, S=1.0, kv_order=0, n_sink=4,
                          count_collapse=True, per_row=True, out_dtype=torch.float32,
                          stream=side)
        torch.cuda.current_stream().synchronize()
        assert_o_close(O.cpu().numpy().reshape(-1, d), Oe, "side stream", slack)
        assert_counts_close(st.collapse_rows.cpu().numpy().reshape(-1), cr, "side stream")
        assert abs(st.collapse - int(ctot.sum())) <= total_tol(ctot.sum())
        assert abs(st.collapse_sink_block - int(ctot[0])) <= total_tol(ctot[0])


def test_attention_rejects_mixed_devices():
    """Inputs on different devices (or a host tensor among device tensors) are
    refused before anything is launched."""
    import torch
    from online_softmax_tcgen05_b200 import attention
    q = torch.zeros((1, 1, 128, 64), dtype=torch.uint8, device="cuda")
    with pytest.raises(ValueError):
        attention(q, q.cpu(), q)
    with pytest.raises(ValueError):
        attention(q, q, q, out=torch.empty((1, 1, 128, 64), dtype=torch.bfloat16))


# ------------------------------------------------- two-tile schedule --------
SCHED_CASES = [
    # B, H, Hkv, N, d, block_n, causal, S, order, qk_bf16, denominator, o_f32
    (1, 8, 2, 4096, 128, 128, 1, 256.0, 1, False, 0, False),   # GQA: head pairs
    (1, 8, 2, 4096, 128, 128, 0, 1.0, 0, False, 0, True),
    (2, 3, 3, 1000, 128, 128, 1, 256.0, 1, False, 0, True),    # MHA: tile pairs, odd tiles
    (1, 2, 2, 1000, 128, 64, 1, 448.0, 0, False, 0, True),     # block_n 64, S = 448
    (2, 4, 2, 520, 64, 64, 0, 300.0, 1, False, 0, False),      # d 64, S = 300
    (1, 4, 1, 777, 64, 128, 1, 16.0, 0, False, 0, True),       # group 4, ragged
    (1, 5, 1, 333, 128, 128, 1, 256.0, 1, False, 0, True),     # odd group: tile pairs
    (1, 4, 2, 700, 128, 128, 1, 256.0, 1, True, 0, True),      # BF16 Q/K
    (1, 2, 1, 700, 128, 128, 1, 448.0, 0, False, 1, True),     # cast-value denominator
    (1, 2, 2, 100, 128, 128, 1, 256.0, 1, False, 0, True),     # one tile: B tile empty
]


@pytest.mark.parametrize("case", SCHED_CASES)
def test_two_tile_schedule_equals_one_tile(case):
    """The two-tile schedule (two query tiles per CTA, exponential turns) against
    the default one-tile schedule: same O bit for bit, same counters and per-row
    counts.  The one-tile kernel is the one checked against the oracle above."""
    from online_softmax_tcgen05_b200 import SCHEDULE_ONE_TILE, SCHEDULE_TWO_TILES, set_schedule
    B, H, Hkv, N, d, block_n, causal, S, order, qk_bf16, denom, f32 = case
    W = workload.make_sink_workload(B, H, Hkv, N, d, 4, 9.0, seed=3000 + N + H)
    ins = gpu_inputs_bf16(W) if qk_bf16 else gpu_inputs(W)
    outs = []
    try:
        for sched in (SCHEDULE_ONE_TILE, SCHEDULE_TWO_TILES):
            set_schedule(sched)
            outs.append(run_gpu(ins, B, H, Hkv, N, d, causal, S, order, block_n, 4, f32,
                                denominator=denom))
    finally:
        set_schedule(SCHEDULE_ONE_TILE)
    (O1, t1, s1, r1), (O2, t2, s2, r2) = outs
    assert np.array_equal(O1, O2, equal_nan=False), (case, np.abs(O1 - O2).max())
    assert (t1, s1) == (t2, s2) and np.array_equal(r1, r2), case


def test_two_tile_schedule_row_ranges():
    """Query-row ranges with the two-tile schedule (a range of an odd number of
    tiles leaves the second tile of the last pair outside the range): the rows
    of each range equal the full launch's, the others stay untouched."""
    import torch
    from online_softmax_tcgen05_b200 import (O_F32, SCHEDULE_ONE_TILE, SCHEDULE_TWO_TILES,
                                             fp8_attn_fwd_ex, set_schedule)
    B, H, Hkv, N, d = 1, 4, 4, 1000, 128
    W = workload.make_sink_workload(B, H, Hkv, N, d, 4, 8.0, seed=23)
    ins = gpu_inputs(W)
    (Qg, _), (Kg, _), (Vg, _) = ins
    full, tot, sink_tot, crow = run_gpu(ins, B, H, Hkv, N, d, 1, 256.0, 1, 128, 4)
    full = full.reshape(B, H, N, d)
    try:
        set_schedule(SCHEDULE_TWO_TILES)
        O = torch.full((B, H, N, d), float("nan"), dtype=torch.float32, device=Qg.device)
        ctr = torch.zeros(2, dtype=torch.int64, device=Qg.device)
        done = np.zeros(N, dtype=bool)
        for lo, hi in ((384, 640), (0, 128), (640, N), (128, 384)):
            fp8_attn_fwd_ex(Qg, Kg, Vg, O, B=B, H=H, H_kv=Hkv, N=N, d=d, causal=1, S=256.0,
                            kv_order=1, n_sink=4, o_dtype=O_F32, collapse_ctr=ctr[0:1],
                            collapse_sink_ctr=ctr[1:2], q_begin=lo, q_end=hi)
            torch.cuda.synchronize()
            done[lo:hi] = True
            Oc = O.cpu().numpy()
            assert np.array_equal(Oc[:, :, done], full[:, :, done])
            assert np.isnan(Oc[:, :, ~done]).all()
        c = ctr.cpu().numpy()
        assert int(c[0]) == tot and int(c[1]) == sink_tot
    finally:
        set_schedule(SCHEDULE_ONE_TILE)


@pytest.mark.parametrize("schedule", [0, 1])
@pytest.mark.parametrize("order", [0, 1])
def test_nan_input_reaches_exactly_the_rows_that_see_it(schedule, order):
    """A NaN E4M3 byte in K makes the O rows of every query that sees that key
    NaN (both on a key whose exponential takes the FMA-pipe 2^x and on one that
    takes MUFU ex2), a NaN byte in Q makes its own row NaN, and every other row
    equals the clean run bit for bit (with the same counts per row)."""
    import torch
    from online_softmax_tcgen05_b200 import SCHEDULE_ONE_TILE, set_schedule
    B, H, Hkv, N, d = 1, 2, 1, 1000, 128
    W = workload.make_sink_workload(B, H, Hkv, N, d, 4, 8.0, seed=41)
    ins = gpu_inputs(W)
    (Qg, Q8), (Kg, K8), (Vg, V8) = ins
    # key 300: key pair 150, position 150 % 8 = 6 of its group of 8 pairs (MUFU);
    # key 513: pair 256, position 0 (the FMA-pipe positions are the first ones)
    kbad, qbad = (300, 513), 100
    K2, Q2 = Kg.clone(), Qg.clone()
    for j in kbad:
        K2[0, 0, j, 5] = 0x7F
    Q2[0, 1, qbad, 9] = 0x7F
    ins2 = ((Q2, Q8), (K2, K8), (Vg, V8))
    try:
        set_schedule(schedule)
        clean = run_gpu(ins, B, H, Hkv, N, d, 1, 256.0, order, 128, 4)
        bad = run_gpu(ins2, B, H, Hkv, N, d, 1, 256.0, order, 128, 4)
    finally:
        set_schedule(SCHEDULE_ONE_TILE)
    Oc, Ob = clean[0].reshape(H, N, d), bad[0].reshape(H, N, d)
    rc, rb = clean[3].reshape(H, N), bad[3].reshape(H, N)
    sees = np.zeros((H, N), dtype=bool)
    sees[:, min(kbad):] = True          # causal: query i sees key j iff j <= i
    sees[1, qbad] = True
    assert np.isnan(Ob[sees]).all()
    assert np.isfinite(Oc).all()
    assert np.array_equal(Ob[~sees], Oc[~sees])
    assert np.array_equal(rb[~sees], rc[~sees])
