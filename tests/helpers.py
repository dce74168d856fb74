"""Shared helpers of the GPU parity tests: seeded inputs cast on both sides,
and the comparison rules.

Attention output: max |dO| <= 2e-2 and relative RMS <= 5e-3 against the
oracle's emulation (the tensor core accumulates in another order).

Collapse counts: per query row the kernel's count may differ from the
oracle's by at most 2 keys, and a whole-problem (or whole-sample) total by at
most max(2, 1e-4 of the oracle's total).  The kernel's exponential (ex2) and
its QK^T accumulation order move a probability by a few FP32 ulps, which can
flip only an entry that lies within those ulps of the cast's zero threshold
2^-10 (or of an E4M3 rounding midpoint); a systematic miscount (a masking or
sink-boundary error) moves whole columns of keys and fails these bounds.
"""
import numpy as np

import oracle
import workload

O_MAX_ABS = 2e-2
O_REL_RMS = 5e-3
COLLAPSE_ROW_KEYS = 2
COLLAPSE_TOTAL_REL = 1e-4


def total_tol(ref_total):
    """Allowed |kernel - oracle| of a collapse total."""
    return max(2.0, COLLAPSE_TOTAL_REL * float(ref_total))


def assert_counts_close(gpu_rows, ref_rows, what=""):
    """Per-row collapse counts within COLLAPSE_ROW_KEYS, their sum within total_tol."""
    g = np.asarray(gpu_rows, dtype=np.int64)
    r = np.asarray(ref_rows, dtype=np.int64)
    d = np.abs(g - r)
    worst = int(d.max()) if d.size else 0
    assert worst <= COLLAPSE_ROW_KEYS, (what, "row", worst, int(np.argmax(d)))
    assert abs(int(g.sum()) - int(r.sum())) <= total_tol(r.sum()), (what, g.sum(), r.sum())
    return worst, int(g.sum()) - int(r.sum())


def gpu_inputs(W, dev="cuda"):
    """E4M3 bytes of W's Q, K, V cast on the GPU by the library, plus the
    oracle's own cast of the same FP32 values (they must agree bit for bit)."""
    import torch
    from online_softmax_tcgen05_b200 import e4m3_cast
    out = []
    for x in (W.q, W.k, W.v):
        g = e4m3_cast(torch.from_numpy(x).to(dev))
        o = oracle.e4m3_encode(x)
        assert np.array_equal(g.cpu().numpy(), o), "GPU and oracle E4M3 casts of the inputs differ"
        out.append((g, o))
    return out


def gpu_inputs_bf16(W, dev="cuda"):
    """BF16 Q and K (the kernel-faithful mode) and E4M3 V: the GPU side rounds
    with torch, the oracle side with its own RNE; the bits must agree."""
    import torch
    from online_softmax_tcgen05_b200 import e4m3_cast
    out = []
    for x in (W.q, W.k):
        g = torch.from_numpy(x).to(dev).to(torch.bfloat16)
        o = oracle.bf16_bits(x)
        assert np.array_equal(g.view(torch.int16).cpu().numpy().view(np.uint16), o)
        out.append((g, o))
    g = e4m3_cast(torch.from_numpy(W.v).to(dev))
    o = oracle.e4m3_encode(W.v)
    assert np.array_equal(g.cpu().numpy(), o)
    out.append((g, o))
    return out


def compare_o(O_gpu, O_ref):
    O_gpu = np.asarray(O_gpu, dtype=np.float64)
    O_ref = np.asarray(O_ref, dtype=np.float64)
    diff = O_gpu - O_ref
    max_abs = float(np.abs(diff).max()) if diff.size else 0.0
    rms_ref = float(np.sqrt(np.mean(O_ref ** 2))) if diff.size else 1.0
    rel_rms = float(np.sqrt(np.mean(diff ** 2)) / max(rms_ref, 1e-30)) if diff.size else 0.0
    return max_abs, rel_rms


def assert_o_close(O_gpu, O_ref, what="", slack=None):
    """Relative RMS <= O_REL_RMS over all rows; per row max |dO| <= O_MAX_ABS plus
    that row's flip slack from the oracle (attn_emulate(..., flip_slack=True)):
    where the oracle's fl32(S p) lies within a relative 2^-14 of an E4M3 rounding
    boundary, the kernel's p (a few ulps away: another exponential, another
    QK^T summation order) may round to the neighbouring E4M3 value, and that
    one step of a large P entry moves O by more than the accumulation-order
    tolerance.  Both sides take the decision in FP32; only the ulps differ."""
    max_abs, rel_rms = compare_o(O_gpu, O_ref)
    assert rel_rms <= O_REL_RMS, (what, max_abs, rel_rms)
    if max_abs > O_MAX_ABS:
        assert slack is not None, (what, max_abs, rel_rms)
        d = np.abs(np.asarray(O_gpu, np.float64) - np.asarray(O_ref, np.float64)).max(axis=1)
        excess = d - (O_MAX_ABS + np.asarray(slack, np.float64))
        assert excess.max() <= 0, (what, max_abs, rel_rms, int(np.argmax(excess)),
                                   float(d.max()), float(np.asarray(slack)[np.argmax(excess)]))
    return max_abs, rel_rms


def sample_rows(B, H, N, n, seed=0, include=()):
    rng = np.random.default_rng(seed)
    total = B * H * N
    rows = set(int(r) for r in rng.choice(total, min(n, total), replace=False))
    rows.update(int(r) for r in include if 0 <= r < total)
    return np.array(sorted(rows), dtype=np.int64)


def coverage_rows(B, H, N, per_plane, seed=0, block_n=128):
    """Sampled query rows that cover every (batch, head) plane: per plane the
    first and last row, a row of the last query tile, a row just below the
    diagonal of a random tile (i % 128 = 127: the last row of its tile, whose
    diagonal KV block is the fullest), a row at the start of a tile, and the rest
    at random.  Global row indices (b * H + h) * N + i, sorted."""
    rng = np.random.default_rng(seed)
    out = []
    nt = (N + 127) // 128
    for bh in range(B * H):
        base = bh * N
        picks = {0, N - 1, max(N - 1 - int(rng.integers(0, min(128, N))), 0)}
        t = int(rng.integers(0, nt))
        picks.add(min(t * 128 + 127, N - 1))
        picks.add(min(int(rng.integers(0, nt)) * 128, N - 1))
        while len(picks) < min(per_plane, N):
            picks.add(int(rng.integers(0, N)))
        out.extend(base + i for i in picks)
    return np.array(sorted(out), dtype=np.int64)


__all__ = ["gpu_inputs", "gpu_inputs_bf16", "compare_o", "assert_o_close", "sample_rows",
           "coverage_rows", "assert_counts_close", "total_tol", "O_MAX_ABS", "O_REL_RMS",
           "COLLAPSE_ROW_KEYS", "COLLAPSE_TOTAL_REL", "oracle", "workload"]
