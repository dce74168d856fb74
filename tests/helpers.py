"""Shared helpers of the GPU parity tests: seeded inputs cast on both sides,
and the comparison rules (tolerances of the attention forward:
max |dO| <= 2e-2, relative RMS <= 5e-3, collapse fraction within 1% absolute)."""
import numpy as np

import oracle
import workload

O_MAX_ABS = 2e-2
O_REL_RMS = 5e-3
COLLAPSE_ABS = 0.01


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


def assert_o_close(O_gpu, O_ref, what=""):
    max_abs, rel_rms = compare_o(O_gpu, O_ref)
    assert max_abs <= O_MAX_ABS and rel_rms <= O_REL_RMS, (what, max_abs, rel_rms)
    return max_abs, rel_rms


def sample_rows(B, H, N, n, seed=0, include=()):
    rng = np.random.default_rng(seed)
    total = B * H * N
    rows = set(int(r) for r in rng.choice(total, min(n, total), replace=False))
    rows.update(int(r) for r in include if 0 <= r < total)
    return np.array(sorted(rows), dtype=np.int64)


__all__ = ["gpu_inputs", "gpu_inputs_bf16", "compare_o", "assert_o_close", "sample_rows", "O_MAX_ABS", "O_REL_RMS",
           "COLLAPSE_ABS", "oracle", "workload"]
