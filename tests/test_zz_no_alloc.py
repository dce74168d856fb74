"""fp8_attn_fwd_host_noalloc: the host-buffer attention entry for callers that
cannot allocate device memory (code living under another allocator that owns
the device, serving loops that forbid allocation after start-up, plain C
callers without a CUDA allocator).  It stages through the library's own fixed
device array instead of a caller workspace.

The GPU test calls it through the C ABI twice in a row, on two different
problems (so the second call runs over the first call's leftover staging
contents), and checks each result against the existing host-buffer entry
fp8_attn_fwd_host on the same inputs: O within the attention tolerances
(max |dO| <= 2e-2, relative RMS <= 5e-3), collapse counts and per-row counts
equal.  This file is collected last on purpose.
"""
import ctypes

import numpy as np
import pytest

from helpers import assert_o_close, gpu_inputs, workload


def _kw(B, H, Hkv, N, d, causal, S, order, o_f32):
    from online_softmax_tcgen05_b200 import O_BF16, O_F32
    return dict(B=B, H=H, H_kv=Hkv, N=N, d=d, causal=causal, S=S, kv_order=order, n_sink=4,
                o_dtype=O_F32 if o_f32 else O_BF16)


def _run_pair(case, seed, plan):
    """One problem through both host entries; returns nothing, asserts parity."""
    import torch
    from online_softmax_tcgen05_b200 import (fp8_attn_fwd_host, fp8_attn_fwd_host_noalloc,
                                             host_workspace_bytes)
    B, H, Hkv, N, d, causal, S, order, o_f32, pinned = case
    W = workload.make_sink_workload(B, H, Hkv, N, d, 4, 8.0, seed=seed)
    (Qg, _), (Kg, _), (Vg, _) = gpu_inputs(W)
    host = [t.cpu() for t in (Qg, Kg, Vg)]
    if pinned:
        host = [t.pin_memory() for t in host]
    kw = _kw(B, H, Hkv, N, d, causal, S, order, o_f32)
    dev = Qg.device
    o_dt = torch.float32 if o_f32 else torch.bfloat16
    outs = []
    for noalloc in (False, True):
        O = torch.full((B, H, N, d), float("nan"), dtype=o_dt)
        if pinned:
            O = O.pin_memory()
        ctr = torch.zeros(2, dtype=torch.int64, device=dev)
        rows = torch.full((B, H, N), -1, dtype=torch.int32, device=dev)
        status = torch.zeros(1, dtype=torch.int32, device=dev)
        cnt = dict(collapse_ctr=ctr[0:1], collapse_sink_ctr=ctr[1:2], collapse_rows=rows,
                   status_word=status)
        stream = torch.cuda.current_stream()
        if noalloc:
            fp8_attn_fwd_host_noalloc(*host, O, stream=stream, **cnt, **kw)
        else:
            ws = torch.empty(host_workspace_bytes(B=B, H=H, H_kv=Hkv, N=N, d=d,
                                                  o_dtype=kw["o_dtype"], host_chunks=4),
                             dtype=torch.uint8, device=dev)
            fp8_attn_fwd_host(*host, O, plan=plan, workspace=ws, host_chunks=4, stream=stream,
                              **cnt, **kw)
        stream.synchronize()
        assert int(status.item()) == 0, hex(int(status.item()))
        outs.append((O.float().numpy().reshape(-1, d), ctr.cpu().numpy(), rows.cpu().numpy()))
    (O_ref, c_ref, r_ref), (O_na, c_na, r_na) = outs
    assert np.isfinite(O_na).all()
    assert_o_close(O_na, O_ref, "noalloc vs fp8_attn_fwd_host %s" % (case,))
    assert np.array_equal(c_na, c_ref), (c_na, c_ref)
    assert np.array_equal(r_na, r_ref)


@pytest.mark.gpu
def test_noalloc_entry_matches_host_entry_twice():
    """Two calls in a row: a causal GQA problem (BF16 O, pinned memory, every kv
    head of a batch element in one piece), then a larger non-causal one (FP32 O,
    pageable memory) whose kv heads do not fit the array together, so it runs
    as several pieces over the first call's leftovers."""
    from online_softmax_tcgen05_b200 import HostPlan
    plan = HostPlan()
    try:
        _run_pair((2, 6, 3, 700, 128, 1, 256.0, 1, False, True), 71, plan)
        _run_pair((1, 4, 2, 32768, 128, 0, 448.0, 0, True, False), 72, plan)
    finally:
        plan.close()


def test_noalloc_rejects_a_problem_beyond_its_array():
    """One kv head whose staging exceeds the fixed array is refused on the host
    (no device call), with the sizes in the last-error text."""
    from online_softmax_tcgen05_b200 import EINVAL, _binding
    from online_softmax_tcgen05_b200._binding import Params
    lib = _binding.load_library()
    fake = 0x10000   # never dereferenced: the size check fails first
    # N = 131072, d = 128, 4 query heads per kv head, BF16 O: 208 MiB per kv head
    p = Params(Q=fake, K=fake, V=fake, O=fake, B=1, H=8, H_kv=2, N=131072, d=128, causal=1,
               scale=0.088, S=256.0, kv_order=1, n_sink=4)
    st = lib.fp8_attn_fwd_host_noalloc(ctypes.byref(p), None)
    assert st == EINVAL
    msg = _binding.last_error()
    assert "static array" in msg and str(_binding.HOST_NOALLOC_BYTES) in msg, msg
