"""Failure detection on the GPU without a fault: every mbarrier wait of the
attention kernel is bounded in time.  The test-only hook debug_skip_kv_step
leaves one K tile unloaded, so the MMA warp's wait for it can only run out;
the kernel must then record where in the status word, free its TMEM and
return, leaving the context usable for the next launch."""
import math

import pytest

from helpers import assert_o_close, gpu_inputs, oracle, workload

pytestmark = pytest.mark.gpu


def test_expired_wait_reports_status_and_context_survives():
    import torch
    from online_softmax_tcgen05_b200 import O_F32, device_status_string, fp8_attn_fwd_ex
    B, H, N, d = 1, 1, 512, 128
    W = workload.make_sink_workload(B, H, H, N, d, 4, 8.0, seed=9)
    ins = gpu_inputs(W)
    (q, Q8), (k, K8), (v, V8) = ins
    O = torch.zeros((B, H, N, d), dtype=torch.float32, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    fp8_attn_fwd_ex(q, k, v, O, B=B, H=H, H_kv=H, N=N, d=d, S=256.0, kv_order=1, n_sink=4,
                    o_dtype=O_F32, status_word=status, timeout_ns=50_000_000,
                    debug_skip_kv_step=2)
    torch.cuda.synchronize()
    word = int(status.item())
    # whichever bounded wait runs out first (the MMA warp's for the K tile, the
    # producer's for the stage that tile's QK^T would free, the softmax warps'
    # for S) records itself; the others then leave on the abort flag
    assert (word & ~0xFF) == 0x100 and (word & 0xFF) != 0, hex(word)
    assert device_status_string(word).startswith("timeout")
    # the same context runs a normal launch correctly afterwards
    status.zero_()
    fp8_attn_fwd_ex(q, k, v, O, B=B, H=H, H_kv=H, N=N, d=d, S=256.0, kv_order=1, n_sink=4,
                    o_dtype=O_F32, status_word=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    Oe, _, _ = oracle.attn_emulate(Q8, K8, V8, B, H, H, N, d, 0, 1 / math.sqrt(d), 256.0, 1, 128, 4)
    assert_o_close(O.cpu().numpy().reshape(-1, d), Oe, "after timeout")


def test_host_entry_reports_expired_wait_and_recovers():
    """The same failure through the host-buffer entry: the call returns, the
    status word (a device word) records the expired wait once the caller's
    stream has passed the call, and the next call on the same plan and
    workspace is correct."""
    import torch
    from online_softmax_tcgen05_b200 import (O_F32, HostPlan, device_status_string,
                                             fp8_attn_fwd_host, host_workspace_bytes)
    B, H, Hkv, N, d = 1, 2, 1, 512, 128
    W = workload.make_sink_workload(B, H, Hkv, N, d, 4, 8.0, seed=10)
    ins = gpu_inputs(W)
    (_, Q8), (_, K8), (_, V8) = ins
    host = [torch.from_numpy(x).pin_memory() for x in (Q8, K8, V8)]
    shape = dict(B=B, H=H, H_kv=Hkv, N=N, d=d)
    plan = HostPlan()
    ws = torch.empty(host_workspace_bytes(o_dtype=O_F32, host_chunks=1, **shape),
                     dtype=torch.uint8, device="cuda")
    O = torch.zeros((B, H, N, d), dtype=torch.float32).pin_memory()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    kw = dict(S=256.0, kv_order=1, n_sink=4, o_dtype=O_F32, status_word=status, **shape)
    fp8_attn_fwd_host(*host, O, plan=plan, workspace=ws, host_chunks=1, timeout_ns=50_000_000,
                      debug_skip_kv_step=2, **kw)
    torch.cuda.synchronize()
    word = int(status.item())
    assert (word & ~0xFF) == 0x100 and (word & 0xFF) != 0, hex(word)
    assert device_status_string(word).startswith("timeout")
    status.zero_()
    fp8_attn_fwd_host(*host, O, plan=plan, workspace=ws, host_chunks=1, **kw)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    Oe, _, _ = oracle.attn_emulate(Q8, K8, V8, B, H, Hkv, N, d, 0, 1 / math.sqrt(d), 256.0, 1, 128,
                                   4)
    assert_o_close(O.numpy().reshape(-1, d), Oe, "host entry after timeout")
    plan.close()


def test_expired_wait_with_two_tile_schedule():
    """The same expired wait under the two-tile schedule, whose softmax warps
    take turns on named barriers: the aborting warps keep taking their turns
    (without touching TMEM), so the launch ends, reports the timeout, and the
    next launch on the same context is correct."""
    import torch
    from online_softmax_tcgen05_b200 import (O_F32, SCHEDULE_ONE_TILE, SCHEDULE_TWO_TILES,
                                             fp8_attn_fwd_ex, set_schedule)
    B, H, N, d = 1, 1, 512, 128
    W = workload.make_sink_workload(B, H, H, N, d, 4, 8.0, seed=9)
    ins = gpu_inputs(W)
    (q, Q8), (k, K8), (v, V8) = ins
    O = torch.zeros((B, H, N, d), dtype=torch.float32, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    try:
        set_schedule(SCHEDULE_TWO_TILES)
        fp8_attn_fwd_ex(q, k, v, O, B=B, H=H, H_kv=H, N=N, d=d, S=256.0, kv_order=1, n_sink=4,
                        o_dtype=O_F32, status_word=status, timeout_ns=50_000_000,
                        debug_skip_kv_step=2)
        torch.cuda.synchronize()
        word = int(status.item())
        assert (word & ~0xFF) == 0x100 and (word & 0xFF) != 0, hex(word)
        status.zero_()
        fp8_attn_fwd_ex(q, k, v, O, B=B, H=H, H_kv=H, N=N, d=d, S=256.0, kv_order=1, n_sink=4,
                        o_dtype=O_F32, status_word=status)
        torch.cuda.synchronize()
        assert int(status.item()) == 0
    finally:
        set_schedule(SCHEDULE_ONE_TILE)
    Oe, _, _ = oracle.attn_emulate(Q8, K8, V8, B, H, H, N, d, 0, 1 / math.sqrt(d), 256.0, 1, 128, 4)
    assert_o_close(O.cpu().numpy().reshape(-1, d), Oe, "two-tile schedule after timeout")
