"""B200 (sm_100a) FP8 attention forward with P-cast scale S and KV-block order.

The hot path lives in the CUDA library libfp8attn.so (C ABI:
include/fp8attn.h); this package only marshals arguments to it.

    from online_softmax_tcgen05_b200 import attention
    O, stats = attention(q8, k8, v8, causal=True, S=256.0, kv_order=KV_REVERSE,
                         n_sink=4, count_collapse=True)

``attention`` takes E4M3 tensors (torch.float8_e4m3fn or uint8 bytes) laid out
[B, H, N, d] (K, V: [B, H_kv, N, d]).  Tensors on the GPU are used in place;
tensors in host memory are copied to the current device, the kernel runs, and
the output is copied back (the end-to-end path).
"""
from __future__ import annotations

import math
from dataclasses import dataclass

from ._binding import (DENOM_CAST_P, DENOM_FP32_P, ECUDA, EINVAL, ETIMEOUT, EUNSUPPORTED,
                       KV_FORWARD, KV_REVERSE, O_BF16, O_F32, OK, QK_BF16, QK_E4M3,
                       SCHEDULE_ONE_TILE, SCHEDULE_TWO_TILES, Fp8AttnError, set_schedule,
                       HostPlan, device_status_string, fp8_attn_fwd, fp8_attn_fwd_ex,
                       fp8_attn_fwd_host, fp8_attn_fwd_host_noalloc, fp8_e4m3_scale_cast,
                       host_workspace_bytes, last_error, load_library, status_string)

__all__ = ["attention", "AttentionStats", "fp8_attn_fwd", "fp8_attn_fwd_ex",
           "fp8_attn_fwd_host", "fp8_attn_fwd_host_noalloc", "HostPlan", "host_workspace_bytes",
           "fp8_e4m3_scale_cast", "load_library", "status_string", "last_error",
           "device_status_string", "Fp8AttnError", "KV_FORWARD", "KV_REVERSE", "O_BF16",
           "O_F32", "OK", "EINVAL", "EUNSUPPORTED", "ECUDA", "ETIMEOUT", "e4m3_cast",
           "DENOM_FP32_P", "DENOM_CAST_P", "QK_E4M3", "QK_BF16", "set_schedule",
           "SCHEDULE_ONE_TILE", "SCHEDULE_TWO_TILES"]


@dataclass
class AttentionStats:
    collapse: int = 0          # collapsed non-sink entries (all KV blocks)
    collapse_sink_block: int = 0   # of which in KV blocks holding a sink key
    collapse_rows: object = None   # per-row counts [B, H, N] (torch.int32) or None


def _as_bytes(t, allow_bf16=False):
    import torch
    if t.dtype == torch.float8_e4m3fn:
        return t.view(torch.uint8)
    if allow_bf16 and t.dtype == torch.bfloat16:
        return t
    if t.dtype != torch.uint8:
        raise TypeError("inputs must be E4M3 (torch.float8_e4m3fn or uint8 bytes)%s, got %s"
                        % (" or BF16 (q, k)" if allow_bf16 else "", t.dtype))
    return t


def e4m3_cast(x, S: float = 1.0):
    """E4M3 bytes of fl32(S * x) computed on the GPU (x: float32 CUDA tensor)."""
    import torch
    out = torch.empty(x.shape, dtype=torch.uint8, device=x.device)
    fp8_e4m3_scale_cast(x.contiguous(), out, S)
    return out


def _launch(q, k, v, o, ctr, rows, *, causal, scale, S, kv_order, n_sink, block_n,
            denominator, o_code, stream):
    import torch
    B, H, N, d = q.shape
    fp8_attn_fwd_ex(q, k, v, o, B=B, H=H, H_kv=k.shape[1], N=N, d=d, causal=causal,
                    scale=scale, S=S, kv_order=kv_order, n_sink=n_sink, o_dtype=o_code,
                    block_n=block_n, denominator=denominator,
                    qk_dtype=QK_BF16 if q.dtype == torch.bfloat16 else QK_E4M3,
                    collapse_ctr=None if ctr is None else ctr[0:1],
                    collapse_sink_ctr=None if ctr is None else ctr[1:2],
                    collapse_rows=rows, stream=stream)


def attention(q, k, v, *, causal: bool = False, scale: float | None = None, S: float = 256.0,
              kv_order: int = KV_REVERSE, n_sink: int = 0, block_n: int = 0,
              denominator: int = DENOM_FP32_P,
              out_dtype=None, count_collapse: bool = False, per_row: bool = False,
              out=None, stream=None, host_chunks: int = 16):
    """FP8 attention forward.  Returns (O, AttentionStats).

    q, k: E4M3 (float8_e4m3fn or uint8 bytes) or both BF16 (the kernel-faithful
    mode: QK^T on BF16 operands, P~ and V in E4M3); v: E4M3.

    Host (CPU) tensors: one call of the library's host-buffer entry point
    (fp8_attn_fwd_host), which cuts the work into up to ``host_chunks`` pieces
    along the (batch, kv-head) axis and pipelines, on its own streams, each
    piece's upload, kernels and download against its neighbours'.  Pinned host
    memory makes the copies asynchronous.  ``stream`` (default: the current
    stream) is ordered before and after the whole call, which returns once O is
    in host memory.

    CUDA tensors: q, k, v (and ``out``) must share one device; the kernel runs
    there on ``stream`` (default: that device's current stream), ordered after
    the device's current stream, which in turn waits for the kernel."""
    import torch
    q, k, v = _as_bytes(q, True), _as_bytes(k, True), _as_bytes(v)
    if (q.dtype == torch.bfloat16) != (k.dtype == torch.bfloat16):
        raise TypeError("q and k must both be E4M3 or both be BF16")
    if q.dim() != 4 or k.dim() != 4 or v.dim() != 4:
        raise ValueError("q, k, v must be [B, H, N, d]")
    B, H, N, d = q.shape
    H_kv = k.shape[1]
    if k.shape != (B, H_kv, N, d) or v.shape != k.shape:
        raise ValueError("k and v must be [B, H_kv, N, d] matching q")
    out_dtype = torch.bfloat16 if out_dtype is None else out_dtype
    o_code = {torch.bfloat16: O_BF16, torch.float32: O_F32}[out_dtype]
    scale = scale if scale is not None else 1.0 / math.sqrt(d)
    kw = dict(causal=causal, scale=scale, S=S, kv_order=kv_order, n_sink=n_sink,
              block_n=block_n, denominator=denominator, o_code=o_code)
    if out is not None:
        if (tuple(out.shape) != (B, H, N, d) or out.dtype != out_dtype
                or not out.is_contiguous()
                or (out.device != q.device if q.is_cuda else out.device.type != "cpu")):
            raise ValueError("out must be a contiguous %s tensor of shape %s on %s"
                             % (out_dtype, (B, H, N, d), q.device))
    if q.is_cuda or k.is_cuda or v.is_cuda:
        devs = {t.device for t in (q, k, v)}
        if out is not None:
            devs.add(out.device)
        if len(devs) != 1 or q.device.type != "cuda":
            raise ValueError("q, k, v (and out) must all be on one CUDA device, got %s"
                             % sorted(str(x) for x in devs))
        if stream is not None and stream.device != q.device:
            raise ValueError("stream is on %s, the tensors on %s" % (stream.device, q.device))
    stats = AttentionStats()
    if B * H * N == 0:   # nothing to compute: an empty O (per-row counts empty too)
        import torch
        dev = q.device
        o = out if out is not None else torch.empty((B, H, N, d), dtype=out_dtype, device=dev)
        if count_collapse and per_row:
            stats.collapse_rows = torch.zeros((B, H, N), dtype=torch.int32, device=dev)
        return o, stats
    if q.is_cuda:
        # The library launches on the current device and on `s`; the tensors made
        # here come from the caching allocator on the current stream `cur`.
        dev = q.device
        with torch.cuda.device(dev):
            cur = torch.cuda.current_stream(dev)
            s = cur if stream is None else stream
            q, k, v = q.contiguous(), k.contiguous(), v.contiguous()
            o = out if out is not None else torch.empty((B, H, N, d), dtype=out_dtype,
                                                        device=dev)
            ctr = torch.zeros(2, dtype=torch.int64, device=dev) if count_collapse else None
            rows = (torch.zeros((B, H, N), dtype=torch.int32, device=dev)
                    if (count_collapse and per_row) else None)
            if s is not cur:
                s.wait_stream(cur)   # the copies and zeroed counters above, on cur
            _launch(q, k, v, o, ctr, rows, stream=s, **kw)
            if s is not cur:
                for t in (q, k, v, o, ctr, rows):
                    if t is not None:
                        t.record_stream(s)
                cur.wait_stream(s)   # the counters are read on cur below
            if ctr is not None:
                c = ctr.cpu()
                stats.collapse, stats.collapse_sink_block = int(c[0]), int(c[1])
                stats.collapse_rows = rows
        return o, stats

    # ---- host tensors: the library's host-buffer pipeline (fp8_attn_fwd_host) ----
    q, k, v = q.contiguous(), k.contiguous(), v.contiguous()
    dev = torch.device("cuda", torch.cuda.current_device())
    res = out if out is not None else torch.empty((B, H, N, d), dtype=out_dtype,
                                                  pin_memory=True)
    cur = torch.cuda.current_stream(dev)
    caller = cur if stream is None else stream
    pipe = _host_pipeline(dev)
    qk_code = QK_BF16 if q.dtype == torch.bfloat16 else QK_E4M3
    chunks = max(1, int(host_chunks))
    ws = pipe.workspace(host_workspace_bytes(B=B, H=H, H_kv=H_kv, N=N, d=d, qk_dtype=qk_code,
                                             o_dtype=o_code, host_chunks=chunks))
    ctr = torch.zeros(2, dtype=torch.int64, device=dev) if count_collapse else None
    rows = (torch.zeros((B, H, N), dtype=torch.int32, device=dev)
            if (count_collapse and per_row) else None)
    if caller is not cur:
        caller.wait_stream(cur)   # the counters were zeroed on the current stream
    fp8_attn_fwd_host(q, k, v, res, plan=pipe.plan, workspace=ws, host_chunks=chunks,
                      stream=caller, B=B, H=H, H_kv=H_kv, N=N, d=d, causal=causal, scale=scale,
                      S=S, kv_order=kv_order, n_sink=n_sink, o_dtype=o_code, block_n=block_n,
                      denominator=denominator, qk_dtype=qk_code,
                      collapse_ctr=None if ctr is None else ctr[0:1],
                      collapse_sink_ctr=None if ctr is None else ctr[1:2], collapse_rows=rows)
    caller.synchronize()
    if ctr is not None:
        c = ctr.cpu()
        stats.collapse, stats.collapse_sink_block = int(c[0]), int(c[1])
        stats.collapse_rows = rows
    return res, stats


class _HostPipeline:
    """Per-device state of the host-tensor path of attention(), kept across calls
    so that the steady state creates and allocates nothing: the library's host
    plan (its copy and compute streams and events) and the device workspace that
    holds its staging buffers.  Not for concurrent use from several host threads."""

    def __init__(self, dev):
        import torch
        self.dev = dev
        with torch.cuda.device(dev):
            self.plan = HostPlan()
        self.ws = None

    def workspace(self, nbytes):
        import torch
        if self.ws is None or self.ws.numel() < nbytes:
            self.ws = None   # free the old buffer before allocating the new one
            self.ws = torch.empty(max(int(nbytes), 1), dtype=torch.uint8, device=self.dev)
        return self.ws


_pipelines = {}


def _host_pipeline(dev):
    if dev.index not in _pipelines:
        _pipelines[dev.index] = _HostPipeline(dev)
    return _pipelines[dev.index]
