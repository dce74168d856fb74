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
                       KV_FORWARD, KV_REVERSE, O_BF16, O_F32, OK, QK_BF16, QK_E4M3, Fp8AttnError, device_status_string, fp8_attn_fwd,
                       fp8_attn_fwd_ex, fp8_e4m3_scale_cast, last_error, load_library,
                       status_string)

__all__ = ["attention", "AttentionStats", "fp8_attn_fwd", "fp8_attn_fwd_ex",
           "fp8_e4m3_scale_cast", "load_library", "status_string", "last_error",
           "device_status_string", "Fp8AttnError", "KV_FORWARD", "KV_REVERSE", "O_BF16",
           "O_F32", "OK", "EINVAL", "EUNSUPPORTED", "ECUDA", "ETIMEOUT", "e4m3_cast",
           "DENOM_FP32_P", "DENOM_CAST_P", "QK_E4M3", "QK_BF16"]


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


# Pieces at the start and at the end of the host path that run as one kernel
# per query head.
_SPLIT_FIRST = 1
_SPLIT_LAST = 1


def attention(q, k, v, *, causal: bool = False, scale: float | None = None, S: float = 256.0,
              kv_order: int = KV_REVERSE, n_sink: int = 0, block_n: int = 0,
              denominator: int = DENOM_FP32_P,
              out_dtype=None, count_collapse: bool = False, per_row: bool = False,
              out=None, stream=None, host_chunks: int = 16):
    """FP8 attention forward.  Returns (O, AttentionStats).

    q, k: E4M3 (float8_e4m3fn or uint8 bytes) or both BF16 (the kernel-faithful
    mode: QK^T on BF16 operands, P~ and V in E4M3); v: E4M3.

    Host (CPU) tensors: the work is cut into up to ``host_chunks`` pieces along
    the (batch, kv-head) axis.  The copy of piece g+1 to the device runs on its
    own stream while piece g computes, and piece g's output returns on another.
    Consecutive pieces compute on two alternating streams, so that one piece's
    kernel can fill the SMs that the previous piece's last wave leaves idle.
    Pinned host memory makes the copies asynchronous.  ``stream`` (default: the
    current stream) is ordered before and after the whole call."""
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
    stats = AttentionStats()
    if B * H * N == 0:   # nothing to compute: an empty O (per-row counts empty too)
        import torch
        dev = q.device
        o = out if out is not None else torch.empty((B, H, N, d), dtype=out_dtype, device=dev)
        if count_collapse and per_row:
            stats.collapse_rows = torch.zeros((B, H, N), dtype=torch.int32, device=dev)
        return o, stats
    if q.is_cuda:
        q, k, v = q.contiguous(), k.contiguous(), v.contiguous()
        dev = q.device
        o = out if out is not None else torch.empty((B, H, N, d), dtype=out_dtype, device=dev)
        ctr = torch.zeros(2, dtype=torch.int64, device=dev) if count_collapse else None
        rows = (torch.zeros((B, H, N), dtype=torch.int32, device=dev)
                if (count_collapse and per_row) else None)
        _launch(q, k, v, o, ctr, rows, stream=stream, **kw)
        if ctr is not None:
            c = ctr.cpu()
            stats.collapse, stats.collapse_sink_block = int(c[0]), int(c[1])
            stats.collapse_rows = rows
        return o, stats

    # ---- host tensors: pipelined copies in, compute, copies out ----
    q, k, v = q.contiguous(), k.contiguous(), v.contiguous()
    dev = torch.device("cuda", torch.cuda.current_device())
    group = H // H_kv
    units = [(b, g) for b in range(B) for g in range(H_kv)]       # (batch, kv head)
    nchunk = max(1, min(int(host_chunks), len(units)))
    bounds = [len(units) * i // nchunk for i in range(nchunk + 1)]
    # chunks never cross a batch element, so each piece is one contiguous slice
    pieces = []
    for c in range(nchunk):
        u = bounds[c]
        while u < bounds[c + 1]:
            b = units[u][0]
            e = u
            while e < bounds[c + 1] and units[e][0] == b:
                e += 1
            pieces.append((b, units[u][1], units[e - 1][1] + 1))
            u = e
    max_g = max(g1 - g0 for _, g0, g1 in pieces)
    res = out if out is not None else torch.empty((B, H, N, d), dtype=out_dtype,
                                                  pin_memory=True)
    caller = torch.cuda.current_stream(dev) if stream is None else stream
    pipe = _host_pipeline(dev)
    sets = pipe.staging(max_g * group, max_g, N, d, q.dtype, out_dtype)
    ns = len(sets)
    ctr = torch.zeros(2, dtype=torch.int64, device=dev) if count_collapse else None
    rows = (torch.zeros((B, H, N), dtype=torch.int32, device=dev)
            if (count_collapse and per_row) else None)
    cur = torch.cuda.current_stream(dev)   # the counters were zeroed on it
    pipe.s_in.wait_stream(caller)       # earlier work on the caller's stream comes first
    for sc in pipe.s_comp:
        sc.wait_stream(caller)
        sc.wait_stream(cur)
    step = 0   # sub-steps alternate between the two compute streams
    for i, (b, g0, g1) in enumerate(pieces):
        nq, nk = (g1 - g0) * group, g1 - g0
        qb, kb, vb, ob, ev_free = sets[i % ns]
        qd, kd, vd, od = qb[:, :nq], kb[:, :nk], vb[:, :nk], ob[:, :nq]
        hq = g0 * group
        # The first piece's upload and the last piece's download overlap no
        # compute.  A first or last piece of one kv head therefore runs as one
        # kernel per query head, K and V uploaded once: each head's kernel waits
        # only for its own Q, and each head's O returns as soon as it is done.
        split = (nk == 1 and group > 1 and len(pieces) > 1
                 and (i < _SPLIT_FIRST or i >= len(pieces) - _SPLIT_LAST))
        subs = [(j, j + 1) for j in range(nq)] if split else [(0, nq)]
        with torch.cuda.stream(pipe.s_in):
            if ev_free is not None:
                pipe.s_in.wait_event(ev_free)   # this set's previous chunk has left the device
            kd.copy_(k[b:b + 1, g0:g1], non_blocking=True)
            vd.copy_(v[b:b + 1, g0:g1], non_blocking=True)
            ev_in = []
            for a0, a1 in subs:
                qd[:, a0:a1].copy_(q[b:b + 1, hq + a0:hq + a1], non_blocking=True)
                ev = torch.cuda.Event()
                ev.record(pipe.s_in)
                ev_in.append(ev)
        for (a0, a1), ev in zip(subs, ev_in):
            compute = pipe.s_comp[step % len(pipe.s_comp)]
            step += 1
            compute.wait_event(ev)
            rd = None if rows is None else rows[b:b + 1, hq + a0:hq + a1]
            _launch(qd[:, a0:a1], kd, vd, od[:, a0:a1], ctr, rd, stream=compute, **kw)
            ev_c = torch.cuda.Event()
            ev_c.record(compute)
            pipe.s_out.wait_event(ev_c)
            with torch.cuda.stream(pipe.s_out):
                res[b:b + 1, hq + a0:hq + a1].copy_(od[:, a0:a1], non_blocking=True)
        with torch.cuda.stream(pipe.s_out):
            ev_f = torch.cuda.Event()
            ev_f.record(pipe.s_out)
        sets[i % ns][4] = ev_f
    pipe.s_out.synchronize()
    caller.wait_stream(pipe.s_out)
    for st in sets:
        st[4] = None
    if ctr is not None:
        c = ctr.cpu()
        stats.collapse, stats.collapse_sink_block = int(c[0]), int(c[1])
        stats.collapse_rows = rows
    return res, stats


class _HostPipeline:
    """Per-device copy and compute streams and ``nsets`` sets of device staging
    buffers for the host-tensor path of attention(), kept across calls so that
    the steady state allocates nothing.  A set is reused by the piece ``nsets``
    places later, whose upload therefore waits for this piece's download: with
    two sets each piece would cost a download plus an upload.  Not for
    concurrent use from several host threads."""

    nsets = 3

    def __init__(self, dev):
        import torch
        self.dev = dev
        self.s_in = torch.cuda.Stream(dev)
        self.s_out = torch.cuda.Stream(dev)
        self.s_comp = [torch.cuda.Stream(dev), torch.cuda.Stream(dev)]
        self.key = None
        self.sets = None

    def staging(self, nq, nk, N, d, qk_dtype, o_dtype):
        import torch
        key = (nq, nk, N, d, qk_dtype, o_dtype, self.nsets)
        if self.key != key:
            torch.cuda.current_stream(self.dev).synchronize()
            for st in self.s_comp:
                st.synchronize()
            self.s_out.synchronize()
            mk = lambda h, dt: torch.empty((1, h, N, d), dtype=dt, device=self.dev)
            self.sets = None   # free the old buffers before allocating new ones
            self.sets = [[mk(nq, qk_dtype), mk(nk, qk_dtype), mk(nk, torch.uint8),
                          mk(nq, o_dtype), None] for _ in range(self.nsets)]
            self.key = key
        return self.sets


_pipelines = {}


def _host_pipeline(dev):
    if dev.index not in _pipelines:
        _pipelines[dev.index] = _HostPipeline(dev)
    return _pipelines[dev.index]
