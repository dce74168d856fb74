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
                       KV_FORWARD, KV_REVERSE, O_BF16, O_F32, OK, Fp8AttnError, device_status_string, fp8_attn_fwd,
                       fp8_attn_fwd_ex, fp8_e4m3_scale_cast, last_error, load_library,
                       status_string)

__all__ = ["attention", "AttentionStats", "fp8_attn_fwd", "fp8_attn_fwd_ex",
           "fp8_e4m3_scale_cast", "load_library", "status_string", "last_error",
           "device_status_string", "Fp8AttnError", "KV_FORWARD", "KV_REVERSE", "O_BF16",
           "O_F32", "OK", "EINVAL", "EUNSUPPORTED", "ECUDA", "ETIMEOUT", "e4m3_cast",
           "DENOM_FP32_P", "DENOM_CAST_P"]


@dataclass
class AttentionStats:
    collapse: int = 0          # collapsed non-sink entries (all KV blocks)
    collapse_sink_block: int = 0   # of which in KV blocks holding a sink key
    collapse_rows: object = None   # per-row counts [B, H, N] (torch.int32) or None


def _as_bytes(t):
    import torch
    if t.dtype == torch.float8_e4m3fn:
        return t.view(torch.uint8)
    if t.dtype != torch.uint8:
        raise TypeError("E4M3 inputs must be torch.float8_e4m3fn or uint8, got %s" % t.dtype)
    return t


def e4m3_cast(x, S: float = 1.0):
    """E4M3 bytes of fl32(S * x) computed on the GPU (x: float32 CUDA tensor)."""
    import torch
    out = torch.empty(x.shape, dtype=torch.uint8, device=x.device)
    fp8_e4m3_scale_cast(x.contiguous(), out, S)
    return out


def attention(q, k, v, *, causal: bool = False, scale: float | None = None, S: float = 256.0,
              kv_order: int = KV_REVERSE, n_sink: int = 0, block_n: int = 0,
              denominator: int = DENOM_FP32_P,
              out_dtype=None, count_collapse: bool = False, per_row: bool = False,
              out=None, stream=None):
    """FP8 attention forward.  Returns (O, AttentionStats)."""
    import torch
    q, k, v = _as_bytes(q), _as_bytes(k), _as_bytes(v)
    if q.dim() != 4 or k.dim() != 4 or v.dim() != 4:
        raise ValueError("q, k, v must be [B, H, N, d]")
    B, H, N, d = q.shape
    H_kv = k.shape[1]
    if k.shape != (B, H_kv, N, d) or v.shape != k.shape:
        raise ValueError("k and v must be [B, H_kv, N, d] matching q")
    out_dtype = torch.bfloat16 if out_dtype is None else out_dtype
    o_code = {torch.bfloat16: O_BF16, torch.float32: O_F32}[out_dtype]
    host = not q.is_cuda
    dev = torch.device("cuda", torch.cuda.current_device()) if host else q.device
    if host:
        q, k, v = (t.to(dev, non_blocking=True) for t in (q, k, v))
    q, k, v = q.contiguous(), k.contiguous(), v.contiguous()
    o = out if (out is not None and not host) else torch.empty((B, H, N, d), dtype=out_dtype,
                                                               device=dev)
    ctr = torch.zeros(2, dtype=torch.int64, device=dev) if count_collapse else None
    rows = (torch.zeros((B, H, N), dtype=torch.int32, device=dev)
            if (count_collapse and per_row) else None)
    fp8_attn_fwd_ex(q, k, v, o, B=B, H=H, H_kv=H_kv, N=N, d=d, causal=causal,
                    scale=scale if scale is not None else 1.0 / math.sqrt(d), S=S,
                    kv_order=kv_order, n_sink=n_sink, o_dtype=o_code, block_n=block_n,
                    denominator=denominator,
                    collapse_ctr=None if ctr is None else ctr[0:1],
                    collapse_sink_ctr=None if ctr is None else ctr[1:2],
                    collapse_rows=rows, stream=stream)
    stats = AttentionStats()
    if host:
        res = out if out is not None else torch.empty((B, H, N, d), dtype=out_dtype,
                                                      pin_memory=True)
        res.copy_(o, non_blocking=True)
        o = res
    if ctr is not None:
        c = ctr.cpu()
        stats.collapse, stats.collapse_sink_block = int(c[0]), int(c[1])
        stats.collapse_rows = rows
    elif host:
        torch.cuda.current_stream().synchronize()
    return o, stats
