"""ctypes binding of libfp8attn.so (include/fp8attn.h).

Argument marshalling only: every step of the attention forward and of the
E4M3 cast runs in the library's CUDA kernels.  PyTorch supplies device memory
and the current stream.  There is no CPU fallback: if the library cannot be
built or loaded, every call raises.
"""
from __future__ import annotations

import ctypes
import math

from . import _build

KV_FORWARD, KV_REVERSE = 0, 1
SCHEDULE_ONE_TILE, SCHEDULE_TWO_TILES = 0, 1
O_BF16, O_F32 = 0, 1
DENOM_FP32_P, DENOM_CAST_P = 0, 1
QK_E4M3, QK_BF16 = 0, 1
OK, EINVAL, EUNSUPPORTED, ECUDA, ETIMEOUT = 0, -1, -2, -3, -4


class Fp8AttnError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(message)
        self.status = status


class Params(ctypes.Structure):
    """Mirror of fp8attn_params."""
    _fields_ = [("Q", ctypes.c_void_p), ("K", ctypes.c_void_p), ("V", ctypes.c_void_p),
                ("O", ctypes.c_void_p),
                ("B", ctypes.c_int), ("H", ctypes.c_int), ("H_kv", ctypes.c_int),
                ("N", ctypes.c_int), ("d", ctypes.c_int), ("causal", ctypes.c_int),
                ("scale", ctypes.c_float), ("S", ctypes.c_float),
                ("kv_order", ctypes.c_int), ("n_sink", ctypes.c_int),
                ("o_dtype", ctypes.c_int), ("block_n", ctypes.c_int),
                ("qk_dtype", ctypes.c_int), ("denominator", ctypes.c_int),
                ("collapse_ctr", ctypes.c_void_p), ("collapse_sink_ctr", ctypes.c_void_p),
                ("collapse_rows", ctypes.c_void_p), ("status_word", ctypes.c_void_p),
                ("timeout_ns", ctypes.c_ulonglong), ("debug_skip_kv_step", ctypes.c_int),
                ("q_begin", ctypes.c_int), ("q_end", ctypes.c_int)]


# exported symbol -> (argtypes, restype); every symbol of include/fp8attn.h
SIGNATURES = {
    "fp8_attn_fwd": ([ctypes.c_void_p] * 4 + [ctypes.c_int] * 5 + [ctypes.c_float] * 2
                     + [ctypes.c_int] * 2 + [ctypes.c_void_p, ctypes.c_void_p], ctypes.c_int),
    "fp8_attn_fwd_ex": ([ctypes.POINTER(Params), ctypes.c_void_p], ctypes.c_int),
    "fp8_e4m3_scale_cast": ([ctypes.c_void_p, ctypes.c_void_p, ctypes.c_size_t, ctypes.c_float,
                             ctypes.c_void_p], ctypes.c_int),
    "fp8attn_status_string": ([ctypes.c_int], ctypes.c_char_p),
    "fp8attn_last_error": ([], ctypes.c_char_p),
    "fp8attn_device_status_string": ([ctypes.c_uint], ctypes.c_char_p),
    "fp8attn_version": ([], ctypes.c_int),
    "fp8attn_params_sizeof": ([], ctypes.c_size_t),
    "fp8attn_host_plan_create": ([ctypes.POINTER(ctypes.c_void_p)], ctypes.c_int),
    "fp8attn_host_plan_destroy": ([ctypes.c_void_p], ctypes.c_int),
    "fp8attn_host_workspace_bytes": ([ctypes.POINTER(Params), ctypes.c_int], ctypes.c_size_t),
    "fp8_attn_fwd_host": ([ctypes.POINTER(Params), ctypes.c_void_p, ctypes.c_void_p,
                           ctypes.c_size_t, ctypes.c_int, ctypes.c_void_p], ctypes.c_int),
    "fp8_attn_fwd_host_noalloc": ([ctypes.POINTER(Params), ctypes.c_void_p], ctypes.c_int),
    "fp8attn_set_schedule": ([ctypes.c_int], ctypes.c_int),
}

_lib = None


def load_library(build: bool = True):
    """Load (building first if needed) the sm_100a library; raises if impossible."""
    global _lib
    if _lib is None:
        path = _build.build() if build else _build.LIB_PATH
        lib = ctypes.CDLL(path)
        for name, (argt, rest) in SIGNATURES.items():
            fn = getattr(lib, name)
            fn.argtypes = argt
            fn.restype = rest
        if lib.fp8attn_params_sizeof() != ctypes.sizeof(Params):
            raise RuntimeError("fp8attn_params layout mismatch between binding and library")
        _lib = lib
    return _lib


def status_string(status: int) -> str:
    return load_library().fp8attn_status_string(status).decode()


def last_error() -> str:
    return load_library().fp8attn_last_error().decode()


def device_status_string(word: int) -> str:
    return load_library().fp8attn_device_status_string(word).decode()


def _check(status: int, what: str):
    if status != OK:
        raise Fp8AttnError(status, "%s: %s (%s)" % (what, status_string(status), last_error()))


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def fp8_e4m3_scale_cast(P, out, S: float = 1.0, stream=None):
    """out[i] = E4M3(fl32(S * P[i])) on the device.  P: float32 CUDA tensor,
    out: uint8 (or float8_e4m3fn) CUDA tensor with as many elements."""
    assert P.is_cuda and out.is_cuda and P.numel() == out.numel()
    assert P.is_contiguous() and out.is_contiguous()
    _check(load_library().fp8_e4m3_scale_cast(_ptr(P), _ptr(out), P.numel(), float(S),
                                              _stream(stream)), "fp8_e4m3_scale_cast")
    return out


def fp8_attn_fwd(Q, K, V, O, B, H, N, d, causal, scale, S, kv_order, n_sink, collapse_ctr=None,
                 stream=None):
    """Direct call of the short entry point fp8_attn_fwd (H_kv = H, BF16 O, 128-key
    blocks; all tensors on the device)."""
    _check(load_library().fp8_attn_fwd(_ptr(Q), _ptr(K), _ptr(V), _ptr(O), B, H, N, d,
                                       int(causal), float(scale), float(S), int(kv_order),
                                       int(n_sink), _ptr(collapse_ctr), _stream(stream)),
           "fp8_attn_fwd")


def _params(Q, K, V, O, *, B, H, H_kv, N, d, causal=False, scale=None, S=256.0,
            kv_order=KV_REVERSE, n_sink=0, o_dtype=O_BF16, block_n=0, denominator=0,
            qk_dtype=QK_E4M3, collapse_ctr=None, collapse_sink_ctr=None, collapse_rows=None,
            status_word=None, timeout_ns=0, debug_skip_kv_step=0, q_begin=0, q_end=0):
    return Params(Q=Q.data_ptr(), K=K.data_ptr(), V=V.data_ptr(), O=O.data_ptr(),
                  B=B, H=H, H_kv=H_kv, N=N, d=d, causal=int(causal),
                  scale=float(scale if scale is not None else 1.0 / math.sqrt(d)), S=float(S),
                  kv_order=int(kv_order), n_sink=int(n_sink), o_dtype=int(o_dtype),
                  block_n=int(block_n), denominator=int(denominator), qk_dtype=int(qk_dtype),
                  collapse_ctr=None if collapse_ctr is None else collapse_ctr.data_ptr(),
                  collapse_sink_ctr=(None if collapse_sink_ctr is None
                                     else collapse_sink_ctr.data_ptr()),
                  collapse_rows=None if collapse_rows is None else collapse_rows.data_ptr(),
                  status_word=None if status_word is None else status_word.data_ptr(),
                  timeout_ns=int(timeout_ns), debug_skip_kv_step=int(debug_skip_kv_step),
                  q_begin=int(q_begin), q_end=int(q_end))


def fp8_attn_fwd_ex(Q, K, V, O, *, stream=None, **kw):
    """Full-parameter entry point (all tensors on the device).  Keywords are the
    fields of fp8attn_params (B, H, H_kv, N, d required); ``q_begin``, ``q_end``:
    the query-row range of each (batch, head) plane to compute (0, 0 = all rows)."""
    p = _params(Q, K, V, O, **kw)
    _check(load_library().fp8_attn_fwd_ex(ctypes.byref(p), _stream(stream)), "fp8_attn_fwd_ex")


class HostPlan:
    """The streams and events of the host-buffer pipeline (fp8attn_host_plan),
    created on the current device; reusable across calls, one call at a time."""

    def __init__(self):
        h = ctypes.c_void_p()
        _check(load_library().fp8attn_host_plan_create(ctypes.byref(h)),
               "fp8attn_host_plan_create")
        self._h = h

    @property
    def handle(self):
        return self._h

    def close(self):
        if self._h is not None and self._h.value:
            load_library().fp8attn_host_plan_destroy(self._h)
        self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def host_workspace_bytes(*, B, H, H_kv, N, d, qk_dtype=QK_E4M3, o_dtype=O_BF16,
                         host_chunks=16) -> int:
    """Device workspace bytes that fp8_attn_fwd_host needs for this shape."""
    p = Params(B=B, H=H, H_kv=H_kv, N=N, d=d, qk_dtype=int(qk_dtype), o_dtype=int(o_dtype))
    return int(load_library().fp8attn_host_workspace_bytes(ctypes.byref(p), int(host_chunks)))


def fp8_attn_fwd_host(Q, K, V, O, *, plan, workspace, host_chunks=16, stream=None, **kw):
    """Host-buffer entry point: Q, K, V, O are CPU tensors (pinned for overlap),
    counters and per-row counts CUDA tensors, ``workspace`` a CUDA byte tensor of
    at least host_workspace_bytes(...) bytes.  Ordered after prior work on
    ``stream`` (default: current); synchronise it before reading O."""
    p = _params(Q, K, V, O, **kw)
    nbytes = workspace.numel() * workspace.element_size()
    _check(load_library().fp8_attn_fwd_host(ctypes.byref(p), plan.handle,
                                            ctypes.c_void_p(workspace.data_ptr()), nbytes,
                                            int(host_chunks), _stream(stream)),
           "fp8_attn_fwd_host")


# FP8ATTN_HOST_NOALLOC_BYTES of include/fp8attn.h: the staging array of
# fp8_attn_fwd_host_noalloc
HOST_NOALLOC_BYTES = 64 << 20


def fp8_attn_fwd_host_noalloc(Q, K, V, O, *, stream=None, **kw):
    """Host-buffer entry point that allocates nothing: Q, K, V, O are CPU
    tensors, counters and per-row counts CUDA tensors; staging goes through the
    library's own fixed device array (HOST_NOALLOC_BYTES).  Runs in order on
    ``stream`` (default: current); synchronise it before reading O."""
    p = _params(Q, K, V, O, **kw)
    _check(load_library().fp8_attn_fwd_host_noalloc(ctypes.byref(p), _stream(stream)),
           "fp8_attn_fwd_host_noalloc")


def set_schedule(schedule: int) -> int:
    """Select the kernel schedule (SCHEDULE_ONE_TILE or SCHEDULE_TWO_TILES) for
    later calls, process-wide; returns the previous one."""
    prev = load_library().fp8attn_set_schedule(int(schedule))
    if prev < 0:
        _check(prev, "fp8attn_set_schedule")
    return prev
