"""Seeded synthetic inputs for FP8 sink attention.

This module only draws random numbers and builds the attention-sink input
structure; it holds none of the attention arithmetic (no E4M3 cast, no softmax,
no products of Q and K).  Both the GPU path and the CPU oracle consume what it
produces, each casting the FP32 tensors to E4M3 with its own code.

Generator: a counter-based SplitMix64 stream (Steele, Lea and Flood,
"Fast splittable pseudorandom number generators", OOPSLA 2014) keyed by
(seed, stream id), turned into standard normals with the Box-Muller transform
(one pair of uniforms gives the cos and the sin normal of two consecutive
elements).  Element n of a stream depends only on (seed, stream, n), so any
slice can be regenerated without the rest.

Sink construction (the "attention sink" of the P-cast paper, gist.science
arXiv 2606.06521, Problem statement: the first tokens receive a logit gap over
the rest):

* one unit vector u per (batch, kv head), drawn N(0, I_d) and normalised;
* query row i of head h:  q_i = g_i + 8 u   (u of the kv head that h reads);
* key row j >= n_sink:    k_j = z_j - (z_j . u) u   (u projected out);
* key row j <  n_sink:    k_j = z_j + beta u,  beta = Delta * sqrt(d) / 8;
* value rows: N(0, 1).

With softmax scale 1/sqrt(d) the sink logits exceed the non-sink logits by
Delta on average, since (8u).(beta u)/sqrt(d) = Delta.
"""
from __future__ import annotations

import ctypes
import math
import os
import subprocess
from dataclasses import dataclass

import numpy as np

__all__ = ["SinkWorkload", "make_sink_workload", "normals", "uniforms", "splitmix64",
           "ideal_logits", "CONFIG_SEED_BASE"]

# Per-configuration seeds are CONFIG_SEED_BASE + configuration number.
CONFIG_SEED_BASE = 20260608

# stream ids (arbitrary distinct constants)
STREAM_Q, STREAM_K, STREAM_V, STREAM_U, STREAM_LOGIT = 1, 2, 3, 4, 5

_HERE = os.path.dirname(os.path.abspath(__file__))
_SO = os.path.join(_HERE, "_build", "libwlgen.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile gen.c (plain C, OpenMP) into workload/_build/libwlgen.so."""
    src = os.path.join(_HERE, "gen.c")
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < os.path.getmtime(src):
        os.makedirs(os.path.dirname(_SO), exist_ok=True)
        tmp = _SO + ".tmp%d" % os.getpid()
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-ffp-contract=off",
                               src, "-o", tmp, "-lm"])
        os.replace(tmp, _SO)
    return _SO


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        u64 = ctypes.c_uint64
        lib.wl_normals.argtypes = [u64, u64, u64, u64, ctypes.c_void_p]
        lib.wl_uniforms.argtypes = [u64, u64, u64, u64, ctypes.c_void_p]
        lib.wl_splitmix64.argtypes = [u64, u64, ctypes.c_void_p]
        _lib = lib
    return _lib


def splitmix64(state: int, count: int) -> np.ndarray:
    """The first `count` raw SplitMix64 outputs of the generator started at `state`."""
    out = np.empty(count, dtype=np.uint64)
    _load().wl_splitmix64(state, count, out.ctypes.data)
    return out


def uniforms(seed: int, stream: int, start: int, count: int) -> np.ndarray:
    """Uniform doubles in (0, 1] for counters start .. start+count-1 of a stream."""
    out = np.empty(count, dtype=np.float64)
    _load().wl_uniforms(seed, stream, start, count, out.ctypes.data)
    return out


def normals(seed: int, stream: int, start: int, count: int) -> np.ndarray:
    """Standard normals (float32) for elements start .. start+count-1 of a stream.

    Elements 2t and 2t+1 share the uniform pair (counters 2t, 2t+1).
    """
    out = np.empty(count, dtype=np.float32)
    _load().wl_normals(seed, stream, start, count, out.ctypes.data)
    return out


@dataclass
class SinkWorkload:
    """FP32 inputs of one attention problem, layouts [B, H, N, d] / [B, Hkv, N, d]."""
    q: np.ndarray
    k: np.ndarray
    v: np.ndarray
    B: int
    H: int
    Hkv: int
    N: int
    d: int
    n_sink: int
    delta: float
    seed: int

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)


def _unit_vectors(seed: int, B: int, Hkv: int, d: int) -> np.ndarray:
    u = normals(seed, STREAM_U, 0, B * Hkv * d).astype(np.float64).reshape(B, Hkv, d)
    u /= np.linalg.norm(u, axis=-1, keepdims=True)
    return u


def make_sink_workload(B: int, H: int, Hkv: int, N: int, d: int, n_sink: int = 4,
                       delta: float = 8.0, seed: int = CONFIG_SEED_BASE,
                       kv_heads: tuple[int, int] | None = None) -> SinkWorkload:
    """Build Q, K, V (float32) with the sink construction described above.

    The draws do not depend on delta (common random numbers across a sweep):
    delta only sets the length of the u component of the sink keys.
    kv_heads=(g0, g1) builds only kv heads g0..g1-1 and the query heads that
    read them, with exactly the values the full problem has there (every
    element's counter is its index in the full tensor)."""
    assert H % Hkv == 0 and 0 <= n_sink <= N
    group = H // Hkv
    g0, g1 = (0, Hkv) if kv_heads is None else kv_heads
    assert 0 <= g0 < g1 <= Hkv
    nh, nq = g1 - g0, (g1 - g0) * group
    u = _unit_vectors(seed, B, Hkv, d)                        # [B,Hkv,d] f64

    q = np.empty((B, nq, N, d), dtype=np.float32)
    for b in range(B):
        g = normals(seed, STREAM_Q, (b * H + g0 * group) * N * d, nq * N * d).reshape(nq, N, d)
        for j in range(nq):
            q[b, j] = g[j] + (8.0 * u[b, g0 + j // group]).astype(np.float32)
        del g

    k = np.empty((B, nh, N, d), dtype=np.float32)
    beta = delta * math.sqrt(d) / 8.0
    for b in range(B):
        z = normals(seed, STREAM_K, (b * Hkv + g0) * N * d, nh * N * d).reshape(nh, N, d)
        for j in range(nh):
            uu = u[b, g0 + j]
            zz = z[j].astype(np.float64)
            proj = zz @ uu
            kk = zz - proj[:, None] * uu[None, :]
            if n_sink:
                kk[:n_sink] = zz[:n_sink] + beta * uu[None, :]
            k[b, j] = kk.astype(np.float32)
        del z

    v = np.empty((B, nh, N, d), dtype=np.float32)
    for b in range(B):
        v[b] = normals(seed, STREAM_V, (b * Hkv + g0) * N * d, nh * N * d).reshape(nh, N, d)
    return SinkWorkload(q=q, k=k, v=v, B=B, H=nq, Hkv=nh, N=N, d=d, n_sink=n_sink,
                        delta=float(delta), seed=seed)


def ideal_logits(rows: int, N: int, n_sink: int, delta: float, seed: int) -> np.ndarray:
    """Idealised scaled logits [rows, N] (float32): N(0,1) everywhere, +delta on the
    first n_sink keys.  This is the setting of the paper's closed-form
    underflow fraction (Methodology: sink logits delta + N(0,1), non-sink N(0,1))."""
    x = normals(seed, STREAM_LOGIT, 0, rows * N).reshape(rows, N)
    x[:, :n_sink] += np.float32(delta)
    return x
