"""CPU oracle for FP8 (E4M3) attention with P-cast scale S and KV order.

TEST INFRASTRUCTURE ONLY.  Only tests/, ``__graft_entry__.smoke()`` and
bench.py's CPU-baseline / reference leg may import this package.  It shares no
code with the CUDA path (online_softmax_tcgen05_b200) and never imports it.

Source: "P-Cast Precision in FP8 Attention: Sink-Induced Collapse and the
Optimality of S=2^8" (arXiv 2606.06521), gist.science summaries (pt/de/hi).

* ``oracle.cpp`` (plain C++, OpenMP over rows): the E4M3 codec, float64 exact
  attention, the step-by-step FP8 pipeline emulation and the online softmax on
  given logits.  Built with g++ on first use (``build()``).
* this file: ctypes marshalling plus the paper's closed forms (Methodology:
  F(Delta,S), Delta_c; Optimality of S=256: the quantisation step d_p(S)).

Parity status: every function here is pinned by tests/test_oracle_*.py; see
the pin list in each test module's docstring.
"""
from __future__ import annotations

import ctypes
import math
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SO = os.path.join(_HERE, "_build", "liboracle.so")
_lib = None

LN2 = math.log(2.0)
# E4M3 round-to-zero threshold 2^-10 in natural-log units: 10 ln 2 = 6.9315
# (Methodology: "6.93 ~ 10 ln 2").
ROUND_TO_ZERO_LOG = 10.0 * LN2


def build(force: bool = False) -> str:
    """Compile oracle.cpp into oracle/_build/liboracle.so (g++, -O2, no fast-math,
    no FMA contraction so FP32 expressions round exactly as written)."""
    src = os.path.join(_HERE, "oracle.cpp")
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < os.path.getmtime(src):
        os.makedirs(os.path.dirname(_SO), exist_ok=True)
        tmp = _SO + ".tmp%d" % os.getpid()
        subprocess.check_call(["g++", "-O2", "-std=c++17", "-fopenmp", "-fPIC", "-shared",
                               "-ffp-contract=off", "-fno-fast-math", src, "-o", tmp])
        os.replace(tmp, _SO)
    return _SO


def lib():
    global _lib
    if _lib is None:
        L = ctypes.CDLL(build())
        P = ctypes.c_void_p
        i32, i64, u64, f32, f64 = (ctypes.c_int, ctypes.c_int64, ctypes.c_uint64,
                                   ctypes.c_float, ctypes.c_double)
        L.oracle_e4m3_value.argtypes = [ctypes.c_uint8]
        L.oracle_e4m3_value.restype = f64
        L.oracle_e4m3_encode.argtypes = [f32]
        L.oracle_e4m3_encode.restype = ctypes.c_uint8
        L.oracle_bf16_rne.argtypes = [f32]
        L.oracle_bf16_rne.restype = f32
        L.oracle_e4m3_scale_cast.argtypes = [P, P, i64, f32]
        L.oracle_e4m3_scale_cast_bits.argtypes = [u64, i64, f32, P]
        L.oracle_attn_exact.argtypes = [P, P, P, i32, i32, i32, i32, i32, i32, f64, P, i64, P, i32,
                                        i32]
        L.oracle_attn_exact.restype = i32
        L.oracle_attn_emulate.argtypes = [P, P, P, i32, i32, i32, i32, i32, i32, f32, f32,
                                          i32, i32, i32, i32, P, i64, P, P, P, i32, i32, i32, P]
        L.oracle_attn_emulate.restype = i32
        L.oracle_collapse_logits.argtypes = [P, i64, i32, i32, i32, f32, i32, P, P, i32]
        L.oracle_collapse_logits.restype = i32
        L.oracle_attn_logits.argtypes = [P, P, i64, i32, i32, i32, i32, i32, f32, i32, P, P, P,
                                         i32]
        L.oracle_attn_logits.restype = i32
        _lib = L
    return _lib


def _ptr(a: np.ndarray | None):
    return None if a is None else a.ctypes.data


# ------------------------------------------------------------------ codec ----
def e4m3_table() -> np.ndarray:
    """Decoded value (float64) of each of the 256 E4M3 codes (NaN for 0x7F, 0xFF)."""
    L = lib()
    return np.array([L.oracle_e4m3_value(c) for c in range(256)], dtype=np.float64)


def e4m3_decode(codes: np.ndarray) -> np.ndarray:
    return e4m3_table()[np.asarray(codes, dtype=np.uint8)]


def e4m3_encode(x, S: float = 1.0) -> np.ndarray:
    """E4M3(fl32(S * x)), round to nearest even, saturating to +-448."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    out = np.empty(x.shape, dtype=np.uint8)
    lib().oracle_e4m3_scale_cast(_ptr(x), _ptr(out), x.size, S)
    return out


def e4m3_encode_bits(first: int, n: int, S: float = 1.0) -> np.ndarray:
    """E4M3(fl32(S * x)) for the FP32 bit patterns first .. first+n-1."""
    out = np.empty(n, dtype=np.uint8)
    lib().oracle_e4m3_scale_cast_bits(first, n, S, _ptr(out))
    return out


def bf16_rne(x: np.ndarray) -> np.ndarray:
    L = lib()
    x = np.asarray(x, dtype=np.float32)
    return np.vectorize(lambda v: L.oracle_bf16_rne(float(v)), otypes=[np.float32])(x)


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """BF16 bit patterns (uint16) of x rounded to nearest even (finite x): the
    same rounding as bf16_rne, done on the FP32 bits in bulk."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return u.astype(np.uint16)


# -------------------------------------------------------------- attention ----
def _rows(rows):
    if rows is None:
        return None, 0
    r = np.ascontiguousarray(rows, dtype=np.int64)
    return r, r.size


def _qk_flag(Q, K):
    if Q.dtype == np.uint16 and K.dtype == np.uint16:
        return 1                      # BF16 bit patterns
    assert Q.dtype == np.uint8 and K.dtype == np.uint8
    return 0


def attn_exact(Q8, K8, V8, B, H, Hkv, N, d, causal, scale, rows=None, nthreads=0):
    """float64 O* = softmax(scale Q K^T) V on the decoded inputs, [nrows, d].
    Q, K: E4M3 bytes (uint8) or BF16 bit patterns (uint16); V: E4M3 bytes."""
    r, nr = _rows(rows)
    n_out = nr if r is not None else B * H * N
    O = np.empty((n_out, d), dtype=np.float64)
    rc = lib().oracle_attn_exact(_ptr(Q8), _ptr(K8), _ptr(V8), B, H, Hkv, N, d, int(causal),
                                 float(scale), _ptr(r), nr, _ptr(O), nthreads, _qk_flag(Q8, K8))
    if rc:
        raise ValueError("oracle_attn_exact: bad shape")
    return O


def attn_emulate(Q8, K8, V8, B, H, Hkv, N, d, causal, scale, S, kv_order, block_n, n_sink,
                 o_bf16=False, rows=None, nthreads=0, denom_mode=0, flip_slack=False):
    """FP8 pipeline emulation.  Returns (O [nrows, d] float32, collapse per row
    uint32, totals uint64[2] = {in sink-holding KV blocks, in other blocks}).
    Q, K: E4M3 bytes (uint8) or BF16 bit patterns (uint16, the kernel-faithful
    mode); V: E4M3 bytes.  denom_mode 0: l from the FP32 P, O = acc / (S l); 1: l from the cast values,
    O = acc / l.

    flip_slack=True appends a fourth result, per row: how far O can move if each
    cast whose fl32(S p) lies within a relative 2^-14 of an E4M3 rounding boundary
    went to the neighbouring value (the sum over such casts of the E4M3 step times
    max_k |v_jk|, rescaled like the accumulator, over the denominator; plus
    step * max|O| per cast for the cast-value denominator); 0 for most rows."""
    for a in (Q8, K8, V8):
        assert a.flags.c_contiguous
    assert V8.dtype == np.uint8
    r, nr = _rows(rows)
    n_out = nr if r is not None else B * H * N
    O = np.empty((n_out, d), dtype=np.float32)
    cr = np.zeros(n_out, dtype=np.uint32)
    tot = np.zeros(2, dtype=np.uint64)
    slack = np.zeros(n_out, dtype=np.float32) if flip_slack else None
    rc = lib().oracle_attn_emulate(_ptr(Q8), _ptr(K8), _ptr(V8), B, H, Hkv, N, d, int(causal),
                                   float(scale), float(S), int(kv_order), int(block_n),
                                   int(n_sink), int(bool(o_bf16)), _ptr(r), nr, _ptr(O),
                                   _ptr(cr), _ptr(tot), nthreads, int(denom_mode),
                                   _qk_flag(Q8, K8), _ptr(slack))
    if rc:
        raise ValueError("oracle_attn_emulate: bad shape")
    if flip_slack:
        return O, cr, tot, slack
    return O, cr, tot


def collapse_logits(logits, block_n, n_sink, S, kv_order, nthreads=0):
    """Online softmax + P-cast on given scaled logits [rows, N]; returns
    (collapse per row, totals[2])."""
    x = np.ascontiguousarray(logits, dtype=np.float32)
    rows, N = x.shape
    cr = np.zeros(rows, dtype=np.uint32)
    tot = np.zeros(2, dtype=np.uint64)
    rc = lib().oracle_collapse_logits(_ptr(x), rows, N, int(block_n), int(n_sink), float(S),
                                      int(kv_order), _ptr(cr), _ptr(tot), nthreads)
    if rc:
        raise ValueError("oracle_collapse_logits: bad shape")
    return cr, tot


def attn_logits(logits, V8, rows_per_head, block_n, n_sink, S, kv_order, nthreads=0):
    """The FP8 pipeline on given scaled logits [rows, N] with E4M3 values
    V8 [heads, N, d] (row r reads head r // rows_per_head), non-causal.  Returns
    (O_emu [rows, d] float32, O_exact [rows, d] float64, collapse per row)."""
    x = np.ascontiguousarray(logits, dtype=np.float32)
    V8 = np.ascontiguousarray(V8, dtype=np.uint8)
    rows, N = x.shape
    heads, Nv, d = V8.shape
    assert Nv == N and heads * rows_per_head >= rows
    Oe = np.empty((rows, d), dtype=np.float32)
    Ox = np.empty((rows, d), dtype=np.float64)
    cr = np.zeros(rows, dtype=np.uint32)
    rc = lib().oracle_attn_logits(_ptr(x), _ptr(V8), rows, int(rows_per_head), N, d,
                                  int(block_n), int(n_sink), float(S), int(kv_order), _ptr(Oe),
                                  _ptr(Ox), _ptr(cr), nthreads)
    if rc:
        raise ValueError("oracle_attn_logits: bad shape")
    return Oe, Ox, cr


def collapse_denominator(B, H, N, n_sink, causal):
    """Number of unmasked (query, non-sink key) pairs, the denominator of the
    collapse fraction."""
    if causal:
        m = N - n_sink
        return B * H * m * (m + 1) // 2
    return B * H * N * (N - n_sink)


# ------------------------------------------------------------ closed forms ----
def std_normal_cdf(x: float) -> float:
    return 0.5 * math.erfc(-x / math.sqrt(2.0))


def _max_normal_density_grid(k: int, lo=-10.0, hi=10.0, n=200001):
    x = np.linspace(lo, hi, n)
    phi = np.exp(-0.5 * x * x) / math.sqrt(2 * math.pi)
    cdf = 0.5 * np.vectorize(math.erfc)(-x / math.sqrt(2.0))
    return x, k * phi * cdf ** (k - 1)


def expected_max_normal(k: int) -> float:
    """delta_k = E[max of k iid N(0,1)] (Methodology: ~1.0 for k = 4)."""
    x, f = _max_normal_density_grid(k)
    return float(np.trapezoid(x * f, x))


def underflow_fraction_closed(delta: float, S: float, k: int = 4) -> float:
    """The paper's closed form F(Delta,S) = Phi(Delta + delta_k - 10 ln 2 - ln S)
    (Methodology, theoretical framework)."""
    return std_normal_cdf(delta + expected_max_normal(k) - ROUND_TO_ZERO_LOG - math.log(S))


def underflow_fraction_expected(delta: float, S: float, k: int = 4) -> float:
    """E_M[Phi(Delta + M - 10 ln 2 - ln S)], M the max of k standard normals: the
    same underflow condition averaged over the sink maximum instead of taking
    its mean inside Phi."""
    x, f = _max_normal_density_grid(k)
    c = delta - ROUND_TO_ZERO_LOG - math.log(S)
    Phi = 0.5 * np.vectorize(math.erfc)(-(x + c) / math.sqrt(2.0))
    return float(np.trapezoid(Phi * f, x))


def delta_c(S: float, k: int = 4) -> float:
    """Collapse threshold Delta_c = 10 ln 2 + ln S - delta_k (Contributions 1)."""
    return ROUND_TO_ZERO_LOG + math.log(S) - expected_max_normal(k)


def dp(S: float) -> float:
    """Normalised maximum quantisation step d_p(S): the largest gap between
    adjacent finite E4M3 values below S, divided by S (Optimality of S=256,
    condition 2; the reading is stated with the tests)."""
    t = e4m3_table()
    vals = np.unique(t[np.isfinite(t) & (t >= 0)])
    gaps = np.diff(vals)
    lower = vals[:-1]
    sel = lower < S
    return float(gaps[sel].max() / S)


def expected_max_normal_gt(N: int, c: float) -> float:
    """E[Phi(M_N - c)] for M_N the max of N iid N(0,1): the probability that one
    more standard normal lies more than c below the running max of N of them."""
    x = np.linspace(-8.0, 12.0, 400001)
    logcdf = np.log(np.maximum(0.5 * np.vectorize(math.erfc)(-x / math.sqrt(2.0)), 1e-300))
    logphi = -0.5 * x * x - 0.5 * math.log(2 * math.pi)
    dens = np.exp(math.log(N) + logphi + (N - 1) * logcdf)
    Phi = 0.5 * np.vectorize(math.erfc)(-(x - c) / math.sqrt(2.0))
    return float(np.trapezoid(Phi * dens, x))


def reverse_underflow_prob(N: int, S: float) -> float:
    """Reverse KV order: every non-sink P is cast against a running max made of
    non-sink logits only.  Probability that one non-sink entry underflows,
    Phi(M_N - 10 ln 2 - ln S) averaged over the pre-sink max M_N of N standard
    normal logits (Optimisation 1)."""
    return expected_max_normal_gt(N, ROUND_TO_ZERO_LOG + math.log(S))
