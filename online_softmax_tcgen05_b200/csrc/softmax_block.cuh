// softmax_block.cuh - the per-row arithmetic of one online-softmax block and the
// per-row TMEM and shared-memory steps around it, shared by the one-tile kernel
// (fp8_attn_fwd.cu) and the two-tile kernel (fp8_attn_fwd_pair.cu).  Each thread
// of a softmax warp owns one query row; every function here works on that row's
// share of one KV block held in registers (the arrays are indexed by constants
// after unrolling, so they never leave the register file).
//
// Method: "P-Cast Precision in FP8 Attention: Sink-Induced Collapse and the
// Optimality of S=2^8" (arXiv 2606.06521, gist.science summary), section 1
// (Problem statement): exponentials against the running max, the FP32 row sum,
// the product S*p cast to E4M3, the collapse count of section 1 and the
// epilogue O / (S l).
#pragma once
#include <cuda_runtime.h>

#include <cstdint>

#include "exp2_poly.cuh"
#include "fp8attn.h"
#include "sm100.cuh"

namespace fp8attn {

// Of every 8 pairs of keys in a row of a plain block (no masked key), this many
// take 2^x on the FMA pipe (exp2_poly.cuh) and the rest on MUFU ex2: the two
// units then share the exponentials of the softmax.  Both kernel schedules use
// the same split, so that they compute the same values.
#ifndef FP8ATTN_POLY_OF_8
#define FP8ATTN_POLY_OF_8 2
#endif
constexpr int POLY_OF_8 = FP8ATTN_POLY_OF_8;

template <bool B>
struct BoolTag {
  static constexpr bool value = B;
};

// l <- alpha * l + x as the method's two FP32 operations, each rounded to nearest.
// Explicit roundings keep the code generator from fusing them into one FMA in some
// kernel variants and not in others, so every variant forms the same l (the
// oracle's order of operations).
__device__ __forceinline__ float scale_add(float alpha, float l, float x) {
  return __fadd_rn(__fmul_rn(alpha, l), x);
}

// KV block visited at step t of T (forward 0..T-1, reverse T-1..0)
__device__ __forceinline__ int kv_block_at(int t, int T, int order) {
  return order == FP8ATTN_KV_FORWARD ? t : T - 1 - t;
}

// Scores of the keys after the row's last visible key `lim` become -inf.
template <int BN>
__device__ __forceinline__ void mask_scores(float* s, int j0, int lim) {
#pragma unroll
  for (int j = 0; j < BN; ++j)
    if (j0 + j > lim) s[j] = -INFINITY;
}

// s[2q], s[2q+1] <- 2^(s * c + nm) for key pair q, in place (c2 = (c, c),
// nm2 = (nm, nm)), added to the packed partial row sum acc8[q & 7].  The argument
// is one packed FFMA2; the exponential is MUFU ex2, except for the first POLY of
// every 8 pairs, which take the FMA-pipe 2^x of exp2_poly.cuh (finite arguments
// only: -inf, a masked key, needs the MUFU path; sc23 = 2^23 as a run-time value).
template <int POLY>
__device__ __forceinline__ void exp_pair(float* s, int q, float2 c2, float2 nm2, uint32_t sc23,
                                         float2* acc8) {
  const float2 y = __ffma2_rn(make_float2(s[2 * q], s[2 * q + 1]), c2, nm2);
  if ((q & 7) < POLY) {
    const float2 e = exp2_poly2(y, sc23);
    s[2 * q] = e.x;
    s[2 * q + 1] = e.y;
  } else {
    s[2 * q] = ex2_approx(y.x);
    s[2 * q + 1] = ex2_approx(y.y);
  }
  acc8[q & 7] = __fadd2_rn(acc8[q & 7], make_float2(s[2 * q], s[2 * q + 1]));
}

// The row sum from the 8 packed partial sums, by a fixed tree.
__device__ __forceinline__ float rowsum_tree(float2* acc8) {
#pragma unroll
  for (int w = 4; w >= 1; w >>= 1)
#pragma unroll
    for (int i = 0; i < w; ++i) acc8[i] = __fadd2_rn(acc8[i], acc8[i + w]);
  return __fadd_rn(acc8[0].x, acc8[0].y);
}

// E4M3 word q of a row whose s already holds S*p: keys 4q..4q+3 in bytes 0..3.
__device__ __forceinline__ uint32_t pack_word(const float* s, int q) {
  return pack_e4m3x4(s[4 * q], s[4 * q + 1], s[4 * q + 2], s[4 * q + 3]);
}

// acc + 128 x (the number of nonzero bytes of the E4M3 word w).  P~ is never
// negative, so every byte is 0x00..0x7F (a NaN casts to 0x7F): w + 0x7F7F7F7F
// then carries into no neighbour and sets bit 7 of exactly the nonzero bytes;
// dp4a sums those flags.
__device__ __forceinline__ uint32_t add_nonzero_bytes(uint32_t w, uint32_t acc) {
  return __dp4a((w + 0x7F7F7F7Fu) & 0x80808080u, 0x01010101u, acc);
}

// s[j] <- 2^(s[j] * c + nm) for the row's BN keys in place (exp_pair); returns the
// FP32 row sum.  SPLIT issues every exponential before the first sum (MUFU only).
template <int BN, int POLY, bool SPLIT>
__device__ __forceinline__ float exp2_rowsum(float* s, float2 c2, float2 nm2, uint32_t sc23) {
  float2 acc8[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) acc8[i] = make_float2(0.f, 0.f);
  if constexpr (SPLIT) {
#pragma unroll
    for (int q = 0; q < BN / 2; ++q) {
      const float2 y = __ffma2_rn(make_float2(s[2 * q], s[2 * q + 1]), c2, nm2);
      s[2 * q] = ex2_approx(y.x);
      s[2 * q + 1] = ex2_approx(y.y);
    }
#pragma unroll
    for (int q = 0; q < BN / 2; ++q)
      acc8[q & 7] = __fadd2_rn(acc8[q & 7], make_float2(s[2 * q], s[2 * q + 1]));
  } else {
#pragma unroll
    for (int q = 0; q < BN / 2; ++q) exp_pair<POLY>(s, q, c2, nm2, sc23, acc8);
  }
  return rowsum_tree(acc8);
}

// A block with no masked key and no sink key, S = 2^k, counter on: the
// exponentials, the E4M3 cast and the zero-byte count of the row as one loop over
// groups of 16 keys, the cast and count of group g - 1 following the exponentials
// of group g.  The same operations, and the same order of every sum, as
// exp2_rowsum, cast_e4m3<BN, false> and zero_bytes_all; the interleaving only
// hands the code generator the cast and count work next to the exponentials it
// can overlap (timed 0.7-1.0% faster with the counter on).  Returns the row sum;
// *zeros gets the block's zero-byte count.
template <int BN, int POLY>
__device__ __forceinline__ float exp_cast_count_plain(float* s, float2 c2, float2 nm2,
                                                      uint32_t sc23, uint32_t* pw,
                                                      uint32_t* zeros) {
  float2 acc8[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) acc8[i] = make_float2(0.f, 0.f);
  uint32_t nz4[4] = {0, 0, 0, 0};
#pragma unroll
  for (int g = 0; g <= BN / 16; ++g) {
    if (g < BN / 16) {
#pragma unroll
      for (int q = 8 * g; q < 8 * g + 8; ++q) exp_pair<POLY>(s, q, c2, nm2, sc23, acc8);
    }
    if (g > 0) {
#pragma unroll
      for (int q = 4 * (g - 1); q < 4 * g; ++q) {
        pw[q] = pack_word(s, q);
        nz4[q & 3] = add_nonzero_bytes(pw[q], nz4[q & 3]);
      }
    }
  }
  *zeros = BN - (((nz4[0] + nz4[1]) + (nz4[2] + nz4[3])) >> 7);
  return rowsum_tree(acc8);
}

// The E4M3 cast of S*p, four keys per word (key 4q + k in byte k of pw[q]).
// SCALED = false: s already holds S*p (S = 2^k taken in the exponent).
// SCALED = true: the cast is of fl(s_mul * s), the method's FP32 product S*p when
// S is not a power of two, and an exact multiply by 1 otherwise.
template <int BN, bool SCALED>
__device__ __forceinline__ void cast_e4m3(const float* s, float s_mul, uint32_t* pw) {
  const float2 sm2 = make_float2(s_mul, s_mul);
#pragma unroll
  for (int q = 0; q < BN / 4; ++q) {
    if constexpr (!SCALED) {
      pw[q] = pack_word(s, q);
    } else {
      const float2 a = __fmul2_rn(make_float2(s[4 * q], s[4 * q + 1]), sm2);
      const float2 b = __fmul2_rn(make_float2(s[4 * q + 2], s[4 * q + 3]), sm2);
      pw[q] = pack_e4m3x4(a.x, a.y, b.x, b.y);
    }
  }
}

// Row sum of the cast values (the cast-value denominator).  An E4M3 magnitude's
// 7 bits placed at FP32 bit 20 form a float exactly 2^-120 times the E4M3 value
// (subnormals included, as FP32 subnormals); the partial sums of those are scaled
// back by 2^120 (exact).
template <int BN>
__device__ __forceinline__ float cast_value_sum(const uint32_t* pw) {
  float2 d4[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) d4[i] = make_float2(0.f, 0.f);
#pragma unroll
  for (int q = 0; q < BN / 4; ++q) {
    const uint32_t w = pw[q];
    const float2 lo = make_float2(__uint_as_float((w & 0x7Fu) << 20),
                                  __uint_as_float((w & 0x7F00u) << 12));
    const float2 hi = make_float2(__uint_as_float((w & 0x7F0000u) << 4),
                                  __uint_as_float((w & 0x7F000000u) >> 4));
    d4[q & 3] = __fadd2_rn(d4[q & 3], __fadd2_rn(lo, hi));
  }
  d4[0] = __fadd2_rn(__fadd2_rn(d4[0], d4[1]), __fadd2_rn(d4[2], d4[3]));
  return __fmul_rn(__fadd_rn(d4[0].x, d4[0].y), 0x1p120f);
}

// Collapse count of a block whose keys all count (no sink key, no masked key):
// the number of zero E4M3 bytes (add_nonzero_bytes over the row's words).
template <int BN>
__device__ __forceinline__ uint32_t zero_bytes_all(const uint32_t* pw) {
  uint32_t nz4[4] = {0, 0, 0, 0};
#pragma unroll
  for (int q = 0; q < BN / 4; ++q) nz4[q & 3] = add_nonzero_bytes(pw[q], nz4[q & 3]);
  return BN - (((nz4[0] + nz4[1]) + (nz4[2] + nz4[3])) >> 7);
}

// Collapse count of a block holding a sink key or a masked key: zero bytes among
// the block-local keys lo..hi only (lo = first non-sink key, hi = last visible).
template <int BN>
__device__ __forceinline__ uint32_t zero_bytes_range(const uint32_t* pw, int lo, int hi) {
  uint32_t zacc = 0;
#pragma unroll
  for (int q = 0; q < BN / 4; ++q) {
    const uint32_t w = pw[q];
    const uint32_t y = ~(((w & 0x7F7F7F7Fu) + 0x7F7F7F7Fu) | w | 0x7F7F7F7Fu);
    const int a = lo - 4 * q, bq = hi - 4 * q;   // bytes a..bq of this word count
    const uint32_t mlo = a <= 0 ? 0x80808080u : (a >= 4 ? 0u : 0x80808080u << (8 * a));
    const uint32_t mhi = bq >= 3 ? 0x80808080u : (bq < 0 ? 0u : 0x80808080u >> (8 * (3 - bq)));
    zacc += (y & mlo & mhi) >> 7;
  }
  return (zacc * 0x01010101u) >> 24;   // each byte lane holds at most BN/4
}

// This row's P~ words into the swizzled shared-memory tile that the P~V MMA reads:
// 16-byte chunk q of the row at chunk (q ^ pswz) of row address prow.
template <int BN>
__device__ __forceinline__ void store_p_row(const uint32_t* pw, uint32_t prow, uint32_t pswz) {
#pragma unroll
  for (int q = 0; q < BN / 16; ++q) {
    const uint32_t dst = prow + ((q ^ pswz) << 4);
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(dst), "r"(pw[4 * q]),
                 "r"(pw[4 * q + 1]), "r"(pw[4 * q + 2]), "r"(pw[4 * q + 3])
                 : "memory");
  }
}

// O *= alpha for the warp's 32 rows (its TMEM lane quarter), 64 columns per round
// trip.
template <int D>
__device__ __forceinline__ void rescale_o(uint32_t tO, float alpha) {
  const float2 a2 = make_float2(alpha, alpha);
#pragma unroll
  for (int cc = 0; cc < D / 32; cc += 2) {
    uint32_t o0[32], o1[32];
    tmem_ld32(tO + 32 * cc, o0);
    tmem_ld32(tO + 32 * cc + 32, o1);
    tmem_wait_ld();
#pragma unroll
    for (int k = 0; k < 32; k += 2) {
      const float2 r0 =
          __fmul2_rn(make_float2(__uint_as_float(o0[k]), __uint_as_float(o0[k + 1])), a2);
      const float2 r1 =
          __fmul2_rn(make_float2(__uint_as_float(o1[k]), __uint_as_float(o1[k + 1])), a2);
      o0[k] = __float_as_uint(r0.x);
      o0[k + 1] = __float_as_uint(r0.y);
      o1[k] = __float_as_uint(r1.x);
      o1[k + 1] = __float_as_uint(r1.y);
    }
    tmem_st32(tO + 32 * cc, o0);
    tmem_st32(tO + 32 * cc + 32, o1);
  }
  tmem_wait_st();
}

// Epilogue of one row: O = acc * inv_l from TMEM, stored as BF16 or FP32 at
// element offset obase of O when `live` (every lane takes part in the TMEM loads).
template <int D, bool OUT_BF16>
__device__ __forceinline__ void store_o_row(uint32_t tO, float inv_l, bool live, void* O,
                                            size_t obase) {
#pragma unroll
  for (int cc = 0; cc < D / 32; ++cc) {
    uint32_t o[32];
    tmem_ld32(tO + 32 * cc, o);
    tmem_wait_ld();
    float v[32];
#pragma unroll
    for (int k = 0; k < 32; ++k) v[k] = __uint_as_float(o[k]) * inv_l;
    if (live) {
      if constexpr (OUT_BF16) {
        uint32_t w[16];
#pragma unroll
        for (int k = 0; k < 16; ++k) {
          uint32_t bits;
          asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(bits) : "f"(v[2 * k + 1]), "f"(v[2 * k]));
          w[k] = bits;
        }
        uint4* out = reinterpret_cast<uint4*>(static_cast<uint16_t*>(O) + obase + 32 * cc);
#pragma unroll
        for (int k = 0; k < 4; ++k)
          out[k] = make_uint4(w[4 * k], w[4 * k + 1], w[4 * k + 2], w[4 * k + 3]);
      } else {
        float4* out = reinterpret_cast<float4*>(static_cast<float*>(O) + obase + 32 * cc);
#pragma unroll
        for (int k = 0; k < 8; ++k)
          out[k] = make_float4(v[4 * k], v[4 * k + 1], v[4 * k + 2], v[4 * k + 3]);
      }
    }
  }
}

}  // namespace fp8attn
