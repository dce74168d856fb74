// fp8_attn_fwd.cu - FP8 (E4M3) attention forward for B200 (sm_100a) with the
// P-cast scale S and a run-time KV-block order: the kernels and their launch
// entries (attn_kernel.cuh).  The C ABI of include/fp8attn.h, which validates
// the arguments and builds the tensor maps, is in fp8attn_abi.cu.
//
// Method: "P-Cast Precision in FP8 Attention: Sink-Induced Collapse and the
// Optimality of S=2^8" (arXiv 2606.06521, gist.science summary).  Section 1
// (Problem statement) fixes what is computed: an online softmax with running
// max m over KV blocks visited forward (0..N) or in reverse (N..0), the
// probability tile multiplied by a static S and cast to E4M3 for P.V, and S
// divided back out in the epilogue.  Section 2 (Optimisation 1) is why the
// order is a parameter; the collapse counter measures the P-collapse of
// section 1.
//
// One CTA owns one 128-row query tile of one (batch, head) and runs four
// warp-specialised roles (two CTAs share an SM so that one CTA's softmax
// overlaps the other's tensor-core work):
//   warp 4     TMA producer: Q tile once, then K and V tiles of each KV block in
//              visiting order into a 2-stage ring (3-D tensor maps, so a ragged
//              last block reads zeros past N).
//   warp 5     MMA issuer: S = Q K^T into TMEM (tcgen05 kind::f8f6f4, M=128,
//              N=block_n, K=32 per instruction), then O += P~ V into TMEM
//              (V as an MN-major operand).  Owns the TMEM allocation.
//   warps 0-3  softmax, one thread per query row: tcgen05.ld of its score row,
//              row max, exponentials, FP32 row sum, E4M3 cast of S*p into a
//              swizzled shared-memory P~ tile, collapse count, the O rescale in
//              TMEM when a row max changed, and the epilogue O / (S l).  For
//              S = 2^k, S*p is one exp2 with k added to the argument and the row
//              sum is of S*p (so S divides out with l); for any other S the
//              kernel forms fl(S * p) with an FP32 multiply, as the method states,
//              sums p, and divides by fl(S * l).
// Every mbarrier wait is bounded in time: on expiry the CTA sets a shared
// abort flag, every role leaves its loop, in-flight copies and MMAs are
// drained, TMEM is freed and the status word (if given) records where.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "attn_kernel.cuh"
#include "fp8attn.h"
#include "row_max.cuh"
#include "sm100.cuh"
#include "softmax_block.cuh"

namespace fp8attn {

constexpr int NSTAGE = 2;       // K/V ring depth
constexpr int NTHREADS = 192;   // 4 softmax warps + TMA warp + MMA warp

template <int D, int BN, int QB>
struct Smem {
  static constexpr int Q = 0;
  static constexpr int K = Q + BM * D * QB;
  static constexpr int V = K + NSTAGE * BN * D * QB;
  static constexpr int P = V + NSTAGE * BN * D;
  static constexpr int BAR = P + BM * BN;
  // barriers: q_full, k_full[2], v_full[2], k_empty[2], v_empty[2], s_full, s_free, p_full,
  // o_done, drain
  static constexpr int NBAR = 1 + 4 * NSTAGE + 5;
  static constexpr int MISC = BAR + 8 * NBAR;   // tmem base slot, abort flag
  static constexpr int BYTES = MISC + 16;
  // slack to align the base to 1024, and at least 80 KB so that no more than two
  // CTAs share an SM: two 256-column TMEM allocations fill the SM's 512 columns
  static constexpr int ALLOC = (BYTES + 1024 > 80 * 1024) ? BYTES + 1024 : 80 * 1024;
  static constexpr uint32_t TMEM_COLS = 256;    // S: BN columns, O: D columns
  static_assert(BN + D <= (int)TMEM_COLS, "TMEM budget");
};

// QB: bytes per Q / K element.  1: E4M3 Q and K, QK^T as kind::f8f6f4.
// 2: BF16 Q and K, QK^T as kind::f16 (the "kernel-faithful" reading of the
// P-cast paper's simulation, where only P~ and V are E4M3); each BF16 row is
// staged as D/64 panels of 64 elements (128-byte swizzle atoms).
template <int D, int BN, bool OUT_BF16, bool COUNT, int QB>
__global__ void __launch_bounds__(NTHREADS, 2)
attn_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                const __grid_constant__ CUtensorMap tmV, const KParams p) {
  using L = Smem<D, BN, QB>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t sQ = sbase + L::Q, sK = sbase + L::K, sV = sbase + L::V, sP = sbase + L::P;
  const uint32_t bar0 = sbase + L::BAR;
  const uint32_t bar_q_full = bar0;
  auto bar_k_full = [&](int s) { return bar0 + 8u * (1 + s); };
  auto bar_v_full = [&](int s) { return bar0 + 8u * (1 + NSTAGE + s); };
  auto bar_k_empty = [&](int s) { return bar0 + 8u * (1 + 2 * NSTAGE + s); };
  auto bar_v_empty = [&](int s) { return bar0 + 8u * (1 + 3 * NSTAGE + s); };
  const uint32_t bar_s_full = bar0 + 8u * (1 + 4 * NSTAGE);
  const uint32_t bar_s_free = bar_s_full + 8;
  const uint32_t bar_p_full = bar_s_full + 16;
  const uint32_t bar_o_done = bar_s_full + 24;
  const uint32_t bar_drain = bar_s_full + 32;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::MISC);
  volatile uint32_t* abort_flag = reinterpret_cast<volatile uint32_t*>(smem + L::MISC + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // Causal tiles differ in length (tile i has i + 1 KV blocks).  CTAs are issued
  // one scheduling group of sched_group consecutive (batch, head) planes at a
  // time, longest tile first within the group, so that each group ends with its
  // shortest tiles.  A group spans the query heads of as many KV heads as keep
  // their K and V within a quarter of the L2.  The block scheduler issues CTAs
  // in linear index order (x fastest).
  int tile, bh;
  if (p.causal) {
    const int lin = (int)blockIdx.y * (int)gridDim.x + (int)blockIdx.x;
    const int per_group = p.num_q_tiles * p.sched_group;
    const int g = lin / per_group, inner = lin % per_group;
    tile = p.tile0 + p.num_q_tiles - 1 - inner / p.sched_group;
    bh = g * p.sched_group + inner % p.sched_group;
  } else {
    tile = p.tile0 + (int)blockIdx.x;
    bh = (int)blockIdx.y;
  }
  const int h = bh % p.H, b = bh / p.H;
  const int bkv = b * p.Hkv + h / p.group;
  const int q0 = tile * BM;
  const int last_row = min(q0 + BM - 1, p.N - 1);
  const int T = p.causal ? (last_row / BN + 1) : ((p.N + BN - 1) / BN);
  const WaitCtl ctl{abort_flag, p.timeout_ns};

  if (threadIdx.x == 0) {
    mbar_init(bar_q_full, 1);
    for (int s = 0; s < NSTAGE; ++s) {
      mbar_init(bar_k_full(s), 1);
      mbar_init(bar_v_full(s), 1);
      mbar_init(bar_k_empty(s), 1);
      mbar_init(bar_v_empty(s), 1);
    }
    mbar_init(bar_s_full, 1);
    mbar_init(bar_s_free, 4);
    mbar_init(bar_p_full, 4);
    mbar_init(bar_o_done, 1);
    mbar_init(bar_drain, 1);
    *abort_flag = 0;
    *reinterpret_cast<volatile uint32_t*>(smem + L::MISC + 8) = 0;   // never raised: drain waits
    fence_barrier_init();
  }
  if (warp == 5) {
    tmem_alloc(smem_u32(tmem_slot), L::TMEM_COLS);
    tmem_relinquish();
  }
  if (warp == 4 && lane == 0) {
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 4) {
    // ------------------------------------------------------------ producer --
    if (lane == 0) {
      // Q: E4M3 rows in one box; BF16 rows as D/64 panels of 64 elements
      mbar_arrive_expect_tx(bar_q_full, BM * D * QB);
      if constexpr (QB == 1) {
        tma_load_3d(sQ, &tmQ, bar_q_full, 0, q0, bh);
      } else {
#pragma unroll
        for (int pn = 0; pn < D / 64; ++pn)
          tma_load_3d(sQ + pn * BM * 128, &tmQ, bar_q_full, 64 * pn, q0, bh);
      }
      // K runs one KV step ahead of V: K(t+1) needs only QK^T(t-1) to have
      // released its stage, V(t) needs P~V(t-2).
      int k_issued = 0, v_issued = 0;
      auto load_k = [&](int t) -> bool {
        const int st = t % NSTAGE, n = t / NSTAGE;
        if (t >= NSTAGE && !mbar_wait(bar_k_empty(st), (n - 1) & 1, ctl, WAIT_PROD_KV_EMPTY))
          return false;
        if (t + 1 == p.debug_skip_kv_step) return true;   // testing: leave this K tile out
        mbar_arrive_expect_tx(bar_k_full(st), BN * D * QB);
        {
          const int jrow = kv_block_at(t, T, p.kv_order) * BN;
          if constexpr (QB == 1) {
            tma_load_3d(sK + st * BN * D, &tmK, bar_k_full(st), 0, jrow, bkv);
          } else {
#pragma unroll
            for (int pn = 0; pn < D / 64; ++pn)
              tma_load_3d(sK + st * BN * D * QB + pn * BN * 128, &tmK, bar_k_full(st), 64 * pn,
                          jrow, bkv);
          }
        }
        k_issued = t + 1;
        return true;
      };
      bool ok = load_k(0);
      for (int t = 0; ok && t < T; ++t) {
        if (t + 1 < T && !load_k(t + 1)) break;
        const int st = t % NSTAGE, n = t / NSTAGE;
        if (t >= NSTAGE && !mbar_wait(bar_v_empty(st), (n - 1) & 1, ctl, WAIT_PROD_KV_EMPTY))
          break;
        mbar_arrive_expect_tx(bar_v_full(st), BN * D);
        tma_load_3d(sV + st * BN * D, &tmV, bar_v_full(st), 0, kv_block_at(t, T, p.kv_order) * BN,
                    bkv);
        v_issued = t + 1;
      }
      {
        // drain: the last load issued into each stage must land before the CTA
        // exits (immediate when the consumers took them all; needed after an abort)
        const WaitCtl drain{reinterpret_cast<volatile uint32_t*>(smem + L::MISC + 8),
                            DRAIN_TIMEOUT_NS};
        for (int t = k_issued - 1; t >= 0 && t >= k_issued - NSTAGE; --t)
          mbar_wait(bar_k_full(t % NSTAGE), (t / NSTAGE) & 1, drain, 0);
        for (int t = v_issued - 1; t >= 0 && t >= v_issued - NSTAGE; --t)
          mbar_wait(bar_v_full(t % NSTAGE), (t / NSTAGE) & 1, drain, 0);
        mbar_wait(bar_q_full, 0, drain, 0);
      }
    }
  } else if (warp == 5) {
    // ----------------------------------------------------------------- MMA --
    constexpr uint32_t SWZ_QK = (D == 128) ? SWZ_128B : SWZ_64B;
    constexpr uint32_t SWZ_P = (BN == 128) ? SWZ_128B : SWZ_64B;
    constexpr uint32_t IDESC_QK = idesc_e4m3_f32(BM, BN, 0, 0);
    constexpr uint32_t IDESC_PV = idesc_e4m3_f32(BM, D, 0, 1);
    const uint32_t tS = tmem_base, tO = tmem_base + BN;
    bool ok = mbar_wait(bar_q_full, 0, ctl, WAIT_MMA_Q);
    auto issue_qk = [&](int st) {
      tc_fence_after();
      if (lane == 0) {
        if constexpr (QB == 1) {
#pragma unroll
          for (int kk = 0; kk < D / 32; ++kk) {
            const uint64_t a = smem_desc(sQ + 32 * kk, 16, 8 * D, SWZ_QK);
            const uint64_t bdesc = smem_desc(sK + st * BN * D + 32 * kk, 16, 8 * D, SWZ_QK);
            mma_e4m3_ss(tS, a, bdesc, IDESC_QK, kk > 0);
          }
        } else {
          // BF16: K = 16 per instruction, 4 steps of 32 bytes per 64-element panel
          constexpr uint32_t IDESC_QK16 = idesc_bf16_f32(BM, BN);
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t pn = kk / 4, off = 32 * (kk % 4);
            const uint64_t a = smem_desc(sQ + pn * BM * 128 + off, 16, 1024, SWZ_128B);
            const uint64_t bdesc =
                smem_desc(sK + st * BN * D * QB + pn * BN * 128 + off, 16, 1024, SWZ_128B);
            mma_bf16_ss(tS, a, bdesc, IDESC_QK16, kk > 0);
          }
        }
        mma_commit(bar_s_full);
        mma_commit(bar_k_empty(st));
      }
      __syncwarp();
    };
    if (ok) ok = mbar_wait(bar_k_full(0), 0, ctl, WAIT_MMA_K);
    if (ok) issue_qk(0);
    for (int t = 0; ok && t < T; ++t) {
      if (t + 1 < T) {
        const int st1 = (t + 1) % NSTAGE, ph1 = ((t + 1) / NSTAGE) & 1;
        ok = mbar_wait(bar_k_full(st1), ph1, ctl, WAIT_MMA_K) &&
             mbar_wait(bar_s_free, t & 1, ctl, WAIT_MMA_S_FREE);
        if (!ok) break;
        issue_qk(st1);
      }
      const int st = t % NSTAGE, ph = (t / NSTAGE) & 1;
      ok = mbar_wait(bar_v_full(st), ph, ctl, WAIT_MMA_V) &&
           mbar_wait(bar_p_full, t & 1, ctl, WAIT_MMA_P);
      if (!ok) break;
      tc_fence_after();
      if (lane == 0) {
#pragma unroll
        for (int kk = 0; kk < BN / 32; ++kk) {
          const uint64_t a = smem_desc(sP + 32 * kk, 16, 8 * BN, SWZ_P);
          const uint64_t bdesc =
              smem_desc(sV + st * BN * D + kk * 32 * D, BN * D, 8 * D, SWZ_QK);
          mma_e4m3_ss(tO, a, bdesc, IDESC_PV, (t > 0 || kk > 0) ? 1u : 0u);
        }
        mma_commit(bar_o_done);
        mma_commit(bar_v_empty(st));
      }
      __syncwarp();
    }
    if (!ok) {
      // drain every MMA this warp issued before TMEM is released
      const WaitCtl drain{reinterpret_cast<volatile uint32_t*>(smem + L::MISC + 8),
                          DRAIN_TIMEOUT_NS};
      if (lane == 0) mma_commit(bar_drain);
      __syncwarp();
      mbar_wait(bar_drain, 0, drain, 0);
    }
  } else {
    // ------------------------------------------------------------- softmax --
    const int r = threadIdx.x;   // row within the tile; warp w reads TMEM lanes 32w..32w+31
    const int row = q0 + r;
    const uint32_t lane_off = (uint32_t)(32 * warp) << 16;
    const uint32_t tS = tmem_base + lane_off, tO = tmem_base + lane_off + BN;
    const float c = p.scale_log2;
    const uint32_t sc23 = (uint32_t)(p.N > 0) << 23;   // 2^23, a run-time value (exp2_poly2)
    float m_run = -INFINITY, l = 0.f;
    uint32_t cnt = 0, cnt_sink = 0;
    bool ok = true;
    // this thread's P~ row in the swizzled tile (128B swizzle for 128-byte rows,
    // 64B swizzle for 64-byte rows)
    const uint32_t prow = sP + (r >> 3) * (8 * BN) + (r & 7) * BN;
    const uint32_t pswz = (BN == 128) ? (uint32_t)(r & 7) : (uint32_t)((r & 7) >> 1);

    // S(0) here; S(t+1) at the end of block t (see below)
    ok = __all_sync(0xffffffffu, mbar_wait(bar_s_full, 0, ctl, WAIT_SM_S_FULL));
    for (int t = 0; ok && t < T; ++t) {
      const int j0 = kv_block_at(t, T, p.kv_order) * BN;
      tc_fence_after();
      uint32_t sr[BN];
      if constexpr (COUNT && BN == 128) {
        // one 128-column load: timed 1.7-1.9% faster than four 32-column loads in
        // the counting kernel and 2.5-3% slower in the plain one (same values)
        tmem_ld128(tS, *reinterpret_cast<uint32_t(*)[128]>(&sr[0]));
      } else {
#pragma unroll
        for (int cc = 0; cc < BN / 32; ++cc)
          tmem_ld32(tS + 32 * cc, *reinterpret_cast<uint32_t(*)[32]>(&sr[32 * cc]));
      }
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar_s_free);

      float* s = reinterpret_cast<float*>(sr);
      const bool need_mask = (p.causal && j0 + BN - 1 > q0) || (j0 + BN > p.N);
      const int lim = p.causal ? min(row, p.N - 1) : p.N - 1;   // last visible key
      // Most blocks hold no masked key and no sink key and use the FP32 row sum
      // and a power-of-two S: they take a copy of the block's arithmetic with no
      // branch in it, so that the integer work of the cast and the count can
      // interleave with the exponentials of the same block.
      const bool plain = !need_mask && j0 >= p.n_sink && !p.denom_cast && p.s_mul == 1.f;
      float m_new, alpha;
      uint32_t pw[BN / 4];
      auto block_math = [&](auto plain_tag) {
        constexpr bool PLAIN = decltype(plain_tag)::value;
        if constexpr (!PLAIN) {
          if (need_mask) mask_scores<BN>(s, j0, lim);
        }
        const float mx = row_max<BN>(s);
        m_new = fmax_nan(m_run, mx * c);
        const float m_use = (m_new == -INFINITY) ? 0.f : m_new;
        alpha = (m_new == -INFINITY) ? 1.f : ex2_approx(m_run - m_new);
        // 2^(s*c - m + log2S): for S = 2^k (log2S = k) that is S*p and its row sum
        // carries S; otherwise (log2S = 0) it is p, multiplied by S in the cast.
        const float2 c2 = make_float2(c, c), nm2 = make_float2(p.log2S - m_use, p.log2S - m_use);
        uint32_t zeros_plain = 0;   // the plain counting body's zero bytes
        float rowsum;
        if constexpr (PLAIN && COUNT) {
          rowsum = exp_cast_count_plain<BN, POLY_OF_8>(s, c2, nm2, sc23, pw, &zeros_plain);
        } else {
          rowsum = exp2_rowsum<BN, PLAIN ? POLY_OF_8 : 0, false>(s, c2, nm2, sc23);
          cast_e4m3<BN, !PLAIN>(s, p.s_mul, pw);
        }
        if (PLAIN || !p.denom_cast) l = scale_add(alpha, l, rowsum);
        if constexpr (!PLAIN) {
          if (p.denom_cast) l = scale_add(alpha, l, cast_value_sum<BN>(pw));
        }
        if constexpr (COUNT) {
          // Collapse: a visible non-sink key whose E4M3 byte is zero (P~ is never
          // negative, so byte 0 <=> the cast flushed S*p to zero).  Blocks that
          // hold a sink or a masked key count the keys n_sink <= j <= lim only.
          uint32_t cblk;
          if constexpr (PLAIN)
            cblk = zeros_plain;
          else if (j0 >= p.n_sink && !need_mask)
            cblk = zero_bytes_all<BN>(pw);
          else
            cblk = zero_bytes_range<BN>(pw, max(p.n_sink - j0, 0), min(lim - j0, BN - 1));
          cnt += cblk;
          if constexpr (!PLAIN) {
            if (j0 < p.n_sink) cnt_sink += cblk;
          }
        }
      };
      if (plain)
        block_math(BoolTag<true>{});
      else
        block_math(BoolTag<false>{});
      // P~V(t-1) must be done before the P~ tile is rewritten and O rescaled.  The
      // commit that completes S(t+1) tracks every MMA issued before QK^T(t+1),
      // P~V(t-1) among them, so one wait serves both this block's hand-off and
      // the next block's scores; the last block waits for P~V(t-1) itself.
      if (t + 1 < T) {
        ok = __all_sync(0xffffffffu, mbar_wait(bar_s_full, (t + 1) & 1, ctl, WAIT_SM_S_FULL));
        if (!ok) break;
      } else if (t > 0) {
        ok = __all_sync(0xffffffffu, mbar_wait(bar_o_done, (t - 1) & 1, ctl, WAIT_SM_O_DONE));
        if (!ok) break;
      }
      tc_fence_after();
      store_p_row<BN>(pw, prow, pswz);
      if (t > 0) {
        // O *= alpha for this warp's rows when one of their maxima rose
        if (__any_sync(0xffffffffu, alpha != 1.f)) rescale_o<D>(tO, alpha);
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar_p_full);
      m_run = m_new;
    }

    if (ok) {
      ok = __all_sync(0xffffffffu, mbar_wait(bar_o_done, (T - 1) & 1, ctl, WAIT_EPI_O_DONE));
    }
    if (ok) {
      tc_fence_after();
      // O = acc / (S l): one correctly rounded reciprocal per row, then a
      // multiply per element.  For S = 2^k, l already is the row sum of S*p
      // (s_mul = 1); otherwise the denominator is fl(S * l).  The cast-value row
      // sum carries S in its values.
      const float inv_l = __frcp_rn(p.denom_cast ? l : __fmul_rn(l, p.s_mul));
      const bool live = row < p.N;
      const size_t obase = ((size_t)bh * p.N + (size_t)(live ? row : 0)) * D;
      store_o_row<D, OUT_BF16>(tO, inv_l, live, p.O, obase);
      if constexpr (COUNT) {
        if (!live) cnt = cnt_sink = 0;   // padding rows past a ragged N
        if (p.rows && live) p.rows[(size_t)bh * p.N + row] = cnt;
        const uint32_t wsum = __reduce_add_sync(0xffffffffu, cnt);
        const uint32_t wsink = __reduce_add_sync(0xffffffffu, cnt_sink);
        if (lane == 0) {
          if (wsum) atomicAdd(p.ctr, (unsigned long long)wsum);
          if (p.ctr_sink && wsink) atomicAdd(p.ctr_sink, (unsigned long long)wsink);
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (threadIdx.x == 0 && *abort_flag && p.status) atomicCAS(p.status, 0u, 0x100u | *abort_flag);
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem_base, L::TMEM_COLS);
  }
}

// ------------------------------------------------------------- E4M3 cast --
__global__ void e4m3_scale_cast_kernel(const float* __restrict__ P, uint8_t* __restrict__ out,
                                       size_t n, float S) {
  const size_t n8 = n / 8;
  const size_t stride = (size_t)gridDim.x * blockDim.x;
  for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n8; i += stride) {
    const float4 a = reinterpret_cast<const float4*>(P)[2 * i];
    const float4 b = reinterpret_cast<const float4*>(P)[2 * i + 1];
    const uint32_t w0 = pack_e4m3x4(S * a.x, S * a.y, S * a.z, S * a.w);
    const uint32_t w1 = pack_e4m3x4(S * b.x, S * b.y, S * b.z, S * b.w);
    reinterpret_cast<uint2*>(out)[i] = make_uint2(w0, w1);
  }
  if (blockIdx.x == 0 && threadIdx.x < n - n8 * 8) {
    const size_t i = n8 * 8 + threadIdx.x;
    out[i] = (uint8_t)(cvt_e4m3x2(0.f, S * P[i]) & 0xFFu);
  }
}

// ------------------------------------------------------------- launches --
namespace {

template <int D, int BN, bool OUT_BF16, bool COUNT, int QB>
cudaError_t launch(const CUtensorMap& q, const CUtensorMap& k, const CUtensorMap& v,
                   const KParams& kp, cudaStream_t stream) {
  using L = Smem<D, BN, QB>;
  auto kern = attn_fwd_kernel<D, BN, OUT_BF16, COUNT, QB>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::ALLOC);
  if (e != cudaSuccess) return e;
  dim3 grid(kp.num_q_tiles, kp.B * kp.H);
  kern<<<grid, NTHREADS, L::ALLOC, stream>>>(q, k, v, kp);
  return cudaGetLastError();
}

template <int D, int BN, int QB>
cudaError_t launch_q(bool bf16, bool count, const CUtensorMap& q, const CUtensorMap& k,
                     const CUtensorMap& v, const KParams& kp, cudaStream_t s) {
  if (bf16) return count ? launch<D, BN, true, true, QB>(q, k, v, kp, s)
                         : launch<D, BN, true, false, QB>(q, k, v, kp, s);
  return count ? launch<D, BN, false, true, QB>(q, k, v, kp, s)
               : launch<D, BN, false, false, QB>(q, k, v, kp, s);
}

template <int D, int BN>
cudaError_t launch_dt(bool bf16, bool count, bool qk_bf16, const CUtensorMap& q,
                      const CUtensorMap& k, const CUtensorMap& v, const KParams& kp,
                      cudaStream_t s) {
  return qk_bf16 ? launch_q<D, BN, 2>(bf16, count, q, k, v, kp, s)
                 : launch_q<D, BN, 1>(bf16, count, q, k, v, kp, s);
}

}  // namespace

cudaError_t launch_attn(int d, int bn, bool o_bf16, bool count, bool qk_bf16,
                        const CUtensorMap& q, const CUtensorMap& k, const CUtensorMap& v,
                        const KParams& kp, cudaStream_t stream) {
  if (d == 128)
    return bn == 128 ? launch_dt<128, 128>(o_bf16, count, qk_bf16, q, k, v, kp, stream)
                     : launch_dt<128, 64>(o_bf16, count, qk_bf16, q, k, v, kp, stream);
  return bn == 128 ? launch_dt<64, 128>(o_bf16, count, qk_bf16, q, k, v, kp, stream)
                   : launch_dt<64, 64>(o_bf16, count, qk_bf16, q, k, v, kp, stream);
}

cudaError_t launch_e4m3_scale_cast(const float* P, uint8_t* out, size_t n, float S,
                                   cudaStream_t stream) {
  const size_t n8 = n / 8;
  size_t blocks = (n8 + 255) / 256;
  if (blocks > (size_t)148 * 16) blocks = (size_t)148 * 16;
  if (blocks < 1) blocks = 1;
  e4m3_scale_cast_kernel<<<(unsigned)blocks, 256, 0, stream>>>(P, out, n, S);
  return cudaGetLastError();
}

}  // namespace fp8attn
