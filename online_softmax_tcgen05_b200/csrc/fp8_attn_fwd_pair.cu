// fp8_attn_fwd_pair.cu - the attention forward of fp8_attn_fwd.cu with two
// 128-row query tiles per CTA and one CTA per SM, the tiles' softmax warps
// taking turns on the exponential unit.
//
// Method: "P-Cast Precision in FP8 Attention: Sink-Induced Collapse and the
// Optimality of S=2^8" (arXiv 2606.06521, gist.science summary), section 1
// (Problem statement): an online softmax with running max m over KV blocks
// visited forward (0..N) or in reverse (N..0), S*P cast to E4M3 for P.V, S
// divided back out in the epilogue.  The arithmetic per row is the same as in
// fp8_attn_fwd.cu; only the schedule differs.
//
// Why two tiles: the softmax of one 128x128 score block issues one MUFU ex2
// per score, 1024 cycles of the SM's exponential unit per block, and spends a
// comparable time in work that does not use it (waiting for and loading the
// scores, the row max, the E4M3 cast and the collapse count, the P~ hand-off,
// the O rescale).  Two independent CTAs on an SM overlap those phases only by
// chance.  Here the two tiles of one CTA share each SMSP (softmax warp k of
// tile A and warp k + 4 of tile B), and a pair of named barriers per SMSP
// hands the exponential phase back and forth: while one warp runs its
// exponentials the other does the rest of its block, so the unit is kept busy
// by construction.  The turn is a hardware barrier (the waiting warp is not
// scheduled), never a spin.
//
// Tile pairs: two query tiles that read the same K and V blocks in the same
// order, so one K/V stream feeds both.  With an even GQA group the pair is the
// same tile of two query heads of one kv head (same rows, same mask); otherwise
// it is two consecutive tiles of one head, the block sequence then being the
// second tile's and the first tile seeing one fully masked block (causal), a
// no-op for it.
//
// Roles (320 threads):
//   warps 0-3  softmax of tile A, one thread per row (TMEM lanes 32w..32w+31)
//   warps 4-7  softmax of tile B (lanes 32(w-4)..)
//   warp 8     TMA producer: both Q tiles once, then K and V of each KV block
//   warp 9     MMA issuer and TMEM owner: S_A = Q_A K^T, S_B = Q_B K^T,
//              O_A += P~_A V, O_B += P~_B V (tcgen05 kind::f8f6f4, or kind::f16
//              for BF16 Q and K)
// TMEM: S_A [0, BN), S_B [BN, 2BN), O_A [2BN, 2BN+D), O_B [2BN+D, 2BN+2D).
// Every mbarrier wait is bounded in time; on expiry the CTA aborts as in
// fp8_attn_fwd.cu.  The named-barrier turns cannot deadlock: both warps of an
// SMSP execute the same number of turn operations whatever happens (an
// aborting warp keeps taking its turns without doing the work).
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "attn_kernel.cuh"
#include "fp8attn.h"
#include "row_max.cuh"
#include "sm100.cuh"
#include "softmax_block.cuh"

namespace fp8attn {
namespace pairk {

constexpr int NSTAGE = 2;
constexpr int NTHREADS = 320;

template <int D, int BN, int QB>
struct Smem {
  static constexpr int Q = 0;                            // Q_A, Q_B
  static constexpr int K = Q + 2 * BM * D * QB;
  static constexpr int V = K + NSTAGE * BN * D * QB;
  static constexpr int P = V + NSTAGE * BN * D;           // P~_A, P~_B
  static constexpr int BAR = P + 2 * BM * BN;
  // q_full, k_full[2], v_full[2], k_empty[2], v_empty[2], per tile: s_full,
  // s_free, p_full, o_done; drain
  static constexpr int NBAR = 1 + 4 * NSTAGE + 8 + 1;
  static constexpr int MISC = BAR + 8 * NBAR;   // tmem slot, abort, never, MMA idle flags
  static constexpr int BYTES = MISC + 16;
  // at least 120 KB: one CTA per SM (the CTA takes all 512 TMEM columns)
  static constexpr int ALLOC = (BYTES + 1024 > 120 * 1024) ? BYTES + 1024 : 120 * 1024;
  static constexpr uint32_t TMEM_COLS = 512;
  static_assert(2 * (BN + D) <= 512, "TMEM budget");
};

// Named barriers of the exponential turns: SMSP k uses TURN_A + k (tile A may
// start) and TURN_B + k (tile B may start); two warps (64 threads) each.
constexpr uint32_t TURN_A = 1, TURN_B = 5;
// What a turn covers: 1 = the exponentials and row sums; 2 = those, the E4M3
// cast and the collapse count; 0 = no turns (the two tiles run freely).
#ifndef FP8ATTN_TURN_SCOPE
#define FP8ATTN_TURN_SCOPE 1
#endif
constexpr int TURN_SCOPE = FP8ATTN_TURN_SCOPE;
#ifndef FP8ATTN_EXP_SPLIT
#define FP8ATTN_EXP_SPLIT 0
#endif
constexpr bool EXP_SPLIT = FP8ATTN_EXP_SPLIT != 0;

// Waits of this kernel's roles: with a suspend-time hint (ns) a waiting warp
// sleeps between probes instead of issuing them back to back.
#ifndef FP8ATTN_PAIR_WAIT_HINT_NS
#define FP8ATTN_PAIR_WAIT_HINT_NS 0
#endif
__device__ __forceinline__ bool pwait(uint32_t bar, uint32_t parity, const WaitCtl& ctl,
                                      uint32_t where) {
  if constexpr (FP8ATTN_PAIR_WAIT_HINT_NS > 0)
    return mbar_wait_hint(bar, parity, ctl, where, FP8ATTN_PAIR_WAIT_HINT_NS);
  else
    return mbar_wait(bar, parity, ctl, where);
}

// The turns order execution, not memory (no memory clobber: the scores stay in
// registers across them).  The running max passes through the wait and the row
// sum into the pass, so that the exponentials can be placed neither before the
// wait nor after the pass.
__device__ __forceinline__ float turn_wait(uint32_t id, float m) {
  float r;
  asm volatile("bar.sync %1, 64;\n\tmov.b32 %0, %2;" : "=f"(r) : "r"(id), "f"(m));
  return r;
}
__device__ __forceinline__ void turn_pass(uint32_t id, float after) {
  asm volatile("bar.arrive %0, 64;" ::"r"(id), "f"(after));
}

template <int D, int BN, bool OUT_BF16, bool COUNT, int QB>
__global__ void __launch_bounds__(NTHREADS, 1)
attn_fwd_pair_kernel(const __grid_constant__ CUtensorMap tmQ,
                     const __grid_constant__ CUtensorMap tmK,
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
  const uint32_t bar_tile0 = bar0 + 8u * (1 + 4 * NSTAGE);
  auto bar_s_full = [&](int x) { return bar_tile0 + 32u * x; };
  auto bar_s_free = [&](int x) { return bar_tile0 + 32u * x + 8; };
  auto bar_p_full = [&](int x) { return bar_tile0 + 32u * x + 16; };
  auto bar_o_done = [&](int x) { return bar_tile0 + 32u * x + 24; };
  const uint32_t bar_drain = bar_tile0 + 64;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::MISC);
  volatile uint32_t* abort_flag = reinterpret_cast<volatile uint32_t*>(smem + L::MISC + 4);
  volatile uint32_t* never_flag = reinterpret_cast<volatile uint32_t*>(smem + L::MISC + 8);
  // raised by the MMA warp once every MMA it issued has completed
  volatile uint32_t* mma_idle = reinterpret_cast<volatile uint32_t*>(smem + L::MISC + 12);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // Work unit: a row unit (a tile pair, or one tile for head pairs) of a plane
  // unit (a (batch, head) plane, or two planes of one kv head).  Causal units
  // run longest first within scheduling groups of sched_group plane units, as
  // in fp8_attn_fwd.cu.
  const int nrow = p.pair_heads ? p.num_q_tiles : (p.num_q_tiles + 1) / 2;
  int ru, pu;
  if (p.causal) {
    const int lin = (int)blockIdx.y * (int)gridDim.x + (int)blockIdx.x;
    const int per_group = nrow * p.sched_group;
    const int g = lin / per_group, inner = lin % per_group;
    ru = nrow - 1 - inner / p.sched_group;
    pu = g * p.sched_group + inner % p.sched_group;
  } else {
    ru = (int)blockIdx.x;
    pu = (int)blockIdx.y;
  }
  // (plane, tile) of tile A and of tile B
  const int bhA = p.pair_heads ? 2 * pu : pu, bhB = p.pair_heads ? 2 * pu + 1 : pu;
  const int tileA = p.pair_heads ? p.tile0 + ru : p.tile0 + 2 * ru;
  const int tileB = p.pair_heads ? tileA : tileA + 1;
  const int tile_end = p.tile0 + p.num_q_tiles;   // tiles of the launch's row range
  const int bkv = (bhA / p.H) * p.Hkv + (bhA % p.H) / p.group;   // both tiles read this kv head
  const int q_last = min(tileB * BM + BM - 1, p.N - 1);
  const int T = p.causal ? (q_last / BN + 1) : ((p.N + BN - 1) / BN);
  const WaitCtl ctl{abort_flag, p.timeout_ns};

  if (threadIdx.x == 0) {
    mbar_init(bar_q_full, 1);
    for (int s = 0; s < NSTAGE; ++s) {
      mbar_init(bar_k_full(s), 1);
      mbar_init(bar_v_full(s), 1);
      mbar_init(bar_k_empty(s), 1);
      mbar_init(bar_v_empty(s), 1);
    }
    for (int x = 0; x < 2; ++x) {
      mbar_init(bar_s_full(x), 1);
      mbar_init(bar_s_free(x), 4);
      mbar_init(bar_p_full(x), 4);
      mbar_init(bar_o_done(x), 1);
    }
    mbar_init(bar_drain, 1);
    *abort_flag = 0;
    *never_flag = 0;
    *mma_idle = 0;
    fence_barrier_init();
  }
  if (warp == 9) {
    tmem_alloc(smem_u32(tmem_slot), L::TMEM_COLS);
    tmem_relinquish();
  }
  if (warp == 8 && lane == 0) {
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 8) {
    // ------------------------------------------------------------ producer --
    if (lane == 0) {
      mbar_arrive_expect_tx(bar_q_full, 2 * BM * D * QB);
#pragma unroll
      for (int x = 0; x < 2; ++x) {
        const int qt = x ? tileB : tileA, qbh = x ? bhB : bhA;
        if constexpr (QB == 1) {
          tma_load_3d(sQ + x * BM * D, &tmQ, bar_q_full, 0, qt * BM, qbh);
        } else {
#pragma unroll
          for (int pn = 0; pn < D / 64; ++pn)
            tma_load_3d(sQ + x * BM * D * QB + pn * BM * 128, &tmQ, bar_q_full, 64 * pn, qt * BM,
                        qbh);
        }
      }
      int k_issued = 0, v_issued = 0;
      auto load_k = [&](int t) -> bool {
        const int st = t % NSTAGE, n = t / NSTAGE;
        if (t >= NSTAGE && !pwait(bar_k_empty(st), (n - 1) & 1, ctl, WAIT_PROD_KV_EMPTY))
          return false;
        if (t + 1 == p.debug_skip_kv_step) return true;   // testing: leave this K tile out
        mbar_arrive_expect_tx(bar_k_full(st), BN * D * QB);
        const int jrow = kv_block_at(t, T, p.kv_order) * BN;
        if constexpr (QB == 1) {
          tma_load_3d(sK + st * BN * D, &tmK, bar_k_full(st), 0, jrow, bkv);
        } else {
#pragma unroll
          for (int pn = 0; pn < D / 64; ++pn)
            tma_load_3d(sK + st * BN * D * QB + pn * BN * 128, &tmK, bar_k_full(st), 64 * pn,
                        jrow, bkv);
        }
        k_issued = t + 1;
        return true;
      };
      bool ok = load_k(0);
      for (int t = 0; ok && t < T; ++t) {
        if (t + 1 < T && !load_k(t + 1)) break;
        const int st = t % NSTAGE, n = t / NSTAGE;
        if (t >= NSTAGE && !pwait(bar_v_empty(st), (n - 1) & 1, ctl, WAIT_PROD_KV_EMPTY))
          break;
        mbar_arrive_expect_tx(bar_v_full(st), BN * D);
        tma_load_3d(sV + st * BN * D, &tmV, bar_v_full(st), 0, kv_block_at(t, T, p.kv_order) * BN,
                    bkv);
        v_issued = t + 1;
      }
      // drain: the last load issued into each stage lands before the CTA exits
      const WaitCtl drain{never_flag, DRAIN_TIMEOUT_NS};
      for (int t = k_issued - 1; t >= 0 && t >= k_issued - NSTAGE; --t)
        mbar_wait(bar_k_full(t % NSTAGE), (t / NSTAGE) & 1, drain, 0);
      for (int t = v_issued - 1; t >= 0 && t >= v_issued - NSTAGE; --t)
        mbar_wait(bar_v_full(t % NSTAGE), (t / NSTAGE) & 1, drain, 0);
      mbar_wait(bar_q_full, 0, drain, 0);
    }
  } else if (warp == 9) {
    // ----------------------------------------------------------------- MMA --
    // Per KV step t: QK^T(t+1) of tile A as soon as its softmax has read S_A(t),
    // then of tile B; P~V(t) of tile A as soon as P~_A(t) is stored, then of
    // tile B.  Tile B runs about half a block behind tile A (the turns), and
    // this order lets each tile's next scores be computed under its own softmax.
    constexpr uint32_t SWZ_QK = (D == 128) ? SWZ_128B : SWZ_64B;
    constexpr uint32_t SWZ_P = (BN == 128) ? SWZ_128B : SWZ_64B;
    constexpr uint32_t IDESC_QK = idesc_e4m3_f32(BM, BN, 0, 0);
    constexpr uint32_t IDESC_PV = idesc_e4m3_f32(BM, D, 0, 1);
    bool ok = pwait(bar_q_full, 0, ctl, WAIT_MMA_Q);
    auto issue_qk = [&](int x, int st) {
      tc_fence_after();
      if (lane == 0) {
        const uint32_t tS = tmem_base + x * BN;
        if constexpr (QB == 1) {
#pragma unroll
          for (int kk = 0; kk < D / 32; ++kk) {
            const uint64_t a = smem_desc(sQ + x * BM * D + 32 * kk, 16, 8 * D, SWZ_QK);
            const uint64_t bdesc = smem_desc(sK + st * BN * D + 32 * kk, 16, 8 * D, SWZ_QK);
            mma_e4m3_ss(tS, a, bdesc, IDESC_QK, kk > 0);
          }
        } else {
          constexpr uint32_t IDESC_QK16 = idesc_bf16_f32(BM, BN);
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t pn = kk / 4, off = 32 * (kk % 4);
            const uint64_t a =
                smem_desc(sQ + x * BM * D * QB + pn * BM * 128 + off, 16, 1024, SWZ_128B);
            const uint64_t bdesc =
                smem_desc(sK + st * BN * D * QB + pn * BN * 128 + off, 16, 1024, SWZ_128B);
            mma_bf16_ss(tS, a, bdesc, IDESC_QK16, kk > 0);
          }
        }
        mma_commit(bar_s_full(x));
      }
      __syncwarp();
    };
    auto issue_pv = [&](int x, int st, int t) {
      tc_fence_after();
      if (lane == 0) {
        const uint32_t pbuf = sP + x * BM * BN;
#pragma unroll
        for (int kk = 0; kk < BN / 32; ++kk) {
          const uint64_t a = smem_desc(pbuf + 32 * kk, 16, 8 * BN, SWZ_P);
          const uint64_t bdesc = smem_desc(sV + st * BN * D + kk * 32 * D, BN * D, 8 * D, SWZ_QK);
          mma_e4m3_ss(tmem_base + 2 * BN + x * D, a, bdesc, IDESC_PV,
                      (t > 0 || kk > 0) ? 1u : 0u);
        }
        mma_commit(bar_o_done(x));
      }
      __syncwarp();
    };
    if (ok) ok = pwait(bar_k_full(0), 0, ctl, WAIT_MMA_K);
    if (ok) {
      issue_qk(0, 0);
      issue_qk(1, 0);
      if (lane == 0) mma_commit(bar_k_empty(0));
      __syncwarp();
    }
    // Issue order per step t, the order in which the turns make the operands
    // ready (tile B runs about half a block behind tile A): QK^T_A(t+1),
    // P~V_B(t-1), QK^T_B(t+1), P~V_A(t).  Each tile's S(t+1) commit still
    // follows its own P~V(t-1).
    auto pv_b = [&](int t) -> bool {   // P~V_B(t), then V stage t is free
      const int st = t % NSTAGE;
      if (!pwait(bar_p_full(1), t & 1, ctl, WAIT_MMA_P)) return false;
      issue_pv(1, st, t);
      if (lane == 0) mma_commit(bar_v_empty(st));
      __syncwarp();
      return true;
    };
    for (int t = 0; ok && t < T; ++t) {
      const int st1 = (t + 1) % NSTAGE, ph1 = ((t + 1) / NSTAGE) & 1;
      if (t + 1 < T) {
        ok = pwait(bar_k_full(st1), ph1, ctl, WAIT_MMA_K) &&
             pwait(bar_s_free(0), t & 1, ctl, WAIT_MMA_S_FREE);
        if (!ok) break;
        issue_qk(0, st1);
      }
      if (t > 0 && !(ok = pv_b(t - 1))) break;
      if (t + 1 < T) {
        ok = pwait(bar_s_free(1), t & 1, ctl, WAIT_MMA_S_FREE);
        if (!ok) break;
        issue_qk(1, st1);
        if (lane == 0) mma_commit(bar_k_empty(st1));
        __syncwarp();
      }
      const int st = t % NSTAGE, ph = (t / NSTAGE) & 1;
      ok = pwait(bar_v_full(st), ph, ctl, WAIT_MMA_V) &&
           pwait(bar_p_full(0), t & 1, ctl, WAIT_MMA_P);
      if (!ok) break;
      issue_pv(0, st, t);
    }
    if (ok) ok = pv_b(T - 1);
    {
      // wait for every MMA this warp issued (after an abort too), then tell an
      // aborting softmax warp that TMEM and the P~ tiles are no longer in use
      const WaitCtl drain{never_flag, DRAIN_TIMEOUT_NS};
      if (lane == 0) mma_commit(bar_drain);
      __syncwarp();
      mbar_wait(bar_drain, 0, drain, 0);
      if (lane == 0) *mma_idle = 1;
    }
  } else {
    // ------------------------------------------------------------- softmax --
    const int x = warp >> 2, quarter = warp & 3;   // tile, TMEM lane quarter (= SMSP)
    const int r = 32 * quarter + lane;              // row within the tile
    const int my_tile = x ? tileB : tileA;
    const int q0 = my_tile * BM;
    const int row = q0 + r;
    const int bh = x ? bhB : bhA;
    const bool tile_valid = my_tile < tile_end;
    const uint32_t lane_off = (uint32_t)(32 * quarter) << 16;
    const uint32_t tS = tmem_base + lane_off + x * BN;
    const uint32_t tO = tmem_base + lane_off + 2 * BN + x * D;
    const uint32_t my_turn = (x == 0 ? TURN_A : TURN_B) + quarter;
    const uint32_t other_turn = (x == 0 ? TURN_B : TURN_A) + quarter;
    const float c = p.scale_log2;
    const uint32_t sc23 = (uint32_t)(p.N > 0) << 23;   // 2^23, a run-time value (exp2_poly2)
    float m_run = -INFINITY, l = 0.f;
    uint32_t cnt = 0, cnt_sink = 0;
    const uint32_t prow = sP + x * BM * BN + (r >> 3) * (8 * BN) + (r & 7) * BN;
    const uint32_t pswz = (BN == 128) ? (uint32_t)(r & 7) : (uint32_t)((r & 7) >> 1);
    const int lim = p.causal ? min(row, p.N - 1) : p.N - 1;   // last visible key

    // Tile A takes the first exponential turn.  Every block runs the same code
    // whether or not the CTA is aborting (only the waits are skipped then, and
    // the results are not stored), so both warps of an SMSP always take the
    // same number of turns.  An aborting warp first waits (bounded) until the
    // MMA warp has drained, so that its later TMEM and P~ accesses race with
    // no MMA in flight.
    bool settled = false;
    auto settle = [&](bool ok_now) {
      if (!ok_now && !settled) {
        const uint64_t t0 = globaltimer_ns();
        while (!*mma_idle && globaltimer_ns() - t0 < 2 * DRAIN_TIMEOUT_NS) {
        }
        settled = true;
      }
    };
    if (TURN_SCOPE && x == 1) turn_pass(other_turn, 0.f);
    bool ok = __all_sync(0xffffffffu, pwait(bar_s_full(x), 0, ctl, WAIT_SM_S_FULL));
    settle(ok);
    for (int t = 0; t < T; ++t) {
      const int j0 = kv_block_at(t, T, p.kv_order) * BN;
      uint32_t sr[BN];
      float* s = reinterpret_cast<float*>(sr);
      const bool need_mask = (p.causal && j0 + BN - 1 > q0) || (j0 + BN > p.N);
      const bool plain = !need_mask && j0 >= p.n_sink && !p.denom_cast && p.s_mul == 1.f;
      float m_new, alpha;
      uint32_t pw[BN / 4];
      {
        tc_fence_after();
        if constexpr (COUNT && BN == 128) {
          // one 128-column load in the counting kernel (as in the one-tile kernel;
          // timed 0.9-2.7% faster here, the plain kernel unchanged)
          tmem_ld128(tS, *reinterpret_cast<uint32_t(*)[128]>(&sr[0]));
        } else {
#pragma unroll
          for (int cc = 0; cc < BN / 32; ++cc)
            tmem_ld32(tS + 32 * cc, *reinterpret_cast<uint32_t(*)[32]>(&sr[32 * cc]));
        }
        tmem_wait_ld();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar_s_free(x));
        if (need_mask) mask_scores<BN>(s, j0, lim);
        const float mx = row_max<BN>(s);
        m_new = fmax_nan(m_run, mx * c);
        alpha = (m_new == -INFINITY) ? 1.f : ex2_approx(m_run - m_new);
      }

      // ---- this SMSP's turn on the exponential unit ----
      // 2^(s*c - m + log2S) with its row sums, then the E4M3 cast and the
      // collapse count, as one body (branch-free on plain blocks) so that the
      // integer work fills the issue slots between the exponentials.
      const float m_turn = TURN_SCOPE ? turn_wait(my_turn, m_new) : m_new;
      auto block_body = [&](auto plain_tag) {
        constexpr bool PLAIN = decltype(plain_tag)::value;
        const float m_use = (m_turn == -INFINITY) ? 0.f : m_turn;
        const float2 c2 = make_float2(c, c), nm2 = make_float2(p.log2S - m_use, p.log2S - m_use);
        const float rowsum =
            exp2_rowsum<BN, PLAIN ? POLY_OF_8 : 0, EXP_SPLIT>(s, c2, nm2, sc23);
        if constexpr (TURN_SCOPE == 1) {
          if (x == 0 || t + 1 < T) turn_pass(other_turn, rowsum);
        }
        if (PLAIN || !p.denom_cast) l = scale_add(alpha, l, rowsum);
        cast_e4m3<BN, !PLAIN>(s, p.s_mul, pw);
        if constexpr (!PLAIN) {
          if (p.denom_cast) l = scale_add(alpha, l, cast_value_sum<BN>(pw));
        }
        if constexpr (COUNT) {
          // Collapse: a visible non-sink key whose E4M3 byte is zero; blocks holding
          // a sink or a masked key count the keys n_sink <= j <= lim only
          uint32_t cblk;
          if (PLAIN || (j0 >= p.n_sink && !need_mask))
            cblk = zero_bytes_all<BN>(pw);
          else
            cblk = zero_bytes_range<BN>(pw, max(p.n_sink - j0, 0), min(lim - j0, BN - 1));
          cnt += cblk;
          if constexpr (!PLAIN) {
            if (j0 < p.n_sink) cnt_sink += cblk;
          }
        }
        if constexpr (TURN_SCOPE == 2) {
          // hand the unit to the other tile's warp (tile B's last block has no
          // taker: tile A is done with its turns)
          if (x == 0 || t + 1 < T) turn_pass(other_turn, __uint_as_float(pw[BN / 4 - 1]));
        }
      };
      {
        if (plain)
          block_body(BoolTag<true>{});
        else
          block_body(BoolTag<false>{});
        // P~V(t-1) must be done before the P~ tile is rewritten and O rescaled.
        // The commit that completes S(t+1) tracks every MMA issued before
        // QK^T(t+1), P~V(t-1) among them; the last block waits for P~V(t-1).
        if (t + 1 < T) {
          ok = ok && __all_sync(0xffffffffu,
                                pwait(bar_s_full(x), (t + 1) & 1, ctl, WAIT_SM_S_FULL));
        } else if (t > 0) {
          ok = ok && __all_sync(0xffffffffu,
                                pwait(bar_o_done(x), (t - 1) & 1, ctl, WAIT_SM_O_DONE));
        }
        settle(ok);
      }
      {
        tc_fence_after();
        store_p_row<BN>(pw, prow, pswz);
        if (t > 0) {
          // O *= alpha for this warp's rows when one of their maxima rose
          if (__any_sync(0xffffffffu, alpha != 1.f)) rescale_o<D>(tO, alpha);
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar_p_full(x));
        m_run = m_new;
      }
    }

    if (ok) {
      ok = __all_sync(0xffffffffu, pwait(bar_o_done(x), (T - 1) & 1, ctl, WAIT_EPI_O_DONE));
    }
    if (ok) {
      tc_fence_after();
      // O = acc / (S l): one correctly rounded reciprocal per row, then a
      // multiply per element (s_mul = 1 when l already carries S)
      const float inv_l = __frcp_rn(p.denom_cast ? l : __fmul_rn(l, p.s_mul));
      const bool live = tile_valid && row < p.N;
      const size_t obase = ((size_t)bh * p.N + (size_t)(live ? row : 0)) * D;
      store_o_row<D, OUT_BF16>(tO, inv_l, live, p.O, obase);
      if constexpr (COUNT) {
        if (!live) cnt = cnt_sink = 0;   // rows past N or outside the launch's range
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
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem_base, L::TMEM_COLS);
  }
}

template <int D, int BN, bool OUT_BF16, bool COUNT, int QB>
cudaError_t launch(const CUtensorMap& q, const CUtensorMap& k, const CUtensorMap& v,
                   const KParams& kp, cudaStream_t stream) {
  using L = Smem<D, BN, QB>;
  auto kern = attn_fwd_pair_kernel<D, BN, OUT_BF16, COUNT, QB>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::ALLOC);
  if (e != cudaSuccess) return e;
  const int nrow = kp.pair_heads ? kp.num_q_tiles : (kp.num_q_tiles + 1) / 2;
  const int nplane = kp.pair_heads ? kp.B * kp.H / 2 : kp.B * kp.H;
  dim3 grid(nrow, nplane);
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

}  // namespace pairk

cudaError_t launch_attn_pair(int d, int bn, bool o_bf16, bool count, bool qk_bf16,
                             const CUtensorMap& q, const CUtensorMap& k, const CUtensorMap& v,
                             const KParams& kp, cudaStream_t stream) {
  using namespace pairk;
  if (d == 128)
    return bn == 128 ? launch_dt<128, 128>(o_bf16, count, qk_bf16, q, k, v, kp, stream)
                     : launch_dt<128, 64>(o_bf16, count, qk_bf16, q, k, v, kp, stream);
  return bn == 128 ? launch_dt<64, 128>(o_bf16, count, qk_bf16, q, k, v, kp, stream)
                   : launch_dt<64, 64>(o_bf16, count, qk_bf16, q, k, v, kp, stream);
}

}  // namespace fp8attn
