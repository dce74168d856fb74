// attn_kernel.cuh - what the host side of the library needs from the attention
// kernel: the query-tile height, the kernel's parameter block, the device
// status codes of its bounded waits, and the two launch entries.  The kernels
// themselves are in fp8_attn_fwd.cu; the C ABI of include/fp8attn.h is in
// fp8attn_abi.cu.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstddef>
#include <cstdint>

namespace fp8attn {

constexpr int BM = 128;         // query rows per CTA (= MMA M, = TMEM lanes)
constexpr float LOG2E = 1.4426950408889634f;
// Smallest nonzero bound of a wait the caller may set (timeout_ns), and the
// fixed bound of the drain waits that let in-flight copies and MMAs land
// before an aborting CTA frees TMEM and exits.
constexpr unsigned long long MIN_TIMEOUT_NS = 1000000ull;
constexpr unsigned long long DRAIN_TIMEOUT_NS = 1000000000ull;

// device status codes (status_word): 0x100 | where the wait gave up
enum : uint32_t {
  WAIT_PROD_KV_EMPTY = 1,
  WAIT_MMA_Q = 2,
  WAIT_MMA_K = 3,
  WAIT_MMA_S_FREE = 4,
  WAIT_MMA_V = 5,
  WAIT_MMA_P = 6,
  WAIT_SM_S_FULL = 7,
  WAIT_SM_O_DONE = 8,
  WAIT_EPI_O_DONE = 9,
};

struct KParams {
  int B, H, Hkv, N, group;
  int causal, kv_order, n_sink;
  int tile0;          // first query tile of the launch (q_begin / 128)
  int num_q_tiles;    // query tiles in the launch
  int sched_group;    // plane units per causal scheduling group; divides their number
  int pair_heads;     // two-tile kernel: 1 = a CTA's tiles are one tile of two query
                      // heads of one kv head, 0 = two consecutive tiles of one head
  float scale_log2;   // scale * log2(e)
  // S*p: for S = 2^k, log2S = k and s_mul = 1, S*p is taken as 2^(s*c - m + k)
  // (exact scaling); otherwise log2S = 0 and S*p = fl(p * S) after the
  // exponential, the FP32 product the method casts.
  float log2S;
  float s_mul;
  void* O;
  unsigned long long* ctr;
  unsigned long long* ctr_sink;
  unsigned int* rows;
  unsigned int* status;
  unsigned long long timeout_ns;
  int debug_skip_kv_step;   // testing hook: 1-based KV step whose K load is never issued
  int denom_cast;           // row sum from the cast values (FP8ATTN_DENOM_CAST_P)
};

// Launch the attention forward for head dimension d (64 or 128) and KV block bn
// (64 or 128) over the grid (kp.num_q_tiles, kp.B * kp.H).  q, k, v: 3-D tensor
// maps of [planes, N, d] (E4M3, or BF16 for q and k when qk_bf16).
cudaError_t launch_attn(int d, int bn, bool o_bf16, bool count, bool qk_bf16,
                        const CUtensorMap& q, const CUtensorMap& k, const CUtensorMap& v,
                        const KParams& kp, cudaStream_t stream);

// The same operation with two query tiles per CTA and one CTA per SM
// (fp8_attn_fwd_pair.cu).  Grid: (row units, plane units): kp.pair_heads ?
// (num_q_tiles, B * H / 2) : (ceil(num_q_tiles / 2), B * H).
cudaError_t launch_attn_pair(int d, int bn, bool o_bf16, bool count, bool qk_bf16,
                             const CUtensorMap& q, const CUtensorMap& k, const CUtensorMap& v,
                             const KParams& kp, cudaStream_t stream);

// out[i] = E4M3_RNE_satfinite(fl32(S * P[i])), i < n (P, out 16-byte aligned).
cudaError_t launch_e4m3_scale_cast(const float* P, uint8_t* out, size_t n, float S,
                                   cudaStream_t stream);

}  // namespace fp8attn
