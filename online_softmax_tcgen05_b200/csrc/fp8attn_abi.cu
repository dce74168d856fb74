// fp8attn_abi.cu - the C ABI of include/fp8attn.h: argument validation (every
// check runs before any driver call or launch), the 3-D tensor maps of Q, K and
// V, the kernel's parameter block, status strings and the per-thread last
// error.  The kernels are in fp8_attn_fwd.cu (launch entries: attn_kernel.cuh).
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <atomic>
#include <cstring>
#include <mutex>
#include <string>

#include "abi_internal.h"
#include "attn_kernel.cuh"
#include "fp8attn.h"

namespace {
// fp8attn_set_schedule: the kernel that fp8_attn_fwd_ex launches
std::atomic<int> g_schedule{FP8ATTN_SCHEDULE_ONE_TILE};
}  // namespace

namespace fp8attn {

namespace {
thread_local std::string g_last_error;
}  // namespace

int fail(int status, const std::string& why) {
  g_last_error = why;
  return status;
}

void clear_error() { g_last_error.clear(); }

const char* last_error() { return g_last_error.c_str(); }

int validate(const fp8attn_params* p, bool host_buffers) {
  if (!p) return fail(FP8ATTN_EINVAL, "params is NULL");
  if (p->B < 0 || p->H < 0 || p->N < 0) return fail(FP8ATTN_EINVAL, "B, H, N must be >= 0");
  if (p->H_kv <= 0 && p->H > 0) return fail(FP8ATTN_EINVAL, "H_kv must be >= 1");
  if (p->H > 0 && p->H % p->H_kv) return fail(FP8ATTN_EINVAL, "H must be a multiple of H_kv");
  if (p->d != 64 && p->d != 128) return fail(FP8ATTN_EUNSUPPORTED, "d must be 64 or 128");
  const int bn = p->block_n == 0 ? 128 : p->block_n;
  if (bn != 64 && bn != 128) return fail(FP8ATTN_EUNSUPPORTED, "block_n must be 0, 64 or 128");
  if (p->causal != 0 && p->causal != 1) return fail(FP8ATTN_EINVAL, "causal must be 0 or 1");
  if (!std::isfinite(p->scale) || !(p->scale > 0.f))
    return fail(FP8ATTN_EINVAL, "scale must be finite and > 0");
  if (!std::isfinite(p->S) || !(p->S > 0.f)) return fail(FP8ATTN_EINVAL, "S must be finite and > 0");
  if (p->kv_order != FP8ATTN_KV_FORWARD && p->kv_order != FP8ATTN_KV_REVERSE)
    return fail(FP8ATTN_EINVAL, "kv_order must be 0 (forward) or 1 (reverse)");
  if (p->n_sink < 0 || p->n_sink > p->N) return fail(FP8ATTN_EINVAL, "n_sink must be in [0, N]");
  if (p->denominator != FP8ATTN_DENOM_FP32_P && p->denominator != FP8ATTN_DENOM_CAST_P)
    return fail(FP8ATTN_EINVAL, "denominator must be FP8ATTN_DENOM_FP32_P or FP8ATTN_DENOM_CAST_P");
  if (p->denominator == FP8ATTN_DENOM_CAST_P && std::isfinite(p->S) && p->S < 0x1p-8f)
    return fail(FP8ATTN_EINVAL, "the cast-value denominator needs S >= 2^-8");
  if (p->qk_dtype != FP8ATTN_QK_E4M3 && p->qk_dtype != FP8ATTN_QK_BF16)
    return fail(FP8ATTN_EINVAL, "qk_dtype must be FP8ATTN_QK_E4M3 or FP8ATTN_QK_BF16");
  if (p->o_dtype != FP8ATTN_O_BF16 && p->o_dtype != FP8ATTN_O_F32)
    return fail(FP8ATTN_EINVAL, "o_dtype must be FP8ATTN_O_BF16 or FP8ATTN_O_F32");
  if (p->timeout_ns != 0 && p->timeout_ns < MIN_TIMEOUT_NS)
    return fail(FP8ATTN_EINVAL, "timeout_ns must be 0 (the 2 s default) or at least 1 ms");
  if (p->debug_skip_kv_step < 0) return fail(FP8ATTN_EINVAL, "debug_skip_kv_step must be >= 0");
  if (p->debug_skip_kv_step > 0 && !p->status_word)
    return fail(FP8ATTN_EINVAL, "debug_skip_kv_step needs a status_word to report the timeout");
  if ((p->collapse_sink_ctr || p->collapse_rows) && !p->collapse_ctr)
    return fail(FP8ATTN_EINVAL, "collapse_sink_ctr / collapse_rows need collapse_ctr");
  const bool all_rows = p->q_begin == 0 && p->q_end == 0;
  if (!all_rows) {
    if (host_buffers)
      return fail(FP8ATTN_EINVAL, "the host-buffer entry computes all rows: q_begin = q_end = 0");
    if (p->q_begin < 0 || p->q_end > p->N || p->q_begin >= p->q_end)
      return fail(FP8ATTN_EINVAL, "q_begin, q_end must satisfy 0 <= q_begin < q_end <= N");
    if (p->q_begin % BM || (p->q_end % BM && p->q_end != p->N))
      return fail(FP8ATTN_EINVAL, "q_begin must be a multiple of 128, q_end a multiple of 128 or N");
  }
  if ((long long)p->B * p->H * p->N == 0) return 1;   // nothing to compute
  // grid: (query tiles, B*H); causal CTAs are numbered linearly in an int
  if ((long long)p->B * p->H > 65535) return fail(FP8ATTN_EINVAL, "B*H must be <= 65535");
  if ((long long)((p->N + BM - 1) / BM) * p->B * p->H > 0x7fffffffLL)
    return fail(FP8ATTN_EINVAL, "too many query tiles: ceil(N / 128) * B * H must be < 2^31");
  if (!p->Q || !p->K || !p->V || !p->O) return fail(FP8ATTN_EINVAL, "Q, K, V, O must be non-NULL");
  if (!host_buffers && (!aligned16(p->Q) || !aligned16(p->K) || !aligned16(p->V) ||
                        !aligned16(p->O)))
    return fail(FP8ATTN_EINVAL, "Q, K, V, O must be 16-byte aligned");
  if ((p->collapse_ctr && ((uintptr_t)p->collapse_ctr & 7)) ||
      (p->collapse_sink_ctr && ((uintptr_t)p->collapse_sink_ctr & 7)) ||
      (p->collapse_rows && ((uintptr_t)p->collapse_rows & 3)) ||
      (p->status_word && ((uintptr_t)p->status_word & 3)))
    return fail(FP8ATTN_EINVAL, "counter / status pointers must be naturally aligned");
  return 0;
}

}  // namespace fp8attn

namespace {

using fp8attn::aligned16;
using fp8attn::fail;

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  });
  return fn;
}

// 3-D map over a [planes, rows, d] tensor of E4M3 bytes (box [d, box_rows, 1],
// 128- or 64-byte swizzle by row length) or of BF16 (box [64, box_rows, 1]: one
// 128-byte swizzle atom per row; a row of d = 128 is loaded as two such panels).
bool make_map(CUtensorMap* m, const void* base, int d, int rows, int planes, int box_rows,
              bool bf16) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t esz = bf16 ? 2 : 1;
  cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)rows, (cuuint64_t)planes};
  cuuint64_t strides[2] = {(cuuint64_t)d * esz, (cuuint64_t)d * esz * (cuuint64_t)rows};
  cuuint32_t box[3] = {(cuuint32_t)(bf16 ? 64 : d), (cuuint32_t)box_rows, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUtensorMapSwizzle swz = (bf16 || d == 128) ? CU_TENSOR_MAP_SWIZZLE_128B
                                              : CU_TENSOR_MAP_SWIZZLE_64B;
  CUresult r = fn(m, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_UINT8, 3,
                  const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}


}  // namespace

extern "C" {

int fp8attn_version(void) { return 104; }

size_t fp8attn_params_sizeof(void) { return sizeof(fp8attn_params); }

const char* fp8attn_status_string(int status) {
  switch (status) {
    case FP8ATTN_OK: return "ok";
    case FP8ATTN_EINVAL: return "invalid argument";
    case FP8ATTN_EUNSUPPORTED: return "unsupported configuration";
    case FP8ATTN_ECUDA: return "CUDA error";
    case FP8ATTN_ETIMEOUT: return "bounded wait expired on the device";
    default: return "unknown status";
  }
}

const char* fp8attn_last_error(void) { return fp8attn::last_error(); }

int fp8attn_set_schedule(int schedule) {
  fp8attn::clear_error();
  if (schedule != FP8ATTN_SCHEDULE_ONE_TILE && schedule != FP8ATTN_SCHEDULE_TWO_TILES)
    return fail(FP8ATTN_EINVAL, "schedule must be FP8ATTN_SCHEDULE_ONE_TILE or _TWO_TILES");
  return g_schedule.exchange(schedule);
}

const char* fp8attn_device_status_string(unsigned int word) {
  if (word == 0) return "";
  switch (word & 0xFFu) {
    case fp8attn::WAIT_PROD_KV_EMPTY: return "timeout: producer waiting for a free K/V stage";
    case fp8attn::WAIT_MMA_Q: return "timeout: MMA waiting for the Q tile";
    case fp8attn::WAIT_MMA_K: return "timeout: MMA waiting for a K tile";
    case fp8attn::WAIT_MMA_S_FREE: return "timeout: MMA waiting for the S buffer";
    case fp8attn::WAIT_MMA_V: return "timeout: MMA waiting for a V tile";
    case fp8attn::WAIT_MMA_P: return "timeout: MMA waiting for the P~ tile";
    case fp8attn::WAIT_SM_S_FULL: return "timeout: softmax waiting for S";
    case fp8attn::WAIT_SM_O_DONE: return "timeout: softmax waiting for P~V";
    case fp8attn::WAIT_EPI_O_DONE: return "timeout: epilogue waiting for the last P~V";
    default: return "timeout: unknown wait";
  }
}

int fp8_attn_fwd_ex(const fp8attn_params* p, fp8attn_stream_t stream) {
  fp8attn::clear_error();
  const int v = fp8attn::validate(p, false);
  if (v < 0) return v;
  if (v == 1) return FP8ATTN_OK;   // nothing to compute
  const int bn = p->block_n == 0 ? 128 : p->block_n;

  CUtensorMap mq, mk, mv;
  if (!encode_fn()) return fail(FP8ATTN_ECUDA, "cuTensorMapEncodeTiled is not available");
  const bool qkb = p->qk_dtype == FP8ATTN_QK_BF16;
  if (!make_map(&mq, p->Q, p->d, p->N, p->B * p->H, fp8attn::BM, qkb) ||
      !make_map(&mk, p->K, p->d, p->N, p->B * p->H_kv, bn, qkb) ||
      !make_map(&mv, p->V, p->d, p->N, p->B * p->H_kv, bn, false))
    return fail(FP8ATTN_ECUDA, "cuTensorMapEncodeTiled failed");

  fp8attn::KParams kp;
  kp.B = p->B;
  kp.H = p->H;
  kp.Hkv = p->H_kv;
  kp.N = p->N;
  kp.group = p->H / p->H_kv;
  {
    // scheduling group: the query heads of as many KV heads as keep their K and V
    // (N * d bytes each, K in BF16 takes twice that) within 32 MiB, a quarter of
    // the L2 (measured: half the L2 lost 0.4% at N = 131072, where a group is one
    // KV head; the whole problem at once lost 4% there)
    const double kv_bytes = (double)p->N * p->d * (p->qk_dtype == FP8ATTN_QK_BF16 ? 3.0 : 2.0);
    const int nkv = p->B * p->H_kv;
    int kvg = (int)(32.0 * 1024.0 * 1024.0 / kv_bytes);
    kvg = kvg < 1 ? 1 : (kvg > nkv ? nkv : kvg);
    while (nkv % kvg) --kvg;
    kp.sched_group = kvg * kp.group;
  }
  // two-tile kernel: an even GQA group pairs two query heads of one kv head,
  // otherwise two consecutive tiles of one head; its scheduling groups count
  // plane units (head pairs or planes)
  kp.pair_heads = (kp.group % 2 == 0) ? 1 : 0;
  const bool use_pair = g_schedule.load(std::memory_order_relaxed) == FP8ATTN_SCHEDULE_TWO_TILES;
  if (use_pair && kp.pair_heads) kp.sched_group /= 2;
  kp.causal = p->causal;
  kp.kv_order = p->kv_order;
  kp.n_sink = p->n_sink;
  {
    const bool all_rows = p->q_begin == 0 && p->q_end == 0;
    const int r0 = all_rows ? 0 : p->q_begin, r1 = all_rows ? p->N : p->q_end;
    kp.tile0 = r0 / fp8attn::BM;
    kp.num_q_tiles = (r1 + fp8attn::BM - 1) / fp8attn::BM - kp.tile0;
  }
  kp.scale_log2 = p->scale * fp8attn::LOG2E;
  {
    // S = 2^k enters the exponent (exact scaling); any other S multiplies p
    int e2 = 0;
    const bool pow2 = std::frexp((double)p->S, &e2) == 0.5;
    kp.log2S = pow2 ? (float)(e2 - 1) : 0.f;
    kp.s_mul = pow2 ? 1.f : p->S;
  }
  kp.O = p->O;
  kp.ctr = p->collapse_ctr;
  kp.ctr_sink = p->collapse_sink_ctr;
  kp.rows = p->collapse_rows;
  kp.status = p->status_word;
  kp.timeout_ns = p->timeout_ns ? p->timeout_ns : 2000000000ull;
  kp.debug_skip_kv_step = p->debug_skip_kv_step;
  kp.denom_cast = p->denominator == FP8ATTN_DENOM_CAST_P;

  const bool bf16 = p->o_dtype == FP8ATTN_O_BF16;
  const bool count = p->collapse_ctr != nullptr;
  const bool qk_bf16 = p->qk_dtype == FP8ATTN_QK_BF16;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const cudaError_t e =
      use_pair ? fp8attn::launch_attn_pair(p->d, bn, bf16, count, qk_bf16, mq, mk, mv, kp, s)
               : fp8attn::launch_attn(p->d, bn, bf16, count, qk_bf16, mq, mk, mv, kp, s);
  if (e != cudaSuccess) return fail(FP8ATTN_ECUDA, std::string("launch: ") + cudaGetErrorString(e));
  return FP8ATTN_OK;
}

int fp8_attn_fwd(const void* Q, const void* K, const void* V, void* O, int B, int H, int N, int d,
                 int causal, float scale, float S, int kv_order, int n_sink,
                 unsigned long long* collapse_ctr, fp8attn_stream_t stream) {
  fp8attn_params p;
  std::memset(&p, 0, sizeof(p));
  p.Q = Q;
  p.K = K;
  p.V = V;
  p.O = O;
  p.B = B;
  p.H = H;
  p.H_kv = H;
  p.N = N;
  p.d = d;
  p.causal = causal;
  p.scale = scale;
  p.S = S;
  p.kv_order = kv_order;
  p.n_sink = n_sink;
  p.o_dtype = FP8ATTN_O_BF16;
  p.block_n = 128;
  p.collapse_ctr = collapse_ctr;
  return fp8_attn_fwd_ex(&p, stream);
}

int fp8_e4m3_scale_cast(const float* P, unsigned char* out, size_t n, float S,
                        fp8attn_stream_t stream) {
  fp8attn::clear_error();
  if (n == 0) return FP8ATTN_OK;
  if (!P || !out) return fail(FP8ATTN_EINVAL, "P and out must be non-NULL");
  if (!aligned16(P) || !aligned16(out)) return fail(FP8ATTN_EINVAL, "P and out must be 16-byte aligned");
  if (!std::isfinite(S)) return fail(FP8ATTN_EINVAL, "S must be finite");
  cudaError_t e = fp8attn::launch_e4m3_scale_cast(P, out, n, S,
                                                   reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return fail(FP8ATTN_ECUDA, std::string("launch: ") + cudaGetErrorString(e));
  return FP8ATTN_OK;
}

}  // extern "C"
