// fp8attn_host_noalloc.cu - fp8_attn_fwd_host_noalloc: the attention forward
// for Q, K, V and O in host memory, staged through a fixed device array that
// the library itself holds, so that the call allocates no memory at all.
//
// Who needs it: code that may not allocate device memory once it is running.
// Examples are a plugin inside a host application whose allocator owns the
// whole device, a serving loop that forbids allocation after start-up, and a
// caller with no CUDA allocator of its own (a C program that links only this
// library and a CUDA runtime it does not manage).  fp8_attn_fwd_host needs a
// caller-provided device workspace and a plan of streams and events; this
// entry needs neither.
//
// How: the staging buffers of Q, K, V and O live in g_staging, a file-scope
// __device__ array of FP8ATTN_HOST_NOALLOC_BYTES.  The problem is cut into
// pieces of whole (batch, kv-head) units, as many kv heads of one batch
// element per piece as fit the array.  Each piece runs on the caller's stream
// in order: its K, V and Q are copied in, the attention kernel runs on the
// staged copies, its O is copied back.  One stream, one staging set, so the
// copies do not overlap the kernels (fp8_attn_fwd_host pipelines them).
//
// In host code g_staging names a host-side stand-in, not device memory: the
// kernels and copies get its device address, which cudaGetSymbolAddress gives
// once per device (the first call on that device, with the device current).
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>
#include <mutex>
#include <string>

#include "abi_internal.h"
#include "fp8attn.h"

// The staging array.  Every GPU that loads this module holds it until the
// process exits.  Every call shares it and it keeps the last call's contents;
// a call writes every staged byte it reads before reading it, so nothing has
// to be cleared.
static __device__ __align__(256) unsigned char g_staging[FP8ATTN_HOST_NOALLOC_BYTES];

namespace {

using fp8attn::fail;

constexpr size_t kStagingBytes = FP8ATTN_HOST_NOALLOC_BYTES;
constexpr size_t kAlign = 256;
constexpr int kMaxDevices = 64;

std::mutex g_setup_mu;
void* g_staging_addr[kMaxDevices] = {};   // device address of g_staging per device

size_t round_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

int cuda_fail(cudaError_t e, const char* what) {
  return fail(FP8ATTN_ECUDA, std::string(what) + ": " + cudaGetErrorString(e));
}

// Device address of g_staging on the current device (set up on first use).
int staging_address(void** out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices)
    return fail(FP8ATTN_EUNSUPPORTED, "device ordinal beyond the static staging table");
  std::lock_guard<std::mutex> lock(g_setup_mu);
  if (!g_staging_addr[dev]) {
    void* ptr = nullptr;
    e = cudaGetSymbolAddress(&ptr, g_staging);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(staging array)");
    g_staging_addr[dev] = ptr;
  }
  *out = g_staging_addr[dev];
  return FP8ATTN_OK;
}

}  // namespace

extern "C" {

int fp8_attn_fwd_host_noalloc(const fp8attn_params* p, fp8attn_stream_t stream) {
  fp8attn::clear_error();
  const int v = fp8attn::validate(p, true);
  if (v < 0) return v;
  if (v == 1) return FP8ATTN_OK;   // nothing to compute

  const int group = p->H / p->H_kv;
  const size_t nd = (size_t)p->N * p->d;
  const size_t qk_esz = p->qk_dtype == FP8ATTN_QK_BF16 ? 2 : 1;
  const size_t o_esz = p->o_dtype == FP8ATTN_O_F32 ? 4 : 2;
  const size_t plane_qk = nd * qk_esz, plane_v = nd, plane_o = nd * o_esz;
  // staging bytes of a piece of g kv heads: Q and O of its g * group query
  // heads, K and V of its g kv heads, each buffer 256-byte aligned
  auto piece_bytes = [&](size_t g) {
    return round_up(g * group * plane_qk) + round_up(g * plane_qk) + round_up(g * plane_v) +
           round_up(g * group * plane_o);
  };
  if (piece_bytes(1) > kStagingBytes)
    return fail(FP8ATTN_EINVAL,
                "one kv head needs " + std::to_string(piece_bytes(1)) +
                    " staging bytes, more than the " + std::to_string(kStagingBytes) +
                    "-byte static array of fp8_attn_fwd_host_noalloc; use fp8_attn_fwd_host "
                    "with a caller workspace");
  size_t per = 1;   // kv heads per piece: the most that fit, within one batch element
  while (per < (size_t)p->H_kv && piece_bytes(per + 1) <= kStagingBytes) ++per;

  void* base = nullptr;
  const int st = staging_address(&base);
  if (st != FP8ATTN_OK) return st;
  char* qd = static_cast<char*>(base);
  char* kd = qd + round_up(per * group * plane_qk);
  char* vd = kd + round_up(per * plane_qk);
  char* od = vd + round_up(per * plane_v);

  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const char* Qh = static_cast<const char*>(p->Q);
  const char* Kh = static_cast<const char*>(p->K);
  const char* Vh = static_cast<const char*>(p->V);
  char* Oh = static_cast<char*>(p->O);
  for (int b = 0; b < p->B; ++b) {
    for (int g0 = 0; g0 < p->H_kv; g0 += (int)per) {
      const int nk = std::min((int)per, p->H_kv - g0), nq = nk * group;
      const size_t kv_plane0 = (size_t)b * p->H_kv + g0;
      const size_t q_plane0 = (size_t)b * p->H + (size_t)g0 * group;
      cudaError_t e = cudaMemcpyAsync(kd, Kh + kv_plane0 * plane_qk, nk * plane_qk,
                                      cudaMemcpyHostToDevice, s);
      if (e == cudaSuccess)
        e = cudaMemcpyAsync(vd, Vh + kv_plane0 * plane_v, nk * plane_v, cudaMemcpyHostToDevice, s);
      if (e == cudaSuccess)
        e = cudaMemcpyAsync(qd, Qh + q_plane0 * plane_qk, nq * plane_qk, cudaMemcpyHostToDevice,
                            s);
      if (e != cudaSuccess) return cuda_fail(e, "upload");
      fp8attn_params sub = *p;
      sub.Q = qd;
      sub.K = kd;
      sub.V = vd;
      sub.O = od;
      sub.B = 1;
      sub.H = nq;
      sub.H_kv = nk;
      sub.collapse_rows = p->collapse_rows ? p->collapse_rows + q_plane0 * p->N : nullptr;
      const int r = fp8_attn_fwd_ex(&sub, stream);
      if (r != FP8ATTN_OK) return r;   // last error set by the launch
      e = cudaMemcpyAsync(Oh + q_plane0 * plane_o, od, nq * plane_o, cudaMemcpyDeviceToHost, s);
      if (e != cudaSuccess) return cuda_fail(e, "download");
    }
  }
  return FP8ATTN_OK;
}

}  // extern "C"
