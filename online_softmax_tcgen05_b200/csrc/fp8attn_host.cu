// fp8attn_host.cu - the host-buffer entry of the C ABI (fp8_attn_fwd_host): the
// attention forward for Q, K, V and O in host memory, with the copies in and out
// pipelined against the kernels.
//
// The problem is cut into pieces of whole (batch, kv-head) units; a piece never
// crosses a batch element, so each of its Q, K, V and O slices is one contiguous
// range.  Per piece: K and V are copied in on the upload stream, Q per sub-step;
// the kernel of each sub-step runs on one of two compute streams taken in turn
// (so one piece's kernel fills the SMs the previous one's last wave leaves idle);
// each sub-step's O goes back on the download stream as soon as its kernel is
// done.  Three sets of staging buffers in the caller's workspace rotate over the
// pieces: a set is reused three pieces later, its upload waiting for that
// piece's download.  The first piece (whose upload overlaps no compute) and the
// last (whose download overlaps none), when they hold one kv head of several
// query heads, run one kernel per query head, so that each waits only for its
// own Q and returns its own O.
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>
#include <cstring>
#include <string>
#include <vector>

#include "abi_internal.h"
#include "fp8attn.h"

struct fp8attn_host_plan {
  int device = -1;
  cudaStream_t s_in = nullptr, s_out = nullptr, s_comp[2] = {nullptr, nullptr};
  cudaEvent_t ev_start = nullptr, ev_end = nullptr, ev_done = nullptr;
  cudaEvent_t ev_free[3] = {nullptr, nullptr, nullptr};   // staging set released
  bool free_recorded[3] = {false, false, false};
  std::vector<cudaEvent_t> ev_in;                          // per sub-step Q upload
};

namespace {

using fp8attn::fail;

constexpr int NSETS = 3;
constexpr size_t ALIGN = 256;

size_t round_up(size_t x) { return (x + ALIGN - 1) / ALIGN * ALIGN; }

struct Piece {
  int b, g0, g1;
};

std::vector<Piece> make_pieces(const fp8attn_params* p, int host_chunks) {
  const int units = p->B * p->H_kv;
  const int nchunk = std::max(1, std::min(host_chunks, units));
  std::vector<Piece> pieces;
  for (int c = 0; c < nchunk; ++c) {
    const int lo = (int)((long long)units * c / nchunk), hi = (int)((long long)units * (c + 1) / nchunk);
    int u = lo;
    while (u < hi) {
      const int b = u / p->H_kv;
      int e = u;
      while (e < hi && e / p->H_kv == b) ++e;
      pieces.push_back({b, u % p->H_kv, (e - 1) % p->H_kv + 1});
      u = e;
    }
  }
  return pieces;
}

struct Sizes {
  size_t qk_esz, o_esz, plane_qk, plane_v, plane_o;   // bytes per element / per (head) plane
  size_t q, k, v, o, set;                              // bytes per staging buffer / set
};

Sizes sizes(const fp8attn_params* p, int max_g) {
  Sizes z;
  const size_t nd = (size_t)p->N * p->d;
  const int group = p->H / p->H_kv;
  z.qk_esz = p->qk_dtype == FP8ATTN_QK_BF16 ? 2 : 1;
  z.o_esz = p->o_dtype == FP8ATTN_O_F32 ? 4 : 2;
  z.plane_qk = nd * z.qk_esz;
  z.plane_v = nd;
  z.plane_o = nd * z.o_esz;
  z.q = round_up((size_t)max_g * group * z.plane_qk);
  z.k = round_up((size_t)max_g * z.plane_qk);
  z.v = round_up((size_t)max_g * z.plane_v);
  z.o = round_up((size_t)max_g * group * z.plane_o);
  z.set = z.q + z.k + z.v + z.o;
  return z;
}

int max_piece(const std::vector<Piece>& pieces) {
  int m = 0;
  for (const Piece& pc : pieces) m = std::max(m, pc.g1 - pc.g0);
  return m;
}

int cuda_fail(cudaError_t e, const char* what) {
  return fail(FP8ATTN_ECUDA, std::string(what) + ": " + cudaGetErrorString(e));
}

// A failure after work was enqueued on the plan's streams: before returning
// `status`, order the caller's stream after everything those streams hold, so
// that a caller who frees the workspace or the host buffers once its stream
// has passed the call frees nothing a copy still uses.  Best effort: in a
// context that has itself failed these calls fail too.
int fail_joined(fp8attn_host_plan* pl, cudaStream_t caller, int status) {
  for (cudaStream_t s : {pl->s_in, pl->s_out, pl->s_comp[0], pl->s_comp[1]})
    if (cudaEventRecord(pl->ev_end, s) == cudaSuccess) cudaStreamWaitEvent(caller, pl->ev_end, 0);
  return status;
}

}  // namespace

extern "C" {

int fp8attn_host_plan_create(fp8attn_host_plan** plan) {
  fp8attn::clear_error();
  if (!plan) return fail(FP8ATTN_EINVAL, "plan is NULL");
  *plan = nullptr;
  fp8attn_host_plan* pl = new fp8attn_host_plan();
  cudaError_t e = cudaGetDevice(&pl->device);
  const unsigned sf = cudaStreamNonBlocking;
  const unsigned ef = cudaEventDisableTiming;
  if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&pl->s_in, sf);
  if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&pl->s_out, sf);
  if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&pl->s_comp[0], sf);
  if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&pl->s_comp[1], sf);
  if (e == cudaSuccess) e = cudaEventCreateWithFlags(&pl->ev_start, ef);
  if (e == cudaSuccess) e = cudaEventCreateWithFlags(&pl->ev_end, ef);
  if (e == cudaSuccess) e = cudaEventCreateWithFlags(&pl->ev_done, ef);
  for (int i = 0; i < NSETS && e == cudaSuccess; ++i) e = cudaEventCreateWithFlags(&pl->ev_free[i], ef);
  if (e != cudaSuccess) {
    fp8attn_host_plan_destroy(pl);
    return cuda_fail(e, "plan create");
  }
  *plan = pl;
  return FP8ATTN_OK;
}

int fp8attn_host_plan_destroy(fp8attn_host_plan* pl) {
  if (!pl) return FP8ATTN_OK;
  for (cudaStream_t s : {pl->s_in, pl->s_out, pl->s_comp[0], pl->s_comp[1]})
    if (s) {
      cudaStreamSynchronize(s);
      cudaStreamDestroy(s);
    }
  for (cudaEvent_t ev : {pl->ev_start, pl->ev_end, pl->ev_done, pl->ev_free[0], pl->ev_free[1],
                         pl->ev_free[2]})
    if (ev) cudaEventDestroy(ev);
  for (cudaEvent_t ev : pl->ev_in) cudaEventDestroy(ev);
  delete pl;
  return FP8ATTN_OK;
}

size_t fp8attn_host_workspace_bytes(const fp8attn_params* p, int host_chunks) {
  if (!p || p->B <= 0 || p->H <= 0 || p->H_kv <= 0 || p->N <= 0 || p->H % p->H_kv ||
      host_chunks < 1)
    return 0;
  const std::vector<Piece> pieces = make_pieces(p, host_chunks);
  return NSETS * sizes(p, max_piece(pieces)).set;
}

int fp8_attn_fwd_host(const fp8attn_params* p, fp8attn_host_plan* pl, void* workspace,
                      size_t workspace_bytes, int host_chunks, fp8attn_stream_t stream) {
  fp8attn::clear_error();
  const int v = fp8attn::validate(p, true);
  if (v < 0) return v;
  if (!pl) return fail(FP8ATTN_EINVAL, "plan is NULL");
  if (host_chunks < 1) return fail(FP8ATTN_EINVAL, "host_chunks must be >= 1");
  if (v == 1) return FP8ATTN_OK;   // nothing to compute
  const std::vector<Piece> pieces = make_pieces(p, host_chunks);
  const int max_g = max_piece(pieces);
  const Sizes z = sizes(p, max_g);
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) % ALIGN))
    return fail(FP8ATTN_EINVAL, "workspace must be non-NULL and 256-byte aligned");
  if (workspace_bytes < NSETS * z.set)
    return fail(FP8ATTN_EINVAL, "workspace too small: see fp8attn_host_workspace_bytes");
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev != pl->device) return fail(FP8ATTN_EINVAL, "the plan belongs to another device");
  const int group = p->H / p->H_kv;
  // every sub-step of a split piece needs its own upload event
  while ((int)pl->ev_in.size() < std::max(group, 1)) {
    cudaEvent_t ev;
    e = cudaEventCreateWithFlags(&ev, cudaEventDisableTiming);
    if (e != cudaSuccess) return cuda_fail(e, "cudaEventCreate");
    pl->ev_in.push_back(ev);
  }

  cudaStream_t caller = reinterpret_cast<cudaStream_t>(stream);
  const char* Qh = static_cast<const char*>(p->Q);
  const char* Kh = static_cast<const char*>(p->K);
  const char* Vh = static_cast<const char*>(p->V);
  char* Oh = static_cast<char*>(p->O);
  char* ws = static_cast<char*>(workspace);

  // everything below runs after the caller's earlier work on `stream`
  e = cudaEventRecord(pl->ev_start, caller);
  for (cudaStream_t s : {pl->s_in, pl->s_out, pl->s_comp[0], pl->s_comp[1]})
    if (e == cudaSuccess) e = cudaStreamWaitEvent(s, pl->ev_start, 0);
  if (e != cudaSuccess) return fail_joined(pl, caller, cuda_fail(e, "stream ordering"));

  int step = 0;
  const int np = (int)pieces.size();
  for (int i = 0; i < np; ++i) {
    const Piece& pc = pieces[i];
    const int nk = pc.g1 - pc.g0, nq = nk * group, hq = pc.g0 * group;
    const int set = i % NSETS;
    char* qd = ws + set * z.set;
    char* kd = qd + z.q;
    char* vd = kd + z.k;
    char* od = vd + z.v;
    const bool split = nk == 1 && group > 1 && np > 1 && (i == 0 || i == np - 1);
    const int nsub = split ? nq : 1;

    if (pl->free_recorded[set]) e = cudaStreamWaitEvent(pl->s_in, pl->ev_free[set], 0);
    const size_t kv_plane0 = (size_t)pc.b * p->H_kv + pc.g0;
    if (e == cudaSuccess)
      e = cudaMemcpyAsync(kd, Kh + kv_plane0 * z.plane_qk, nk * z.plane_qk,
                          cudaMemcpyHostToDevice, pl->s_in);
    if (e == cudaSuccess)
      e = cudaMemcpyAsync(vd, Vh + kv_plane0 * z.plane_v, nk * z.plane_v,
                          cudaMemcpyHostToDevice, pl->s_in);
    for (int j = 0; j < nsub && e == cudaSuccess; ++j) {
      const int a0 = split ? j : 0, a1 = split ? j + 1 : nq;
      const size_t q_plane0 = (size_t)pc.b * p->H + hq + a0;
      e = cudaMemcpyAsync(qd + a0 * z.plane_qk, Qh + q_plane0 * z.plane_qk,
                          (a1 - a0) * z.plane_qk, cudaMemcpyHostToDevice, pl->s_in);
      if (e == cudaSuccess) e = cudaEventRecord(pl->ev_in[j], pl->s_in);
    }
    if (e != cudaSuccess) return fail_joined(pl, caller, cuda_fail(e, "upload"));

    for (int j = 0; j < nsub; ++j) {
      const int a0 = split ? j : 0, a1 = split ? j + 1 : nq;
      cudaStream_t comp = pl->s_comp[step++ % 2];
      e = cudaStreamWaitEvent(comp, pl->ev_in[j], 0);
      if (e != cudaSuccess) return fail_joined(pl, caller, cuda_fail(e, "stream ordering"));
      const size_t q_plane0 = (size_t)pc.b * p->H + hq + a0;
      fp8attn_params sub = *p;
      sub.Q = qd + a0 * z.plane_qk;
      sub.K = kd;
      sub.V = vd;
      sub.O = od + a0 * z.plane_o;
      sub.B = 1;
      sub.H = a1 - a0;
      sub.H_kv = nk;
      sub.collapse_rows = p->collapse_rows ? p->collapse_rows + q_plane0 * p->N : nullptr;
      const int st = fp8_attn_fwd_ex(&sub, comp);
      if (st != FP8ATTN_OK) return fail_joined(pl, caller, st);   // last error set by the launch
      e = cudaEventRecord(pl->ev_done, comp);
      if (e == cudaSuccess) e = cudaStreamWaitEvent(pl->s_out, pl->ev_done, 0);
      if (e == cudaSuccess)
        e = cudaMemcpyAsync(Oh + q_plane0 * z.plane_o, od + a0 * z.plane_o,
                            (a1 - a0) * z.plane_o, cudaMemcpyDeviceToHost, pl->s_out);
      if (e != cudaSuccess) return fail_joined(pl, caller, cuda_fail(e, "download"));
    }
    e = cudaEventRecord(pl->ev_free[set], pl->s_out);
    if (e != cudaSuccess) return fail_joined(pl, caller, cuda_fail(e, "cudaEventRecord"));
    pl->free_recorded[set] = true;
  }
  // the caller's stream continues after the last download (and so after every kernel)
  e = cudaEventRecord(pl->ev_end, pl->s_out);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(caller, pl->ev_end, 0);
  if (e != cudaSuccess) return fail_joined(pl, caller, cuda_fail(e, "stream ordering"));
  return FP8ATTN_OK;
}

}  // extern "C"
