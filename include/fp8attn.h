/* fp8attn.h - C ABI of the B200 (sm_100a) FP8 attention forward with P-cast
 * scale S and selectable KV-block order.
 *
 * What the operation is (P-Cast Precision in FP8 Attention: Sink-Induced
 * Collapse and the Optimality of S=2^8, arXiv 2606.06521, gist.science
 * summary, section 1 "Problem statement"): a FlashAttention-style forward
 * pass on E4M3 operands whose online softmax keeps a running row max m,
 * multiplies each probability tile P by a static scale S, casts S*P to E4M3
 * for the P.V product, and divides S back out in the epilogue.  The order in
 * which the online softmax visits the KV blocks (forward 0..N or reverse N..0)
 * is a run-time choice; section 2 "Optimisation 1" shows that the reverse order
 * keeps the attention sink from inflating m before the other blocks are cast.
 * "P-collapse" (section 1) is a non-sink P that is nonzero in FP32 but 0 after
 * the cast; the kernel can count it.  What the kernel counts: every visible
 * non-sink key (j >= n_sink, and j <= i when causal) whose E4M3 byte of S*p is
 * zero.  That equals "p_j > 0 in FP32 and zero after the cast" except where the
 * FP32 p_j itself is 0 (s_j - m' below about -87 nats, where ex2 flushes to
 * zero): such a key is counted here although its FP32 value is not nonzero.
 *
 * Per query row i (query head h, kv head h / (H / H_kv)):
 *   for each KV block of block_n keys, in the chosen order:
 *     s_j  = scale * q_i . k_j        (FP32 accumulate of E4M3 products)
 *     m'   = max(m, max_j s_j),  alpha = exp(m - m')
 *     p_j  = exp(s_j - m')            (FP32)
 *     l    = alpha * l + sum_j p_j    (row sum from the FP32 P, before the cast)
 *     pt_j = E4M3_RNE_satfinite(S * p_j)
 *     acc  = alpha * acc + sum_j pt_j v_j   (E4M3 x E4M3, FP32 accumulate)
 *     m    = m'
 *   O_i = acc / (S * l)
 * For S a power of two the kernel takes S * p_j directly from its exponential,
 * 2^(log2 e * (s_j - m') + log2 S), and sums those, so S divides out with l:
 * the same real numbers, exact scaling.  For any other S it forms the FP32
 * product fl(S * p_j) that is cast, sums the p_j, and divides by fl(S * l).
 * Causal: key j is visible to query i iff j <= i (square prefill, no offset).
 * NaN inputs: a NaN byte in Q or K makes every O row that sees it NaN (the row
 * maximum keeps NaN, so all of that row's exponentials are NaN from that block
 * on); rows that do not see it are unaffected.
 *
 * Conventions for every entry point:
 *   - Tensor pointers are DEVICE pointers owned by the caller (except Q, K, V, O
 *     of fp8_attn_fwd_host, which are host memory).  The library never frees or
 *     retains them and allocates no device memory.
 *   - All work is enqueued asynchronously on `stream` (NULL = legacy default
 *     stream).  A return of FP8ATTN_OK means "validated and launched".
 *   - Arguments are validated on the host before anything is launched; an
 *     invalid call returns a negative status and touches no device memory.
 *     fp8attn_last_error() then gives a one-line reason (per host thread).
 *   - E4M3 means the OCP FP8 E4M3 ("fn") byte encoding, one byte per element.
 */
#ifndef FP8ATTN_H
#define FP8ATTN_H

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t / CUstream. */
typedef struct CUstream_st* fp8attn_stream_t;

typedef enum {
  FP8ATTN_OK = 0,
  FP8ATTN_EINVAL = -1,        /* an argument is out of range or misaligned */
  FP8ATTN_EUNSUPPORTED = -2,  /* a valid request this build does not serve (d, block_n) */
  FP8ATTN_ECUDA = -3,         /* a CUDA runtime / driver call failed */
  FP8ATTN_ETIMEOUT = -4       /* reported through status_word: a bounded wait expired */
} fp8attn_status;

enum { FP8ATTN_KV_FORWARD = 0, FP8ATTN_KV_REVERSE = 1 };
enum { FP8ATTN_O_BF16 = 0, FP8ATTN_O_F32 = 1 };
/* Q and K element type.  E4M3 (default): QK^T on E4M3 operands.  BF16: Q and K
 * are BF16 [.., d] rows and QK^T runs on BF16 operands, with P~ and V still
 * E4M3 -- the P-cast paper's "kernel-faithful" simulation (Contributions 4),
 * which leaves Q, K, V unquantised so that only the P-cast error remains. */
enum { FP8ATTN_QK_E4M3 = 0, FP8ATTN_QK_BF16 = 1 };
/* Row-sum (denominator) source.  FP32_P: l from the FP32 P before the cast and
 * O = acc / (S l) (the P-cast paper's kernel).  CAST_P: l from the cast values,
 * l = sum_j dec(pt_j), and O = acc / l, so numerator and denominator use the same
 * quantised operand (the choice EFQ-Softmax makes). */
enum { FP8ATTN_DENOM_FP32_P = 0, FP8ATTN_DENOM_CAST_P = 1 };

/* fp8_attn_fwd - the attention forward above, square self-attention, H_kv = H,
 * O in BF16, KV block 128.
 *
 *   Q, K, V   E4M3 [B, H, N, d] contiguous (d fastest), 16-byte aligned.
 *   O         BF16 [B, H, N, d] contiguous, 16-byte aligned (written).
 *   B, H, N   batch, heads, sequence length; B*H*N == 0 is a no-op.
 *   d         head dimension, 64 or 128.
 *   causal    0 or 1.
 *   scale     softmax scale (finite, > 0), usually 1/sqrt(d).
 *   S         P-cast scale (finite, > 0).  S > 448 is accepted: S*P then
 *             saturates at 448 (the overflow the paper warns of for 512).
 *   kv_order  FP8ATTN_KV_FORWARD or FP8ATTN_KV_REVERSE.
 *   n_sink    keys j < n_sink are sinks and are never counted (0 <= n_sink <= N).
 *   collapse_ctr  NULL: no counting (the faster kernel variant).  Otherwise a
 *             device uint64 that the kernel ADDS the number of collapsed
 *             entries to (the caller zeroes it): visible non-sink keys whose
 *             E4M3 byte of S*p is zero (see "What the kernel counts" above).
 * Returns an fp8attn_status. */
int fp8_attn_fwd(const void* Q, const void* K, const void* V, void* O,
                 int B, int H, int N, int d, int causal, float scale, float S,
                 int kv_order, int n_sink, unsigned long long* collapse_ctr,
                 fp8attn_stream_t stream);

/* Full parameter set (same operation; see fp8_attn_fwd for shared fields). */
typedef struct {
  const void* Q;          /* [B, H,    N, d], E4M3 or BF16 (qk_dtype) */
  const void* K;          /* [B, H_kv, N, d], E4M3 or BF16 (qk_dtype) */
  const void* V;          /* E4M3 [B, H_kv, N, d] */
  void* O;                /* [B, H, N, d], dtype o_dtype */
  int B, H, H_kv, N, d;   /* H % H_kv == 0; query head h reads kv head h / (H / H_kv) */
  int causal;
  float scale, S;
  int kv_order, n_sink;
  int o_dtype;            /* FP8ATTN_O_BF16 (RNE) or FP8ATTN_O_F32 */
  int block_n;            /* KV block: 0 (= 128), 64 or 128.  N need not be a multiple:
                             the last block then holds the remaining keys. */
  int qk_dtype;           /* FP8ATTN_QK_E4M3 (default, 0) or FP8ATTN_QK_BF16 */
  int denominator;        /* FP8ATTN_DENOM_FP32_P (default, 0) or FP8ATTN_DENOM_CAST_P;
                             CAST_P needs S >= 2^-8 so that the row maximum's cast is
                             nonzero */
  unsigned long long* collapse_ctr;      /* nullable; += all collapsed entries */
  unsigned long long* collapse_sink_ctr; /* nullable; += those in KV blocks holding a
                                            sink key (requires collapse_ctr) */
  unsigned int* collapse_rows;           /* nullable; [B, H, N] per-row counts, written
                                            (requires collapse_ctr) */
  unsigned int* status_word;             /* nullable device word; a kernel whose bounded
                                            wait expires writes a nonzero code here and
                                            leaves O incomplete */
  unsigned long long timeout_ns;         /* bound of each wait: 0 = 2 s, otherwise at
                                            least 1 ms (1000000); smaller values are
                                            rejected.  After an expired wait the CTA
                                            still waits up to 1 s for its own copies
                                            and MMAs in flight before it exits. */
  int debug_skip_kv_step;                /* testing only, normally 0.  k > 0: the producer
                                            never issues the K tile of the k-th KV step
                                            (1-based), so the MMA warp's bounded wait runs
                                            out, status_word records it and the launch ends
                                            with O incomplete */
  int q_begin, q_end;     /* query rows [q_begin, q_end) of every (batch, head) plane are
                             computed; O rows, per-row counts and collapse counts of the
                             other rows are left untouched.  q_begin = q_end = 0 selects
                             all N rows.  Otherwise 0 <= q_begin < q_end <= N, q_begin a
                             multiple of 128 (the query tile), q_end a multiple of 128 or
                             N.  Causal rows see keys 0 .. row whatever the range, so a
                             problem can be computed as several launches over disjoint
                             ranges (short causal tiles last, for instance). */
} fp8attn_params;

int fp8_attn_fwd_ex(const fp8attn_params* p, fp8attn_stream_t stream);

/* fp8_e4m3_scale_cast - out[i] = E4M3_RNE_satfinite(fl32(S * P[i])) for i < n:
 * one FP32 multiply, then the conversion instruction (cvt.rn.satfinite.e4m3x2)
 * that the attention kernel applies to S*p (P-cast paper, section 2
 * "Optimality of S=256": the scaling happens in FP32, then the round-to-nearest
 * cast).  For S not a power of two the attention kernel forms S*p by the same
 * FP32 multiply; for S = 2^k it takes S*p from its exponential and never forms
 * the product, which for finite p without over- or underflow is the same value.  P: device float[n]; out: device uint8[n];
 * both 16-byte aligned.  S finite (any sign).  NaN -> 0x7F, |x| > 448 -> +-448. */
int fp8_e4m3_scale_cast(const float* P, unsigned char* out, size_t n, float S,
                        fp8attn_stream_t stream);

/* ---------------------------------------------------- host-buffer entry ---
 * fp8_attn_fwd_host - the same operation for Q, K, V and O in HOST memory:
 * the copies to and from the device run inside the call's stream work,
 * pipelined against the kernels.
 *
 * The problem is cut into up to host_chunks pieces of whole (batch, kv-head)
 * units, none crossing a batch element.  Each piece's K and V (and Q, per
 * sub-step) are copied into one of three staging sets in `workspace`, its
 * kernels run on two compute streams taken in turn, and each sub-step's O is
 * copied back as soon as its kernel is done.  The first and last pieces, when
 * they hold one kv head of several query heads, run one kernel per query head.
 *
 *   p            as for fp8_attn_fwd_ex, but Q, K, V, O are HOST pointers:
 *                page-locked memory lets the copies overlap the kernels
 *                (pageable memory works, with the copies serialised).
 *                collapse_ctr, collapse_sink_ctr, collapse_rows and status_word
 *                stay DEVICE pointers.  q_begin = q_end = 0 (all rows).
 *   plan         from fp8attn_host_plan_create on the current device.
 *   workspace    DEVICE memory, 256-byte aligned, of at least
 *                fp8attn_host_workspace_bytes(p, host_chunks) bytes, owned by
 *                the caller; not to be reused before `stream` has passed this call.
 *   host_chunks  >= 1; the number of pieces (at most B * H_kv).
 *   stream       the work starts after prior work on `stream`, and `stream` is
 *                ordered after the last copy back: synchronise it before reading
 *                O or the counters.
 * Returns an fp8attn_status.  A failure after work was enqueued (FP8ATTN_ECUDA)
 * leaves O incomplete; `stream` is still ordered after all work the call
 * enqueued (unless the CUDA context itself has failed), so the workspace and
 * the host buffers may be released once `stream` has passed the call. */
typedef struct fp8attn_host_plan fp8attn_host_plan;   /* opaque */

/* Streams and events of the host pipeline, on the current device.  A plan
 * serves one call at a time (not for concurrent use from several threads) and
 * may be reused by any number of calls. */
int fp8attn_host_plan_create(fp8attn_host_plan** plan);

/* Waits for the plan's streams, then releases them.  NULL is a no-op. */
int fp8attn_host_plan_destroy(fp8attn_host_plan* plan);

/* Device workspace bytes that fp8_attn_fwd_host needs for p and host_chunks
 * (0 for an empty or invalid shape). */
size_t fp8attn_host_workspace_bytes(const fp8attn_params* p, int host_chunks);

int fp8_attn_fwd_host(const fp8attn_params* p, fp8attn_host_plan* plan, void* workspace,
                      size_t workspace_bytes, int host_chunks, fp8attn_stream_t stream);

/* ------------------------------------------ host-buffer entry, no allocation ---
 * fp8_attn_fwd_host_noalloc - the same operation as fp8_attn_fwd_host for a
 * caller that cannot allocate device memory: code running where another
 * allocator owns the whole device (a plugin inside a host application, a
 * framework that reserves all of HBM up front), a serving loop whose rules
 * forbid allocation after start-up, or a plain C caller with no CUDA allocator
 * of its own.  It takes no workspace and no plan and calls no allocating
 * routine (no cudaMalloc, cudaFree, stream or event creation).  The P-cast
 * paper has no counterpart: this is a deployment convenience of the library.
 *
 * Staging goes through one array of FP8ATTN_HOST_NOALLOC_BYTES bytes of device
 * memory that the library holds as a static device variable: every GPU that
 * loads the library's module holds it until the process exits.  The problem is
 * cut into pieces of whole (batch, kv-head) units, as many kv heads of one
 * batch element as fit the array; each piece's copies in, its kernel and its
 * copy back run in order on `stream` (no overlap of copies and kernels; the
 * pipelined fp8_attn_fwd_host is the fast path).
 *
 *   p       as for fp8_attn_fwd_host: Q, K, V, O are HOST pointers; the
 *           collapse counters, per-row counts and status word stay DEVICE
 *           pointers; q_begin = q_end = 0.
 *   stream  the call's work runs in order on it, after prior work; synchronise
 *           it before reading O or the counters.
 * Returns an fp8attn_status.  FP8ATTN_EINVAL, with fp8attn_last_error() giving
 * the sizes, when one kv head's Q, K, V and O (H / H_kv query heads) need more
 * than FP8ATTN_HOST_NOALLOC_BYTES of staging, rounded up to 256 bytes per buffer.
 *
 * The first call on a device, with that device current, looks up the array's
 * device address (cudaGetSymbolAddress); make that first call before any stream
 * capture.  All calls share the one array, which keeps the last call's contents
 * (a call reads only staging bytes it wrote first, so nothing needs clearing).
 * Calls that overlap on the GPU (different streams, or several host threads
 * without ordering between their streams) race on it: order them, for instance
 * by issuing them all on one stream. */
#define FP8ATTN_HOST_NOALLOC_BYTES ((size_t)64 << 20)

int fp8_attn_fwd_host_noalloc(const fp8attn_params* p, fp8attn_stream_t stream);

/* Kernel schedule of the device-buffer entries (and of the host-buffer entries,
 * which call them).  Both compute the same operation, in the same order per
 * row and with the same results:
 *   FP8ATTN_SCHEDULE_ONE_TILE   one 128-row query tile per CTA, two CTAs per SM,
 *                               whose softmax phases overlap by chance (default);
 *   FP8ATTN_SCHEDULE_TWO_TILES  two query tiles per CTA that share one K/V
 *                               stream (two heads of one kv head, or two
 *                               consecutive tiles), one CTA per SM, the two
 *                               tiles' softmax warps on each SM sub-partition
 *                               taking turns on the exponential unit.
 * Process-wide; returns the previous schedule, or FP8ATTN_EINVAL for an unknown
 * value (nothing changed).  Calls already enqueued keep their schedule. */
enum { FP8ATTN_SCHEDULE_ONE_TILE = 0, FP8ATTN_SCHEDULE_TWO_TILES = 1 };
int fp8attn_set_schedule(int schedule);

/* Human-readable name of a status code (static string). */
const char* fp8attn_status_string(int status);

/* Reason for the last non-OK return on this host thread ("" if none). */
const char* fp8attn_last_error(void);

/* Decoded device status word value ("" for 0). */
const char* fp8attn_device_status_string(unsigned int word);

/* ABI version of this header (major * 100 + minor). */
int fp8attn_version(void);

/* sizeof(fp8attn_params) as compiled into the library (binding layout check). */
size_t fp8attn_params_sizeof(void);

#ifdef __cplusplus
}
#endif

#endif /* FP8ATTN_H */
