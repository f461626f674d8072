/*
 * attn.h -- C ABI of the B200 (sm_100a) exact-attention library (libattn.so).
 *
 * The library computes exact dense scaled-dot-product attention
 *
 *     O = softmax((Q K^T + M) * scale) V
 *
 * ("FlashAttention and long context: three ledgers", section on why standard
 * attention is not only a FLOP problem) tile by tile with the online softmax of
 * the same page ("the key of FlashAttention is online softmax"), so the
 * L_q x L_k score and probability matrices never reach device memory.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * - Element types: bf16 tensors are passed as `attn_bf16_t` (the raw 16-bit
 *   bfloat16 pattern); statistics are IEEE fp32.
 * - Layout: every tensor is contiguous row-major [batch, heads, length, d]
 *   (the [batch, heads, n, d] layout of the FlashAttention-2 tutorial, 2.1.1).
 *   Q, O, dO, dQ: [B, Hq, Lq, d]; K, V, dK, dV: [B, Hkv, Lk, d];
 *   LSE: [B, Hq, Lq] fp32.  Query head h reads key/value head h / (Hq / Hkv)
 *   (grouped-query attention; Hq must be a multiple of Hkv).
 * - d (head dimension) must be 64 or 128 (the 8-bit forward: 128); anything
 *   else returns ATTN_ERR_UNSUPPORTED.  There is no fallback path of any kind.
 * - All device pointers must be 16-byte aligned (the tensor-memory-accelerator
 *   copies require it) and must not alias one another (except where stated).
 * - Masks: `mask_flags` = ATTN_MASK_NONE or ATTN_MASK_CAUSAL.  Causal is
 *   bottom-right aligned: key j is visible to query i iff j <= i + (Lk - Lq).
 *   Key padding is selected by passing `k_lens` (device int32 [B]): key j of
 *   sequence b is visible iff j < k_lens[b].  Both combine by AND.  A query row
 *   with no visible key gets O = 0, LSE = -inf and zero gradients.
 * - LSE is the natural-log log-sum-exp of the row's scaled, masked scores: the
 *   per-row statistic the backward recomputes from (the three-ledgers page,
 *   online-softmax section: the backward keeps small row statistics and
 *   recomputes score blocks).
 * - Ownership: the caller allocates and owns every buffer, including the
 *   workspace, and the stream.  The library never allocates, frees or
 *   synchronises, except attn_read_device_status (which synchronises `stream`).
 * - Asynchrony: every compute call enqueues kernels on `stream` (a
 *   cudaStream_t; NULL = legacy default stream) and returns at once.
 * - Errors: argument errors are detected on the host before anything is
 *   launched and return ATTN_ERR_INVALID or ATTN_ERR_UNSUPPORTED.  A failed
 *   launch returns ATTN_ERR_CUDA.  Errors found on the device (a k_lens entry
 *   outside [0, Lk], a paged-cache block-table entry outside [0, n_pages), a
 *   malformed packed-sequence offset, an 8-bit scale that is not finite and
 *   positive, an internal wait that timed out) set bits of a status word kept
 *   in the first 16 bytes of the workspace; the affected work units write
 *   zeros (a bad 8-bit scale leaves its results undefined instead).  The word is sticky: read it with attn_read_device_status and
 *   clear it with attn_clear_device_status (a fresh workspace must be cleared
 *   once before first use).
 * - Workspace: each call has an *_workspace_size query; pass at least that
 *   many bytes, 256-byte aligned.  Calls that overlap in time on the device
 *   must not share a workspace.
 */
#ifndef ATTN_H_
#define ATTN_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef uint16_t attn_bf16_t;

typedef enum {
  ATTN_OK = 0,
  ATTN_ERR_INVALID = 1,     /* bad pointer, size, alignment, or workspace too small */
  ATTN_ERR_UNSUPPORTED = 2, /* valid request outside what the kernels implement */
  ATTN_ERR_CUDA = 3,        /* a CUDA runtime/driver call or launch failed */
  ATTN_ERR_TIMEOUT = 4,     /* (device status) a bounded internal wait expired */
  ATTN_ERR_CAPACITY = 5     /* request needs more than the fixed scratch of a no-alloc call */
} attn_status_t;

enum { ATTN_MASK_NONE = 0, ATTN_MASK_CAUSAL = 1 };

/* Device status bits (first int32 of every workspace). */
enum { ATTN_DEV_BAD_KLEN = 1, ATTN_DEV_TIMEOUT = 2, ATTN_DEV_BAD_PAGE = 4, ATTN_DEV_BAD_SCALE = 8 };

/* Human-readable name of a status code (static string, never NULL). */
const char* attn_status_string(attn_status_t s);

/* ------------------------------------------------------------------ forward
 * Prefill / training forward.  Defined by the attention formula and the online
 * softmax of the three-ledgers page (m' = max(m, max S_j); l' = e^{m-m'} l + sum e^{S_j-m'};
 * o' = e^{m-m'} o + sum e^{S_j-m'} V_j; O = o / l), with the tiling of the
 * FlashAttention-2 tutorial, 2.1.2.
 *
 *   Q [B,Hq,Lq,d], K/V [B,Hkv,Lk,d] bf16 (read only); O [B,Hq,Lq,d] bf16 and
 *   lse [B,Hq,Lq] fp32 (written; lse may be NULL when not needed).
 *   scale: multiplies Q K^T (the pages use 1/sqrt(d)); must be finite and > 0.
 *   k_lens: device int32 [B] or NULL (no padding).
 *   Lq, Lk >= 0 (Lq == 0 is a no-op).  B, Hq, Hkv >= 1.
 */
size_t attn_fwd_workspace_size(int B, int Hq, int Hkv, int Lq, int Lk, int d);
attn_status_t attn_fwd(const attn_bf16_t* Q, const attn_bf16_t* K, const attn_bf16_t* V,
                       attn_bf16_t* O, float* lse, int B, int Hq, int Hkv, int Lq, int Lk,
                       int d, float scale, int mask_flags, const int32_t* k_lens,
                       void* workspace, size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------ 8-bit forward
 * The forward of attn_fwd on 8-bit inputs: the low-precision execution that the
 * "FlashAttention" blog (section 10, FlashAttention-3) names, with Q, K and V as
 * E4M3 floats (OCP 8-bit format: 1 sign, 4 exponent bits with bias 7, 3
 * mantissa bits, max 448, no infinities) and one fp32 scale per 128-row tile of
 * each head.  The attention computed is that of the dequantised tensors
 *   Q[b,h,i,:] = Q8[b,h,i,:] * q_scale[b,h,i/128]   (K and V likewise),
 * with S = Q K^T on the 8-bit tensor cores (exact products, fp32 sums) and the
 * probabilities rounded to E4M3 for O += P V; the softmax statistics, O and
 * LSE are kept in fp32.  Accuracy against exact attention of the dequantised
 * inputs: the rounding of P (3 mantissa bits) bounds each O element's error
 * by 2^-4 max|V| and typically gives a relative L2 error of ~2 %; LSE is as
 * accurate as attn_fwd's.
 *
 *   Q8 [B,Hq,Lq,d], K8/V8 [B,Hkv,Lk,d] E4M3 bytes (read only, 16-byte aligned);
 *   q_scale [B,Hq,ceil(Lq/128)], k_scale/v_scale [B,Hkv,ceil(Lk/128)] fp32
 *   device arrays (16-byte aligned), each finite and > 0 -- a scale that is
 *   not sets ATTN_DEV_BAD_SCALE in the status word (results then undefined,
 *   nothing outside the buffers is touched).
 *   O, lse, scale, mask_flags, k_lens, workspace: as attn_fwd.
 *   d must be 128 (else ATTN_ERR_UNSUPPORTED).
 */
attn_status_t attn_fwd_fp8(const void* Q8, const void* K8, const void* V8, const float* q_scale,
                           const float* k_scale, const float* v_scale, attn_bf16_t* O,
                           float* lse, int B, int Hq, int Hkv, int Lq, int Lk, int d, float scale,
                           int mask_flags, const int32_t* k_lens, void* workspace,
                           size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------ merge of partial results
 * Combines partial attention results of the same query rows over disjoint key
 * sets with the normalised merge rule of the FlashAttention-2 tutorial (2.1.3),
 * in LSE form:  LSE = ln(e^{LSE_a} + e^{LSE_b}),
 *               O = e^{LSE_a - LSE} O_a + e^{LSE_b - LSE} O_b.
 * Used by ring (context-parallel) attention to fold in one key chunk per step.
 *
 *   O_part [rows, d] bf16 and lse_part [rows] fp32 (natural log, as attn_fwd
 *   writes them; -inf = no visible key): the partial to fold in (read only).
 *   O_acc [rows, d] fp32 and lse_acc [rows] fp32: the accumulator (in/out);
 *   init = 1 overwrites it with the partial, init = 0 merges into it.
 *   O_out [rows, d] bf16 or NULL: also receives the merged O (last step).
 *   rows >= 0 (any [B, H, L] flattened); d in {8, 16, 32, 64, 128, 256}.
 *   All pointers 16-byte aligned, else ATTN_ERR_INVALID.  Rows whose two LSEs
 *   are both -inf become O = 0, LSE = -inf.
 */
attn_status_t attn_merge_partial(const attn_bf16_t* O_part, const float* lse_part, float* O_acc,
                                 float* lse_acc, attn_bf16_t* O_out, long long rows, int d,
                                 int init, void* stream);

/* The same fold done by the forward kernel itself: attn_fwd of Q against K/V
 * (one chunk of the keys), merged into the accumulator in the kernel's
 * epilogue instead of being written out as a bf16 partial -- one launch per
 * ring step.  Q, K, V, B, Hq, Hkv, Lq, Lk, d, scale, mask_flags, k_lens,
 * workspace: as attn_fwd (d = 64 or 128).  O_acc [B,Hq,Lq,d] fp32 and lse_acc
 * [B,Hq,Lq] fp32: the accumulator (in/out; init = 1 overwrites it); O_out
 * [B,Hq,Lq,d] bf16 or NULL receives the merged O. */
attn_status_t attn_fwd_merge(const attn_bf16_t* Q, const attn_bf16_t* K, const attn_bf16_t* V,
                             float* O_acc, float* lse_acc, attn_bf16_t* O_out, int init, int B,
                             int Hq, int Hkv, int Lq, int Lk, int d, float scale, int mask_flags,
                             const int32_t* k_lens, void* workspace, size_t ws_bytes,
                             void* stream);

/* Adds a bf16 partial [n] into an fp32 accumulator [n] (init = 1: sets it to
 * the partial; part = NULL with init = 0 adds nothing, to convert the sum);
 * out [n] bf16 or NULL receives the running sum.  Used to sum ring attention's
 * per-chunk partial gradients with one rounding at the end.  n >= 0 and a
 * multiple of 8; pointers 16-byte aligned; else ATTN_ERR_INVALID. */
attn_status_t attn_accumulate(const attn_bf16_t* part, float* acc, attn_bf16_t* out, long long n,
                              int init, void* stream);

/* ------------------------------------------------------------------ sliding window
 * Local causal (sliding-window) attention: the causal mask of attn_fwd /
 * attn_bwd plus a lower edge, so query row i sees only keys j with
 *   i + (Lk - Lq) - window < j <= i + (Lk - Lq)   (and j < k_lens[b]).
 * The pages name local / causal / padding masks as variants of M; the window
 * convention (the `window` latest keys, the diagonal included) is ours.  Key
 * tiles entirely outside a query tile's window are skipped, so the work
 * grows with window, not with Lk.  window >= 1 (else ATTN_ERR_INVALID); all
 * other arguments, layouts and errors as attn_fwd / attn_bwd with
 * mask_flags = ATTN_MASK_CAUSAL (attn_bwd_sliding takes the lse that
 * attn_fwd_sliding wrote for the same window).
 */
attn_status_t attn_fwd_sliding(const attn_bf16_t* Q, const attn_bf16_t* K, const attn_bf16_t* V,
                               attn_bf16_t* O, float* lse, int B, int Hq, int Hkv, int Lq, int Lk,
                               int d, float scale, int window, const int32_t* k_lens,
                               void* workspace, size_t ws_bytes, void* stream);
attn_status_t attn_bwd_sliding(const attn_bf16_t* Q, const attn_bf16_t* K, const attn_bf16_t* V,
                               const attn_bf16_t* O, const attn_bf16_t* dO, const float* lse,
                               attn_bf16_t* dQ, attn_bf16_t* dK, attn_bf16_t* dV, int B, int Hq,
                               int Hkv, int Lq, int Lk, int d, float scale, int window,
                               const int32_t* k_lens, void* workspace, size_t ws_bytes,
                               void* stream);

/* ------------------------------------------------------------------ packed forward
 * The forward over variable-length sequences packed back to back (no padding):
 * the same attention per sequence as attn_fwd, with the batch given by
 * offsets instead of a common length.  The pages name varlen batching as the
 * prefill-side partner of the KV-cache ledger; the layout and the offset
 * convention are ours.
 *
 *   Q, O [total_q, Hq, d] bf16; K, V [total_k, Hkv, d] bf16.  cu_seqlens_q and
 *   cu_seqlens_k: device int32 [B + 1], non-decreasing, starting at 0; sequence
 *   b is rows [cu_q[b], cu_q[b+1]) of Q and [cu_k[b], cu_k[b+1]) of K and V,
 *   at most max_seqlen_q / max_seqlen_k rows long and inside total_q / total_k.
 *   lse [Hq, total_q] fp32 (may be NULL).  mask_flags as attn_fwd (the causal
 *   mask is aligned to each sequence's bottom-right corner); no k_lens (the
 *   offsets give each sequence's keys).  A sequence whose offsets break these
 *   rules is skipped (nothing read or written) and sets ATTN_DEV_BAD_KLEN.
 */
size_t attn_fwd_varlen_workspace_size(int B, int Hq, int Hkv, int max_seqlen_q,
                                      int max_seqlen_k, int d);
attn_status_t attn_fwd_varlen(const attn_bf16_t* Q, const attn_bf16_t* K, const attn_bf16_t* V,
                              attn_bf16_t* O, float* lse, const int32_t* cu_seqlens_q,
                              const int32_t* cu_seqlens_k, int B, int Hq, int Hkv,
                              int max_seqlen_q, int max_seqlen_k, int total_q, int total_k,
                              int d, float scale, int mask_flags, void* workspace,
                              size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------ decode
 * Split-KV decode (one query token per sequence over a contiguous KV cache):
 * the "short query scans a long history" case of the three-ledgers page
 * (section on prefill vs decode).
 * The cache rows [0, k_lens[b]) of each sequence are split into chunks; each
 * chunk yields a partial (m, l, O) and the partials are combined with the
 * normalised merge of the FlashAttention-2 tutorial, 2.1.3:
 *   m = max(m_a, m_b); l = e^{m_a-m} l_a + e^{m_b-m} l_b;
 *   O = (e^{m_a-m} l_a / l) O_a + (e^{m_b-m} l_b / l) O_b.
 *
 *   Q [B,Hq,1,d] bf16; Kcache/Vcache [B,Hkv,Lmax,d] bf16; k_lens device int32
 *   [B], required, each in [0, Lmax] (no causal mask inside the cache).
 *   O [B,Hq,1,d] bf16 and lse [B,Hq] fp32 (lse may be NULL).
 *   The workspace holds the fp32 partials; its size depends on Lmax.
 *   Hq / Hkv must be 1, 2, 4 or 8, and Lmax at most 65535 * 2048 =
 *   134,215,680 rows (the cache is split into chunks of 2048 keys, at most
 *   65535 per sequence); else ATTN_ERR_UNSUPPORTED.
 */
size_t attn_decode_workspace_size(int B, int Hq, int Hkv, int Lmax, int d);
attn_status_t attn_fwd_splitkv_decode(const attn_bf16_t* Q, const attn_bf16_t* Kcache,
                                      const attn_bf16_t* Vcache, attn_bf16_t* O, float* lse,
                                      int B, int Hq, int Hkv, int Lmax, int d, float scale,
                                      const int32_t* k_lens, void* workspace, size_t ws_bytes,
                                      void* stream);

/* ------------------------------------------------------------------ paged decode
 * The same split-KV decode over a paged cache: the KV-cache ledger of the
 * three-ledgers page names paged attention as the decode-side companion of
 * FlashAttention; what it computes is unchanged, only where row r of
 * sequence b is read from.
 *
 *   Kpages/Vpages [n_pages, Hkv, page_size, d] bf16 (each head's rows of a
 *   page are contiguous).  block_table device int32 [B, max_blocks]: row r of
 *   sequence b is row r % page_size of page block_table[b, r / page_size].
 *   Only the entries covering rows [0, k_lens[b]) are read; they must lie in
 *   [0, n_pages).  k_lens device int32 [B], required, each in
 *   [0, max_blocks * page_size].  page_size is a power of two in [16, 65536]
 *   (else ATTN_ERR_UNSUPPORTED).  Q, O, lse, scale, the group sizes and the
 *   limit on max_blocks * page_size as attn_fwd_splitkv_decode.
 *   The workspace is attn_decode_workspace_size(B, Hq, Hkv,
 *   max_blocks * page_size, d) bytes.
 *   A chunk whose block-table entries are out of range reads no page: it sets
 *   ATTN_DEV_BAD_PAGE in the status word and contributes nothing to O.
 */
attn_status_t attn_fwd_splitkv_decode_paged(const attn_bf16_t* Q, const attn_bf16_t* Kpages,
                                            const attn_bf16_t* Vpages,
                                            const int32_t* block_table, int max_blocks,
                                            int page_size, int n_pages, attn_bf16_t* O,
                                            float* lse, int B, int Hq, int Hkv, int d,
                                            float scale, const int32_t* k_lens,
                                            void* workspace, size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------ backward
 * Backward by recomputation: the three-ledgers page says the backward keeps only small row
 * statistics and recomputes the score blocks it needs.  From the saved LSE
 * (and D_i = sum_d dO_id O_id) each score tile is rebuilt as
 * P = exp(S * scale - LSE), and
 *   dV = P^T dO; dP = dO V^T; dS = P o (dP - D); dQ = scale dS K;
 *   dK = scale dS^T Q  (summed over the Hq / Hkv query heads of a KV head).
 *
 *   Q, O, dO [B,Hq,Lq,d] bf16; K, V [B,Hkv,Lk,d] bf16; lse [B,Hq,Lq] fp32 as
 *   written by attn_fwd for the same arguments.  dQ [B,Hq,Lq,d], dK, dV
 *   [B,Hkv,Lk,d] bf16 are written.  Same mask arguments as attn_fwd.
 *   The workspace holds the fp32 accumulator for dQ and the per-row log2-LSE
 *   and D (query rows padded to a multiple of 128 per head): nothing of size
 *   Lq x Lk.  d = 64 and d = 128 each have their own kernels.
 */
size_t attn_bwd_workspace_size(int B, int Hq, int Hkv, int Lq, int Lk, int d);
attn_status_t attn_bwd(const attn_bf16_t* Q, const attn_bf16_t* K, const attn_bf16_t* V,
                       const attn_bf16_t* O, const attn_bf16_t* dO, const float* lse,
                       attn_bf16_t* dQ, attn_bf16_t* dK, attn_bf16_t* dV, int B, int Hq, int Hkv,
                       int Lq, int Lk, int d, float scale, int mask_flags, const int32_t* k_lens,
                       void* workspace, size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------ decode without allocation
 * No counterpart in the pages: an interface addition for callers that cannot
 * allocate device memory.  attn_fwd_splitkv_decode needs a workspace for its
 * fp32 per-chunk partials; some callers cannot hand one over: runtimes whose
 * memory plan is fixed up front and that pass only the tensors they own (no
 * scratch pool to draw from), host frameworks whose operator interface gives
 * tensors but no allocator, and latency-critical loops that must not pay a
 * cudaMalloc's implicit device synchronisation.  They use this variant
 * instead.  It computes exactly what attn_fwd_splitkv_decode computes, with
 * the same kernels and arguments minus the workspace.
 *
 * Scratch: a file-scope device array of ATTN_NOALLOC_SCRATCH_BYTES that every
 * GPU loading the library holds until the process exits.  A request whose
 * partials need more (256 + B*Hq*ceil(Lmax/2048)*(4*d + 4) bytes, rounded up to
 * 256) returns ATTN_ERR_CAPACITY before anything is launched.  The first call
 * on a device looks up the array's device address (cudaGetSymbolAddress, with
 * that device current) and raises the kernels' shared-memory limit; later
 * calls make neither API call.  The set-up is repeated when the
 * device's CUDA context changes (after cudaDeviceReset, the next call is a
 * first call again).  The call allocates and frees nothing.
 *
 * All calls share the one array: calls that may overlap on the GPU (different
 * streams, or different host threads on one device) race and corrupt each
 * other's results; serialise them.  Each call clears the status word it keeps
 * at the head of the array; the partials need no clearing.  Device-side
 * errors are not reported (there is no workspace to read a status from):
 * a k_lens entry outside [0, Lmax] zeroes that sequence's outputs, and a wait
 * that expired makes its chunk contribute nothing, so O and LSE are then
 * partial results although the call returned ATTN_OK.
 */
#define ATTN_NOALLOC_SCRATCH_BYTES (16u << 20)
attn_status_t attn_fwd_splitkv_decode_noalloc(const attn_bf16_t* Q, const attn_bf16_t* Kcache,
                                              const attn_bf16_t* Vcache, attn_bf16_t* O,
                                              float* lse, int B, int Hq, int Hkv, int Lmax,
                                              int d, float scale, const int32_t* k_lens,
                                              void* stream);

/* ------------------------------------------------------------------ status
 * Reads (after synchronising `stream`) the device status word of `workspace`:
 * ATTN_OK when clear, ATTN_ERR_TIMEOUT if any wait expired, ATTN_ERR_INVALID
 * if a k_lens entry, a block-table entry, a sequence offset or an 8-bit scale
 * was out of range.  *bits (may be NULL) receives the raw
 * ATTN_DEV_* bits.  Returns ATTN_ERR_CUDA if the copy itself fails. */
attn_status_t attn_read_device_status(const void* workspace, void* stream, int32_t* bits);

/* Enqueues a clear of the status word on `stream`. */
attn_status_t attn_clear_device_status(void* workspace, void* stream);

/* Number of streaming multiprocessors the persistent kernels size their grids
 * for (the current device's count); 0 when no device is visible. */
int attn_num_sms(void);

#ifdef __cplusplus
}
#endif

#endif /* ATTN_H_ */
