// attn_api.cu -- the C ABI (include/attn.h): argument validation, tensor-map
// encoding, grid planning and kernel launches on the caller's stream.  It
// allocates no memory and never synchronises (attn_read_device_status aside).
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "../../include/attn.h"
#include "accum_kernel.cuh"
#include "bwd_kernel.cuh"
#include "decode_kernel.cuh"
#include "fwd_kernel.cuh"
#include "launch_cache.cuh"
#include "merge_kernel.cuh"

namespace {

constexpr size_t kStatusBytes = 256;  // status word + scheduler counters, 256-byte aligned

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned256(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 255u) == 0; }

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// 3-D bf16 view [heads][rows][d] of a [B, H, L, d] tensor, boxes of
// 64 columns x `box_rows` rows x 1 head, 128-byte swizzle.
bool make_tmap(CUtensorMap* m, const void* base, int d, int L, long long heads, int box_rows) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(L > 0 ? L : 1),
                        static_cast<cuuint64_t>(heads)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * 2,
                           static_cast<cuuint64_t>(d) * 2 * static_cast<cuuint64_t>(L > 0 ? L : 1)};
  cuuint32_t box[3] = {64, static_cast<cuuint32_t>(box_rows), 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// 3-D bf16 view of a packed [T, H, d] tensor as [rows = T][heads = H][d] with the
// kernels' coordinate order (column, row, head): dimension 1 steps over tokens
// (stride H * d), dimension 2 over heads (stride d).
bool make_tmap_packed(CUtensorMap* m, const void* base, int d, int T, int heads, int box_rows) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(T > 0 ? T : 1),
                        static_cast<cuuint64_t>(heads)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * 2 * static_cast<cuuint64_t>(heads),
                           static_cast<cuuint64_t>(d) * 2};
  cuuint32_t box[3] = {64, static_cast<cuuint32_t>(box_rows), 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// 3-D 8-bit view [heads][rows][d] of a [B, H, L, d] E4M3 tensor, boxes of
// 128 columns (128 bytes) x `box_rows` rows x 1 head, 128-byte swizzle.
bool make_tmap_u8(CUtensorMap* m, const void* base, int d, int L, long long heads, int box_rows) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(L > 0 ? L : 1),
                        static_cast<cuuint64_t>(heads)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(d),
                           static_cast<cuuint64_t>(d) * static_cast<cuuint64_t>(L > 0 ? L : 1)};
  cuuint32_t box[3] = {128, static_cast<cuuint32_t>(box_rows), 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

int device_sms() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  int n = 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
  return n;
}

bool shapes_ok(int B, int Hq, int Hkv, int Lq, int Lk) {
  if (B < 1 || Hq < 1 || Hkv < 1 || Lq < 0 || Lk < 0) return false;
  if (Hq % Hkv != 0) return false;
  // every element index must fit the kernels' 64-bit offsets and the tensor
  // maps' 32-bit coordinates
  if (static_cast<long long>(B) * Hq > (1LL << 30)) return false;
  if (Lq > (1 << 30) || Lk > (1 << 30)) return false;
  return true;
}

using attn_host::set_smem;

}  // namespace

bool attn_bwd_impl::make_tmap_rows(CUtensorMap* m, const void* base, int d, int L,
                                   long long heads, int box_rows) {
  return make_tmap(m, base, d, L, heads, box_rows);
}

bool attn_decode_impl::make_tmap_paged(CUtensorMap* m, const void* base, int d, int page,
                                       int Hkv, int n_pages, int box_rows) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[4] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(page),
                        static_cast<cuuint64_t>(Hkv), static_cast<cuuint64_t>(n_pages)};
  const cuuint64_t row = static_cast<cuuint64_t>(d) * 2;
  cuuint64_t strides[3] = {row, row * static_cast<cuuint64_t>(page),
                           row * static_cast<cuuint64_t>(page) * static_cast<cuuint64_t>(Hkv)};
  cuuint32_t box[4] = {64, static_cast<cuuint32_t>(box_rows), 1, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool attn_bwd_impl::make_tmap_acc64(CUtensorMap* m, float* base, int Lqp, long long heads) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {64, static_cast<cuuint64_t>(Lqp), static_cast<cuuint64_t>(heads)};
  cuuint64_t strides[2] = {64 * 4, static_cast<cuuint64_t>(Lqp) * 64 * 4};
  cuuint32_t box[3] = {32, 128, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, base, dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Shared launch of the forward kernel; p carries the layout-specific fields.
static attn_status_t launch_fwd(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                         attn_fwd_impl::Params p, attn_bf16_t* O, float* lse, int B, int Hq,
                         int Hkv, int d, float scale, int mask_flags, void* workspace,
                         void* stream) {
  const int sms = device_sms();
  if (sms <= 0) return ATTN_ERR_CUDA;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int n_pairs = (p.Lq + 2 * attn_fwd_impl::BM - 1) / (2 * attn_fwd_impl::BM);
  const int n_items = B * Hq * n_pairs;
  p.O = reinterpret_cast<__nv_bfloat16*>(O);
  p.lse = lse;
  p.status = reinterpret_cast<int*>(workspace);
  p.sched = reinterpret_cast<int*>(workspace) + 1;
  p.B = B;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.causal = (mask_flags & ATTN_MASK_CAUSAL) ? 1 : 0;
  p.n_pairs = n_pairs;
  p.n_items = n_items;
  const int grid = n_items < sms ? n_items : sms;
  const int mode = p.cu_q      ? attn_fwd_impl::MODE_VARLEN
                   : p.q_scale ? attn_fwd_impl::MODE_FP8
                   : p.o_acc   ? attn_fwd_impl::MODE_MERGE
                   : p.window > 0 ? attn_fwd_impl::MODE_WINDOW
                                  : attn_fwd_impl::MODE_PLAIN;
  cudaError_t e = cudaSuccess;
  auto run = [&](auto kernel, int smem) {
    e = set_smem(kernel, smem);
    if (e == cudaSuccess) kernel<<<grid, attn_fwd_impl::NTHREADS, smem, s>>>(tq, tk, tv, p);
  };
  using namespace attn_fwd_impl;
  if (d == 128) {
    constexpr int smem = Cfg<128>::SMEM_BYTES;
    if (mode == MODE_PLAIN) run(fwd_kernel<128, MODE_PLAIN>, smem);
    else if (mode == MODE_WINDOW) run(fwd_kernel<128, MODE_WINDOW>, smem);
    else if (mode == MODE_FP8) run(fwd_kernel<128, MODE_FP8>, Cfg<128, 1>::SMEM_BYTES);
    else if (mode == MODE_MERGE) run(fwd_kernel<128, MODE_MERGE>, smem);
    else run(fwd_kernel<128, MODE_VARLEN>, smem);
  } else {
    if (mode == MODE_FP8) return ATTN_ERR_UNSUPPORTED;
    constexpr int smem = Cfg<64>::SMEM_BYTES;
    if (mode == MODE_PLAIN) run(fwd_kernel<64, MODE_PLAIN>, smem);
    else if (mode == MODE_WINDOW) run(fwd_kernel<64, MODE_WINDOW>, smem);
    else if (mode == MODE_MERGE) run(fwd_kernel<64, MODE_MERGE>, smem);
    else run(fwd_kernel<64, MODE_VARLEN>, smem);
  }
  if (e != cudaSuccess) return ATTN_ERR_CUDA;
  return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

extern "C" {

const char* attn_status_string(attn_status_t s) {
  switch (s) {
    case ATTN_OK: return "ok";
    case ATTN_ERR_INVALID: return "invalid argument";
    case ATTN_ERR_UNSUPPORTED: return "unsupported";
    case ATTN_ERR_CUDA: return "cuda error";
    case ATTN_ERR_TIMEOUT: return "device wait timed out";
    case ATTN_ERR_CAPACITY: return "request exceeds the fixed scratch of the no-alloc call";
  }
  return "unknown status";
}

int attn_num_sms(void) { return device_sms(); }

// ------------------------------------------------------------------ forward

size_t attn_fwd_workspace_size(int, int, int, int, int, int) { return kStatusBytes; }

static attn_status_t fwd_batched(const attn_bf16_t* Q, const attn_bf16_t* K,
                                 const attn_bf16_t* V, attn_bf16_t* O, float* lse, int B, int Hq,
                                 int Hkv, int Lq, int Lk, int d, float scale, int mask_flags,
                                 int window, const int32_t* k_lens, void* workspace,
                                 size_t ws_bytes, void* stream) {
  if (!shapes_ok(B, Hq, Hkv, Lq, Lk)) return ATTN_ERR_INVALID;
  if (!Q || !K || !V || !O || !workspace) return ATTN_ERR_INVALID;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O) ||
      (lse && !aligned16(lse)) || (k_lens && !aligned16(k_lens)) || !aligned256(workspace))
    return ATTN_ERR_INVALID;
  if (!(std::isfinite(scale) && scale > 0.f)) return ATTN_ERR_INVALID;
  if (mask_flags != ATTN_MASK_NONE && mask_flags != ATTN_MASK_CAUSAL) return ATTN_ERR_INVALID;
  if (ws_bytes < attn_fwd_workspace_size(B, Hq, Hkv, Lq, Lk, d)) return ATTN_ERR_INVALID;
  if (d != 64 && d != 128) return ATTN_ERR_UNSUPPORTED;
  if (Lq == 0) return ATTN_OK;

  CUtensorMap tq, tk, tv;
  if (!make_tmap(&tq, Q, d, Lq, static_cast<long long>(B) * Hq, 128) ||
      !make_tmap(&tk, K, d, Lk, static_cast<long long>(B) * Hkv, 128) ||
      !make_tmap(&tv, V, d, Lk, static_cast<long long>(B) * Hkv, 128))
    return ATTN_ERR_CUDA;
  attn_fwd_impl::Params p{};
  p.k_lens = k_lens;
  p.Lq = Lq;
  p.Lk = Lk;
  p.window = window;
  return launch_fwd(tq, tk, tv, p, O, lse, B, Hq, Hkv, d, scale, mask_flags, workspace, stream);
}

attn_status_t attn_fwd(const attn_bf16_t* Q, const attn_bf16_t* K, const attn_bf16_t* V,
                       attn_bf16_t* O, float* lse, int B, int Hq, int Hkv, int Lq, int Lk, int d,
                       float scale, int mask_flags, const int32_t* k_lens, void* workspace,
                       size_t ws_bytes, void* stream) {
  return fwd_batched(Q, K, V, O, lse, B, Hq, Hkv, Lq, Lk, d, scale, mask_flags, 0, k_lens,
                     workspace, ws_bytes, stream);
}

attn_status_t attn_fwd_sliding(const attn_bf16_t* Q, const attn_bf16_t* K, const attn_bf16_t* V,
                               attn_bf16_t* O, float* lse, int B, int Hq, int Hkv, int Lq, int Lk,
                               int d, float scale, int window, const int32_t* k_lens,
                               void* workspace, size_t ws_bytes, void* stream) {
  if (window < 1) return ATTN_ERR_INVALID;
  return fwd_batched(Q, K, V, O, lse, B, Hq, Hkv, Lq, Lk, d, scale, ATTN_MASK_CAUSAL, window,
                     k_lens, workspace, ws_bytes, stream);
}

attn_status_t attn_fwd_fp8(const void* Q8, const void* K8, const void* V8, const float* q_scale,
                           const float* k_scale, const float* v_scale, attn_bf16_t* O, float* lse,
                           int B, int Hq, int Hkv, int Lq, int Lk, int d, float scale,
                           int mask_flags, const int32_t* k_lens, void* workspace,
                           size_t ws_bytes, void* stream) {
  if (!shapes_ok(B, Hq, Hkv, Lq, Lk)) return ATTN_ERR_INVALID;
  if (!Q8 || !K8 || !V8 || !q_scale || !k_scale || !v_scale || !O || !workspace)
    return ATTN_ERR_INVALID;
  if (!aligned16(Q8) || !aligned16(K8) || !aligned16(V8) || !aligned16(O) ||
      !aligned16(q_scale) || !aligned16(k_scale) || !aligned16(v_scale) ||
      (lse && !aligned16(lse)) || (k_lens && !aligned16(k_lens)) || !aligned256(workspace))
    return ATTN_ERR_INVALID;
  if (!(std::isfinite(scale) && scale > 0.f)) return ATTN_ERR_INVALID;
  if (mask_flags != ATTN_MASK_NONE && mask_flags != ATTN_MASK_CAUSAL) return ATTN_ERR_INVALID;
  if (ws_bytes < attn_fwd_workspace_size(B, Hq, Hkv, Lq, Lk, d)) return ATTN_ERR_INVALID;
  if (d != 128) return ATTN_ERR_UNSUPPORTED;
  if (Lq == 0) return ATTN_OK;
  CUtensorMap tq, tk, tv;
  if (!make_tmap_u8(&tq, Q8, d, Lq, static_cast<long long>(B) * Hq, 128) ||
      !make_tmap_u8(&tk, K8, d, Lk, static_cast<long long>(B) * Hkv, 128) ||
      !make_tmap_u8(&tv, V8, d, Lk, static_cast<long long>(B) * Hkv, 128))
    return ATTN_ERR_CUDA;
  attn_fwd_impl::Params p{};
  p.k_lens = k_lens;
  p.Lq = Lq;
  p.Lk = Lk;
  p.q_scale = q_scale;
  p.k_scale = k_scale;
  p.v_scale = v_scale;
  p.n_qt = (Lq + attn_fwd_impl::BM - 1) / attn_fwd_impl::BM;
  p.n_kt = (Lk + attn_fwd_impl::BN - 1) / attn_fwd_impl::BN;
  return launch_fwd(tq, tk, tv, p, O, lse, B, Hq, Hkv, d, scale, mask_flags, workspace, stream);
}

attn_status_t attn_fwd_merge(const attn_bf16_t* Q, const attn_bf16_t* K, const attn_bf16_t* V,
                             float* O_acc, float* lse_acc, attn_bf16_t* O_out, int init, int B,
                             int Hq, int Hkv, int Lq, int Lk, int d, float scale, int mask_flags,
                             const int32_t* k_lens, void* workspace, size_t ws_bytes,
                             void* stream) {
  if (!shapes_ok(B, Hq, Hkv, Lq, Lk)) return ATTN_ERR_INVALID;
  if (!Q || !K || !V || !O_acc || !lse_acc || !workspace) return ATTN_ERR_INVALID;
  if (init != 0 && init != 1) return ATTN_ERR_INVALID;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O_acc) ||
      !aligned16(lse_acc) || (O_out && !aligned16(O_out)) || (k_lens && !aligned16(k_lens)) ||
      !aligned256(workspace))
    return ATTN_ERR_INVALID;
  if (!(std::isfinite(scale) && scale > 0.f)) return ATTN_ERR_INVALID;
  if (mask_flags != ATTN_MASK_NONE && mask_flags != ATTN_MASK_CAUSAL) return ATTN_ERR_INVALID;
  if (ws_bytes < attn_fwd_workspace_size(B, Hq, Hkv, Lq, Lk, d)) return ATTN_ERR_INVALID;
  if (d != 64 && d != 128) return ATTN_ERR_UNSUPPORTED;
  if (Lq == 0) return ATTN_OK;
  CUtensorMap tq, tk, tv;
  if (!make_tmap(&tq, Q, d, Lq, static_cast<long long>(B) * Hq, 128) ||
      !make_tmap(&tk, K, d, Lk, static_cast<long long>(B) * Hkv, 128) ||
      !make_tmap(&tv, V, d, Lk, static_cast<long long>(B) * Hkv, 128))
    return ATTN_ERR_CUDA;
  attn_fwd_impl::Params p{};
  p.k_lens = k_lens;
  p.Lq = Lq;
  p.Lk = Lk;
  p.o_acc = O_acc;
  p.merge_init = init;
  return launch_fwd(tq, tk, tv, p, O_out, lse_acc, B, Hq, Hkv, d, scale, mask_flags, workspace,
                    stream);
}

size_t attn_fwd_varlen_workspace_size(int, int, int, int, int, int) { return kStatusBytes; }

attn_status_t attn_fwd_varlen(const attn_bf16_t* Q, const attn_bf16_t* K, const attn_bf16_t* V,
                              attn_bf16_t* O, float* lse, const int32_t* cu_seqlens_q,
                              const int32_t* cu_seqlens_k, int B, int Hq, int Hkv,
                              int max_seqlen_q, int max_seqlen_k, int total_q, int total_k,
                              int d, float scale, int mask_flags, void* workspace,
                              size_t ws_bytes, void* stream) {
  if (!shapes_ok(B, Hq, Hkv, max_seqlen_q, max_seqlen_k)) return ATTN_ERR_INVALID;
  if (total_q < 0 || total_k < 0 || total_q > (1 << 30) || total_k > (1 << 30))
    return ATTN_ERR_INVALID;
  if (!Q || !K || !V || !O || !cu_seqlens_q || !cu_seqlens_k || !workspace)
    return ATTN_ERR_INVALID;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O) ||
      (lse && !aligned16(lse)) || !aligned16(cu_seqlens_q) || !aligned16(cu_seqlens_k) ||
      !aligned256(workspace))
    return ATTN_ERR_INVALID;
  if (!(std::isfinite(scale) && scale > 0.f)) return ATTN_ERR_INVALID;
  if (mask_flags != ATTN_MASK_NONE && mask_flags != ATTN_MASK_CAUSAL) return ATTN_ERR_INVALID;
  if (ws_bytes < attn_fwd_varlen_workspace_size(B, Hq, Hkv, max_seqlen_q, max_seqlen_k, d))
    return ATTN_ERR_INVALID;
  if (d != 64 && d != 128) return ATTN_ERR_UNSUPPORTED;
  if (max_seqlen_q == 0 || total_q == 0) return ATTN_OK;
  CUtensorMap tq, tk, tv;
  if (!make_tmap_packed(&tq, Q, d, total_q, Hq, 128) ||
      !make_tmap_packed(&tk, K, d, total_k, Hkv, 128) ||
      !make_tmap_packed(&tv, V, d, total_k, Hkv, 128))
    return ATTN_ERR_CUDA;
  attn_fwd_impl::Params p{};
  p.Lq = max_seqlen_q;
  p.Lk = max_seqlen_k;
  p.cu_q = cu_seqlens_q;
  p.cu_k = cu_seqlens_k;
  p.total_q = total_q;
  p.total_k = total_k;
  return launch_fwd(tq, tk, tv, p, O, lse, B, Hq, Hkv, d, scale, mask_flags, workspace, stream);
}

// ------------------------------------------------------------------ merge of partials

attn_status_t attn_merge_partial(const attn_bf16_t* O_part, const float* lse_part, float* O_acc,
                                 float* lse_acc, attn_bf16_t* O_out, long long rows, int d,
                                 int init, void* stream) {
  if (rows < 0 || !(d == 8 || d == 16 || d == 32 || d == 64 || d == 128 || d == 256))
    return ATTN_ERR_INVALID;
  if (init != 0 && init != 1) return ATTN_ERR_INVALID;
  if (!O_part || !lse_part || !O_acc || !lse_acc) return ATTN_ERR_INVALID;
  if (!aligned16(O_part) || !aligned16(O_acc) || (O_out && !aligned16(O_out)) ||
      !aligned16(lse_part) || !aligned16(lse_acc))
    return ATTN_ERR_INVALID;
  if (rows == 0) return ATTN_OK;
  const int sms = device_sms();
  if (sms <= 0) return ATTN_ERR_CUDA;
  attn_merge_impl::Params p;
  p.O_part = reinterpret_cast<const __nv_bfloat16*>(O_part);
  p.lse_part = lse_part;
  p.O_acc = O_acc;
  p.lse_acc = lse_acc;
  p.O_out = reinterpret_cast<__nv_bfloat16*>(O_out);
  p.rows = rows;
  p.d = d;
  p.init = init;
  const long long rpb = attn_merge_impl::NTHREADS / (d / 8);
  const long long need = (rows + rpb - 1) / rpb;
  const long long cap = static_cast<long long>(sms) * 8;  // 8 resident blocks per SM
  const int grid = static_cast<int>(need < cap ? need : cap);
  attn_merge_impl::merge_kernel<<<grid, attn_merge_impl::NTHREADS, 0,
                                  reinterpret_cast<cudaStream_t>(stream)>>>(p);
  return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

attn_status_t attn_accumulate(const attn_bf16_t* part, float* acc, attn_bf16_t* out, long long n,
                              int init, void* stream) {
  if (n < 0 || n % 8 != 0 || (init != 0 && init != 1) || !acc) return ATTN_ERR_INVALID;
  if (!part && init) return ATTN_ERR_INVALID;
  if ((part && !aligned16(part)) || !aligned16(acc) || (out && !aligned16(out)))
    return ATTN_ERR_INVALID;
  if (n == 0) return ATTN_OK;
  const int sms = device_sms();
  if (sms <= 0) return ATTN_ERR_CUDA;
  attn_accum_impl::Params p;
  p.part = reinterpret_cast<const __nv_bfloat16*>(part);
  p.acc = acc;
  p.out = reinterpret_cast<__nv_bfloat16*>(out);
  p.n8 = n / 8;
  p.init = init;
  const long long need = (p.n8 + attn_accum_impl::NTHREADS - 1) / attn_accum_impl::NTHREADS;
  const long long cap = static_cast<long long>(sms) * 8;
  attn_accum_impl::accum_kernel<<<static_cast<int>(need < cap ? need : cap),
                                  attn_accum_impl::NTHREADS, 0,
                                  reinterpret_cast<cudaStream_t>(stream)>>>(p);
  return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

// ------------------------------------------------------------------ decode

size_t attn_decode_workspace_size(int B, int Hq, int Hkv, int Lmax, int d) {
  return kStatusBytes + attn_decode_impl::partials_bytes(B, Hq, Hkv, Lmax, d);
}

attn_status_t attn_fwd_splitkv_decode(const attn_bf16_t* Q, const attn_bf16_t* Kc,
                                      const attn_bf16_t* Vc, attn_bf16_t* O, float* lse, int B,
                                      int Hq, int Hkv, int Lmax, int d, float scale,
                                      const int32_t* k_lens, void* workspace, size_t ws_bytes,
                                      void* stream) {
  if (!shapes_ok(B, Hq, Hkv, 1, Lmax)) return ATTN_ERR_INVALID;
  if (!Q || !Kc || !Vc || !O || !k_lens || !workspace) return ATTN_ERR_INVALID;
  if (!aligned16(Q) || !aligned16(Kc) || !aligned16(Vc) || !aligned16(O) ||
      (lse && !aligned16(lse)) || !aligned16(k_lens) || !aligned256(workspace))
    return ATTN_ERR_INVALID;
  if (!(std::isfinite(scale) && scale > 0.f)) return ATTN_ERR_INVALID;
  if (ws_bytes < attn_decode_workspace_size(B, Hq, Hkv, Lmax, d)) return ATTN_ERR_INVALID;
  if (d != 128 && d != 64) return ATTN_ERR_UNSUPPORTED;
  if (!attn_decode_impl::supported_group(Hq / Hkv)) return ATTN_ERR_UNSUPPORTED;
  if (!attn_decode_impl::supported_shape(B, Hkv, Lmax, 0)) return ATTN_ERR_UNSUPPORTED;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int sms = device_sms();
  if (sms <= 0) return ATTN_ERR_CUDA;
  cudaError_t e = attn_decode_impl::launch(
      reinterpret_cast<const __nv_bfloat16*>(Q), reinterpret_cast<const __nv_bfloat16*>(Kc),
      reinterpret_cast<const __nv_bfloat16*>(Vc), reinterpret_cast<__nv_bfloat16*>(O), lse, B, Hq,
      Hkv, Lmax, d, scale, k_lens, reinterpret_cast<int*>(workspace),
      reinterpret_cast<uint8_t*>(workspace) + kStatusBytes, sms, s);
  return e == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

attn_status_t attn_fwd_splitkv_decode_paged(const attn_bf16_t* Q, const attn_bf16_t* Kp,
                                            const attn_bf16_t* Vp, const int32_t* block_table,
                                            int max_blocks, int page_size, int n_pages,
                                            attn_bf16_t* O, float* lse, int B, int Hq, int Hkv,
                                            int d, float scale, const int32_t* k_lens,
                                            void* workspace, size_t ws_bytes, void* stream) {
  if (max_blocks <= 0 || n_pages <= 0 || page_size <= 0) return ATTN_ERR_INVALID;
  int page_log2 = 0;
  while ((1 << page_log2) < page_size && page_log2 < 17) ++page_log2;
  if ((1 << page_log2) != page_size || page_size < 16 || page_size > 65536)
    return ATTN_ERR_UNSUPPORTED;
  const long long lmax = static_cast<long long>(max_blocks) * page_size;
  if (lmax > (1 << 30)) return ATTN_ERR_INVALID;
  const int Lmax = static_cast<int>(lmax);
  if (!shapes_ok(B, Hq, Hkv, 1, Lmax)) return ATTN_ERR_INVALID;
  if (!Q || !Kp || !Vp || !block_table || !O || !k_lens || !workspace) return ATTN_ERR_INVALID;
  if (!aligned16(Q) || !aligned16(Kp) || !aligned16(Vp) || !aligned16(block_table) ||
      !aligned16(O) || (lse && !aligned16(lse)) || !aligned16(k_lens) || !aligned256(workspace))
    return ATTN_ERR_INVALID;
  if (!(std::isfinite(scale) && scale > 0.f)) return ATTN_ERR_INVALID;
  if (ws_bytes < attn_decode_workspace_size(B, Hq, Hkv, Lmax, d)) return ATTN_ERR_INVALID;
  if (d != 128 && d != 64) return ATTN_ERR_UNSUPPORTED;
  if (!attn_decode_impl::supported_group(Hq / Hkv)) return ATTN_ERR_UNSUPPORTED;
  if (!attn_decode_impl::supported_shape(B, Hkv, Lmax, page_size)) return ATTN_ERR_UNSUPPORTED;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int sms = device_sms();
  if (sms <= 0) return ATTN_ERR_CUDA;
  const attn_decode_impl::PagedKV pg{block_table, max_blocks, page_log2, n_pages};
  cudaError_t e = attn_decode_impl::launch(
      reinterpret_cast<const __nv_bfloat16*>(Q), reinterpret_cast<const __nv_bfloat16*>(Kp),
      reinterpret_cast<const __nv_bfloat16*>(Vp), reinterpret_cast<__nv_bfloat16*>(O), lse, B, Hq,
      Hkv, Lmax, d, scale, k_lens, reinterpret_cast<int*>(workspace),
      reinterpret_cast<uint8_t*>(workspace) + kStatusBytes, sms, s, &pg);
  return e == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

// ------------------------------------------------------------------ backward

size_t attn_bwd_workspace_size(int B, int Hq, int Hkv, int Lq, int Lk, int d) {
  return kStatusBytes + attn_bwd_impl::scratch_bytes(B, Hq, Hkv, Lq, Lk, d);
}

static attn_status_t bwd_batched(const attn_bf16_t* Q, const attn_bf16_t* K,
                                 const attn_bf16_t* V, const attn_bf16_t* O,
                                 const attn_bf16_t* dO, const float* lse, attn_bf16_t* dQ,
                                 attn_bf16_t* dK, attn_bf16_t* dV, int B, int Hq, int Hkv, int Lq,
                                 int Lk, int d, float scale, int mask_flags, int window,
                                 const int32_t* k_lens, void* workspace, size_t ws_bytes,
                                 void* stream) {
  if (!shapes_ok(B, Hq, Hkv, Lq, Lk)) return ATTN_ERR_INVALID;
  if (!Q || !K || !V || !O || !dO || !lse || !dQ || !dK || !dV || !workspace)
    return ATTN_ERR_INVALID;
  const void* ptrs[] = {Q, K, V, O, dO, lse, dQ, dK, dV};
  for (const void* q : ptrs)
    if (!aligned16(q)) return ATTN_ERR_INVALID;
  if ((k_lens && !aligned16(k_lens)) || !aligned256(workspace)) return ATTN_ERR_INVALID;
  if (!(std::isfinite(scale) && scale > 0.f)) return ATTN_ERR_INVALID;
  if (mask_flags != ATTN_MASK_NONE && mask_flags != ATTN_MASK_CAUSAL) return ATTN_ERR_INVALID;
  if (ws_bytes < attn_bwd_workspace_size(B, Hq, Hkv, Lq, Lk, d)) return ATTN_ERR_INVALID;
  if (d != 64 && d != 128) return ATTN_ERR_UNSUPPORTED;
  if (Lq == 0 && Lk == 0) return ATTN_OK;
  const int sms = device_sms();
  if (sms <= 0) return ATTN_ERR_CUDA;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  attn_bwd_impl::Args a;
  a.Q = reinterpret_cast<const __nv_bfloat16*>(Q);
  a.K = reinterpret_cast<const __nv_bfloat16*>(K);
  a.V = reinterpret_cast<const __nv_bfloat16*>(V);
  a.O = reinterpret_cast<const __nv_bfloat16*>(O);
  a.dO = reinterpret_cast<const __nv_bfloat16*>(dO);
  a.lse = lse;
  a.dQ = reinterpret_cast<__nv_bfloat16*>(dQ);
  a.dK = reinterpret_cast<__nv_bfloat16*>(dK);
  a.dV = reinterpret_cast<__nv_bfloat16*>(dV);
  a.B = B;
  a.Hq = Hq;
  a.Hkv = Hkv;
  a.Lq = Lq;
  a.Lk = Lk;
  a.d = d;
  a.scale = scale;
  a.causal = (mask_flags & ATTN_MASK_CAUSAL) ? 1 : 0;
  a.window = window;
  a.k_lens = k_lens;
  a.status = reinterpret_cast<int*>(workspace);
  a.scratch = reinterpret_cast<uint8_t*>(workspace) + kStatusBytes;
  a.sms = sms;
  return attn_bwd_impl::launch(a, s);
}

attn_status_t attn_bwd(const attn_bf16_t* Q, const attn_bf16_t* K, const attn_bf16_t* V,
                       const attn_bf16_t* O, const attn_bf16_t* dO, const float* lse,
                       attn_bf16_t* dQ, attn_bf16_t* dK, attn_bf16_t* dV, int B, int Hq, int Hkv,
                       int Lq, int Lk, int d, float scale, int mask_flags, const int32_t* k_lens,
                       void* workspace, size_t ws_bytes, void* stream) {
  return bwd_batched(Q, K, V, O, dO, lse, dQ, dK, dV, B, Hq, Hkv, Lq, Lk, d, scale, mask_flags, 0,
                     k_lens, workspace, ws_bytes, stream);
}

attn_status_t attn_bwd_sliding(const attn_bf16_t* Q, const attn_bf16_t* K, const attn_bf16_t* V,
                               const attn_bf16_t* O, const attn_bf16_t* dO, const float* lse,
                               attn_bf16_t* dQ, attn_bf16_t* dK, attn_bf16_t* dV, int B, int Hq,
                               int Hkv, int Lq, int Lk, int d, float scale, int window,
                               const int32_t* k_lens, void* workspace, size_t ws_bytes,
                               void* stream) {
  if (window < 1) return ATTN_ERR_INVALID;
  return bwd_batched(Q, K, V, O, dO, lse, dQ, dK, dV, B, Hq, Hkv, Lq, Lk, d, scale,
                     ATTN_MASK_CAUSAL, window, k_lens, workspace, ws_bytes, stream);
}

// ------------------------------------------------------------------ status

attn_status_t attn_read_device_status(const void* workspace, void* stream, int32_t* bits) {
  if (!workspace) return ATTN_ERR_INVALID;
  int32_t v = 0;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (cudaMemcpyAsync(&v, workspace, sizeof(v), cudaMemcpyDeviceToHost, s) != cudaSuccess)
    return ATTN_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return ATTN_ERR_CUDA;
  if (bits) *bits = v;
  if (v & ATTN_DEV_TIMEOUT) return ATTN_ERR_TIMEOUT;
  if (v & (ATTN_DEV_BAD_KLEN | ATTN_DEV_BAD_PAGE | ATTN_DEV_BAD_SCALE)) return ATTN_ERR_INVALID;
  return ATTN_OK;
}

attn_status_t attn_clear_device_status(void* workspace, void* stream) {
  if (!workspace) return ATTN_ERR_INVALID;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  return cudaMemsetAsync(workspace, 0, kStatusBytes, s) == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

}  // extern "C"

#ifdef ATTN_SELFTEST
// Self-test of the bounded-wait machinery, compiled only into test builds of
// the library (-DATTN_SELFTEST): one CTA waits on an mbarrier that nothing
// arrives on.  The wait must give up after its cycle budget, record
// ATTN_DEV_TIMEOUT and the site id in the status words and let the kernel end
// normally, leaving the CUDA context usable.
namespace {
__global__ void selftest_expired_wait_kernel(int* status, int site) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    sm100::mbar_init(&bar, 1);
    abort_flag = 0;
    sm100::fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0)
    sm100::mbar_wait(&bar, 0, reinterpret_cast<volatile int*>(&abort_flag), status, site);
}
}  // namespace

extern "C" attn_status_t attn_selftest_expired_wait(void* workspace, int site, void* stream) {
  if (!workspace) return ATTN_ERR_INVALID;
  selftest_expired_wait_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      reinterpret_cast<int*>(workspace), site);
  return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}
#endif
