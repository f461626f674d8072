// merge_kernel.cuh -- merge of partial attention results over disjoint key sets.
//
// Two partial results of the same query rows, (O_a, LSE_a) over key set A and
// (O_b, LSE_b) over a disjoint key set B, combine into the result over A u B
// with the normalised merge rule of the FlashAttention-2 tutorial (2.1.3),
// written with LSE = m + ln l:
//   LSE = ln(e^{LSE_a} + e^{LSE_b}),
//   O   = e^{LSE_a - LSE} O_a + e^{LSE_b - LSE} O_b.
// A partial with LSE = -inf (no visible key) contributes nothing; if both are
// -inf the merged row is O = 0, LSE = -inf.  The accumulator is fp32 so that a
// chain of merges (one per ring step) rounds only once, at the end.
//
// HBM-bound elementwise work: per row, 4d bytes of accumulator read and
// written, 2d bytes of bf16 partial read, 12 bytes of LSE.  One thread per 8
// elements of a row, rows laid out back to back: the thread's 32 bytes of the
// fp32 accumulator move as one 32-byte access (whole sectors) when the
// accumulator is 32-byte aligned (measured on B200, 131,072 rows of d = 128:
// 4.6-4.8 TB/s with two 16-byte accesses).
#pragma once

#include <cuda_bf16.h>
#include <cstdint>

namespace attn_merge_impl {

struct Params {
  const __nv_bfloat16* O_part;  // [rows][d]
  const float* lse_part;        // [rows]
  float* O_acc;                 // [rows][d] in/out
  float* lse_acc;               // [rows] in/out
  __nv_bfloat16* O_out;         // [rows][d] merged result as bf16, or nullptr
  long long rows;
  int d;     // 8, 16, 32, 64, 128 or 256: a row's d / 8 threads sit in one warp
  int init;  // 1: the accumulator is (re)initialised from the partial
};

constexpr int NTHREADS = 256;

__device__ __forceinline__ void ld_global_v8(const void* p, uint32_t* v) {
  asm volatile("ld.global.v8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
               : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]),
                 "=r"(v[6]), "=r"(v[7])
               : "l"(p)
               : "memory");
}
__device__ __forceinline__ void st_global_v8(void* p, const uint32_t* v) {
  asm volatile("st.global.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(p), "r"(v[0]),
               "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7])
               : "memory");
}

__global__ void __launch_bounds__(NTHREADS) merge_kernel(const Params p) {
  const int tpr = p.d / 8;  // threads per row
  const int rows_per_block = NTHREADS / tpr;
  const int sub = threadIdx.x / tpr;
  const int lane = threadIdx.x % tpr;
  // the lanes of this row within the warp (tpr divides 32)
  const unsigned row_mask =
      (tpr == 32 ? 0xffffffffu : ((1u << tpr) - 1u)) << ((threadIdx.x & 31) - lane);
  if (sub >= rows_per_block) return;
  const bool wide = (reinterpret_cast<uintptr_t>(p.O_acc) & 31) == 0;
  for (long long row = static_cast<long long>(blockIdx.x) * rows_per_block + sub; row < p.rows;
       row += static_cast<long long>(gridDim.x) * rows_per_block) {
    const size_t off = static_cast<size_t>(row) * p.d + lane * 8;
    const float lb = p.lse_part[row];
    const float la = p.init ? -INFINITY : p.lse_acc[row];
    const float M = fmaxf(la, lb);
    float wa = 0.f, wb = 0.f, lse = -INFINITY;
    if (M != -INFINITY) {
      wa = (la == -INFINITY) ? 0.f : expf(la - M);
      wb = (lb == -INFINITY) ? 0.f : expf(lb - M);
      const float s = wa + wb;
      lse = M + logf(s);
      wa /= s;
      wb /= s;
    }
    const uint4 pb = *reinterpret_cast<const uint4*>(p.O_part + off);
    const __nv_bfloat162* b2 = reinterpret_cast<const __nv_bfloat162*>(&pb);
    float o[8];
    if (p.init) {
#pragma unroll
      for (int e = 0; e < 8; ++e) o[e] = 0.f;
    } else if (wide) {
      uint32_t a[8];
      ld_global_v8(p.O_acc + off, a);
#pragma unroll
      for (int e = 0; e < 8; ++e) o[e] = __uint_as_float(a[e]);
    } else {
      const float4 a0 = *reinterpret_cast<const float4*>(p.O_acc + off);
      const float4 a1 = *reinterpret_cast<const float4*>(p.O_acc + off + 4);
      o[0] = a0.x; o[1] = a0.y; o[2] = a0.z; o[3] = a0.w;
      o[4] = a1.x; o[5] = a1.y; o[6] = a1.z; o[7] = a1.w;
    }
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 f = __bfloat1622float2(b2[e]);
      o[2 * e] = wa * o[2 * e] + wb * f.x;
      o[2 * e + 1] = wa * o[2 * e + 1] + wb * f.y;
    }
    if (wide) {
      uint32_t a[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) a[e] = __float_as_uint(o[e]);
      st_global_v8(p.O_acc + off, a);
    } else {
      *reinterpret_cast<float4*>(p.O_acc + off) = make_float4(o[0], o[1], o[2], o[3]);
      *reinterpret_cast<float4*>(p.O_acc + off + 4) = make_float4(o[4], o[5], o[6], o[7]);
    }
    if (p.O_out) {
      uint4 ob;
      __nv_bfloat162* o2 = reinterpret_cast<__nv_bfloat162*>(&ob);
#pragma unroll
      for (int e = 0; e < 4; ++e) o2[e] = __floats2bfloat162_rn(o[2 * e], o[2 * e + 1]);
      *reinterpret_cast<uint4*>(p.O_out + off) = ob;
    }
    __syncwarp(row_mask);  // every lane of the row has read lse_acc[row]
    if (lane == 0) p.lse_acc[row] = lse;
  }
}

}  // namespace attn_merge_impl
