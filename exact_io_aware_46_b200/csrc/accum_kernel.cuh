// accum_kernel.cuh -- sum of partial gradients.
//
// Ring attention's backward produces each gradient as a sum of per-chunk
// partials (dQ of a query chunk over every key chunk; dK and dV of a key chunk
// over every query chunk).  This kernel adds one bf16 partial into an fp32
// accumulator (or initialises it), optionally writing the running sum as bf16,
// so that the sum is rounded once at the end.  HBM-bound: per element 2 bytes of
// partial read, 4 bytes of accumulator read (unless initialising) and written.
// A thread's 8 accumulator elements (32 bytes) move as one 32-byte access, whole
// sectors, when the accumulator is 32-byte aligned.
#pragma once

#include <cuda_bf16.h>
#include <cstdint>

namespace attn_accum_impl {

struct Params {
  const __nv_bfloat16* part;  // [n], or nullptr: add nothing (convert the sum only)
  float* acc;                 // [n] in/out
  __nv_bfloat16* out;         // [n] or nullptr
  long long n8;               // n / 8
  int init;
};

constexpr int NTHREADS = 256;

__device__ __forceinline__ void ld_global_v8(const void* q, uint32_t* v) {
  asm volatile("ld.global.v8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
               : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]),
                 "=r"(v[6]), "=r"(v[7])
               : "l"(q)
               : "memory");
}
__device__ __forceinline__ void st_global_v8(void* q, const uint32_t* v) {
  asm volatile("st.global.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(q), "r"(v[0]),
               "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7])
               : "memory");
}

__global__ void __launch_bounds__(NTHREADS) accum_kernel(const Params p) {
  const bool wide = (reinterpret_cast<uintptr_t>(p.acc) & 31) == 0;
  for (long long i = static_cast<long long>(blockIdx.x) * NTHREADS + threadIdx.x; i < p.n8;
       i += static_cast<long long>(gridDim.x) * NTHREADS) {
    const uint4 pb = p.part ? reinterpret_cast<const uint4*>(p.part)[i] : make_uint4(0, 0, 0, 0);
    const __nv_bfloat162* b2 = reinterpret_cast<const __nv_bfloat162*>(&pb);
    float4* a4 = reinterpret_cast<float4*>(p.acc) + 2 * i;
    float4 a0 = make_float4(0.f, 0.f, 0.f, 0.f), a1 = a0;
    if (!p.init) {
      if (wide) {
        uint32_t v[8];
        ld_global_v8(a4, v);
        a0 = make_float4(__uint_as_float(v[0]), __uint_as_float(v[1]), __uint_as_float(v[2]),
                         __uint_as_float(v[3]));
        a1 = make_float4(__uint_as_float(v[4]), __uint_as_float(v[5]), __uint_as_float(v[6]),
                         __uint_as_float(v[7]));
      } else {
        a0 = a4[0];
        a1 = a4[1];
      }
    }
    const float2 f0 = __bfloat1622float2(b2[0]), f1 = __bfloat1622float2(b2[1]);
    const float2 f2 = __bfloat1622float2(b2[2]), f3 = __bfloat1622float2(b2[3]);
    a0 = make_float4(a0.x + f0.x, a0.y + f0.y, a0.z + f1.x, a0.w + f1.y);
    a1 = make_float4(a1.x + f2.x, a1.y + f2.y, a1.z + f3.x, a1.w + f3.y);
    if (wide) {
      const uint32_t v[8] = {__float_as_uint(a0.x), __float_as_uint(a0.y), __float_as_uint(a0.z),
                             __float_as_uint(a0.w), __float_as_uint(a1.x), __float_as_uint(a1.y),
                             __float_as_uint(a1.z), __float_as_uint(a1.w)};
      st_global_v8(a4, v);
    } else {
      a4[0] = a0;
      a4[1] = a1;
    }
    if (p.out) {
      uint4 ob;
      __nv_bfloat162* o2 = reinterpret_cast<__nv_bfloat162*>(&ob);
      o2[0] = __floats2bfloat162_rn(a0.x, a0.y);
      o2[1] = __floats2bfloat162_rn(a0.z, a0.w);
      o2[2] = __floats2bfloat162_rn(a1.x, a1.y);
      o2[3] = __floats2bfloat162_rn(a1.z, a1.w);
      reinterpret_cast<uint4*>(p.out)[i] = ob;
    }
  }
}

}  // namespace attn_accum_impl
