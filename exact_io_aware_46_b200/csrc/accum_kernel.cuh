// accum_kernel.cuh -- sum of partial gradients.
//
// Ring attention's backward produces each gradient as a sum of per-chunk
// partials (dQ of a query chunk over every key chunk; dK and dV of a key chunk
// over every query chunk).  This kernel adds one bf16 partial into an fp32
// accumulator (or initialises it), optionally writing the running sum as bf16,
// so that the sum is rounded once at the end.  HBM-bound: per element 2 bytes of
// partial read, 4 bytes of accumulator read (unless initialising) and written.
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

__global__ void __launch_bounds__(NTHREADS) accum_kernel(const Params p) {
  for (long long i = static_cast<long long>(blockIdx.x) * NTHREADS + threadIdx.x; i < p.n8;
       i += static_cast<long long>(gridDim.x) * NTHREADS) {
    const uint4 pb = p.part ? reinterpret_cast<const uint4*>(p.part)[i] : make_uint4(0, 0, 0, 0);
    const __nv_bfloat162* b2 = reinterpret_cast<const __nv_bfloat162*>(&pb);
    float4* a4 = reinterpret_cast<float4*>(p.acc) + 2 * i;
    float4 a0 = make_float4(0.f, 0.f, 0.f, 0.f), a1 = a0;
    if (!p.init) {
      a0 = a4[0];
      a1 = a4[1];
    }
    const float2 f0 = __bfloat1622float2(b2[0]), f1 = __bfloat1622float2(b2[1]);
    const float2 f2 = __bfloat1622float2(b2[2]), f3 = __bfloat1622float2(b2[3]);
    a0 = make_float4(a0.x + f0.x, a0.y + f0.y, a0.z + f1.x, a0.w + f1.y);
    a1 = make_float4(a1.x + f2.x, a1.y + f2.y, a1.z + f3.x, a1.w + f3.y);
    a4[0] = a0;
    a4[1] = a1;
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
