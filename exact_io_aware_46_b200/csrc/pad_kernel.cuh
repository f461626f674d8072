// pad_kernel.cuh -- row copies between head dimensions.
//
// The backward kernels are written for d = 128.  A d = 64 problem is the same
// problem with 64 zero columns appended to every row of Q, K, V, O and dO: the
// zero columns add nothing to S = Q K^T, dP = dO V^T or D = rowsum(dO o O), so P,
// dS and the first 64 columns of dQ, dK, dV are unchanged and their last 64
// columns are zero.  This kernel writes the padded copies (dst wider than src:
// zeros after the copied columns) and takes the first columns back out (dst
// narrower).  HBM-bound: 16-byte chunks, one per thread and step.
#pragma once

#include <cstdint>

namespace attn_pad_impl {

constexpr int NTHREADS = 256;

// dst row r = the first min(src_w, dst_w) 16-byte chunks of src row r, then zeros
__global__ void __launch_bounds__(NTHREADS)
    copy_rows_kernel(const uint4* __restrict__ src, int src_w, uint4* __restrict__ dst, int dst_w,
                     long long rows) {
  const long long n = rows * dst_w;
  for (long long i = static_cast<long long>(blockIdx.x) * NTHREADS + threadIdx.x; i < n;
       i += static_cast<long long>(gridDim.x) * NTHREADS) {
    const long long r = i / dst_w;
    const int c = static_cast<int>(i - r * dst_w);
    dst[i] = c < src_w ? src[r * src_w + c] : make_uint4(0, 0, 0, 0);
  }
}

}  // namespace attn_pad_impl
