// bwd_kernel.cuh -- backward by recomputation (placeholder until the kernels land).
#pragma once

#include "sm100.cuh"

namespace attn_bwd_impl {

struct Args {
  const __nv_bfloat16 *Q, *K, *V, *O, *dO;
  const float* lse;
  __nv_bfloat16 *dQ, *dK, *dV;
  int B, Hq, Hkv, Lq, Lk, d;
  float scale;
  int causal;
  const int* k_lens;
  int* status;
  uint8_t* scratch;
  int sms;
};

inline size_t scratch_bytes(int B, int Hq, int, int Lq, int, int d) {
  const size_t rows = static_cast<size_t>(B) * Hq * Lq;
  size_t bytes = rows * d * 4 + rows * 4;
  return (bytes + 255) & ~static_cast<size_t>(255);
}

inline attn_status_t launch(const Args&, cudaStream_t) { return ATTN_ERR_UNSUPPORTED; }

}  // namespace attn_bwd_impl
