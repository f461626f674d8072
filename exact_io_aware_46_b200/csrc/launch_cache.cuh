// launch_cache.cuh -- host-side, once-per-context set-up shared by the entry
// points: a kernel's dynamic shared-memory limit is raised once per (kernel,
// device, context), so repeated launches make no attribute call.
//
// The key includes the CUDA context: cudaDeviceReset (or any other end of the
// primary context) drops the attributes set in it, and a cache keyed on the
// device alone would then skip the call the new context needs.  The context
// is identified by cuCtxGetId, taken through cudaGetDriverEntryPoint so the
// library has no link-time dependency on libcuda.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <set>
#include <tuple>

namespace attn_host {

// Unique id of the calling thread's current CUDA context; 0 when there is none
// yet (the runtime creates the primary context lazily) or the driver cannot
// say.  A value of 0 is never cached.
inline unsigned long long current_context_id() {
  static PFN_cuCtxGetCurrent_v4000 get_current = nullptr;
  static PFN_cuCtxGetId_v12000 get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(p);
    p = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<PFN_cuCtxGetId_v12000>(p);
  });
  if (!get_current || !get_id) return 0;
  CUcontext c = nullptr;
  if (get_current(&c) != CUDA_SUCCESS || !c) return 0;
  unsigned long long id = 0;
  return get_id(c, &id) == CUDA_SUCCESS ? id : 0;
}

// Raises `kernel`'s dynamic shared-memory limit to `bytes` unless that was
// already done in the current context.
template <typename K>
cudaError_t set_smem(K kernel, int bytes) {
  static std::mutex mu;
  static std::set<std::tuple<const void*, int, unsigned long long, int>> done;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return cudaErrorInvalidDevice;
  const unsigned long long ctx = current_context_id();
  const auto key = std::make_tuple(reinterpret_cast<const void*>(kernel), dev, ctx, bytes);
  std::lock_guard<std::mutex> lock(mu);
  if (ctx != 0 && done.count(key)) return cudaSuccess;
  const cudaError_t e =
      cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  // the attribute call itself creates the context when there was none yet
  const unsigned long long ctx_after = ctx != 0 ? ctx : current_context_id();
  if (e == cudaSuccess && ctx_after != 0)
    done.insert(std::make_tuple(reinterpret_cast<const void*>(kernel), dev, ctx_after, bytes));
  return e;
}

// With the environment variable ATTN_DEBUG set (to anything but "0"), a failed
// CUDA call is reported on stderr with its site; the entry point still returns
// ATTN_ERR_CUDA.  Returns `e`.
inline cudaError_t report(cudaError_t e, const char* where) {
  if (e != cudaSuccess) {
    static const bool on = [] {
      const char* v = std::getenv("ATTN_DEBUG");
      return v && std::strcmp(v, "0") != 0;
    }();
    if (on) std::fprintf(stderr, "attn: %s: %s\n", where, cudaGetErrorString(e));
  }
  return e;
}

// report() for a kernel launch, adding the kernel's compiled resources.
template <typename K>
cudaError_t report_launch(K kernel, const char* where) {
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess && report(e, where) != cudaSuccess) {
    const char* v = std::getenv("ATTN_DEBUG");
    cudaFuncAttributes a;
    if (v && std::strcmp(v, "0") != 0 &&
        cudaFuncGetAttributes(&a, reinterpret_cast<const void*>(kernel)) == cudaSuccess)
      std::fprintf(stderr,
                   "attn: %s: %d registers per thread, at most %d threads per block, "
                   "%zu bytes static and at most %d bytes dynamic shared memory\n",
                   where, a.numRegs, a.maxThreadsPerBlock, a.sharedSizeBytes,
                   a.maxDynamicSharedSizeBytes);
  }
  return e;
}

}  // namespace attn_host
