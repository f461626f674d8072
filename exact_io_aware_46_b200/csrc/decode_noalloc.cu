// decode_noalloc.cu -- split-KV decode for callers that cannot allocate device
// memory.
//
// attn_fwd_splitkv_decode needs a caller-provided workspace for its fp32
// per-chunk partials.  Some callers have no way to provide one: runtimes that
// hand the library only the tensors they already own (a memory plan fixed up
// front, with no scratch pool to draw from), host frameworks whose operator
// interface passes tensors but no allocator, and latency-critical loops where
// a cudaMalloc's implicit device synchronisation is not acceptable.
// attn_fwd_splitkv_decode_noalloc serves them: the same two kernels, with the
// partials in a fixed, file-scope device array instead of a workspace.
//
// The array is static device memory: every GPU that loads the library holds
// ATTN_NOALLOC_SCRATCH_BYTES of it until the process exits.  In host code the
// array's name is only a host-side stand-in for the symbol, not a device
// address, so the real address is looked up with cudaGetSymbolAddress (with
// the device current) and passed to the kernels.  The lookup is done once per
// device and CUDA context and repeated when the context changes (after a
// cudaDeviceReset the old address is no longer valid).
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <mutex>

#include "../../include/attn.h"
#include "decode_kernel.cuh"

// Layout: bytes [0, 256) status header (device status word first), then the
// partial outputs and log-sum-exps exactly as in the workspace variant.
static __device__ __align__(256) uint8_t g_noalloc_scratch[ATTN_NOALLOC_SCRATCH_BYTES];

namespace {

constexpr size_t kHeader = 256;
constexpr int kMaxDevices = 64;

struct ScratchSlot {
  uint8_t* addr = nullptr;
  unsigned long long ctx = 0;  // context the address was looked up in
};

std::mutex g_mutex;
ScratchSlot g_slot[kMaxDevices];

// Device address of the scratch array in the current device's current
// context; looked up on the first call there and again whenever the context
// has changed (or cannot be identified); nullptr if the lookup fails.
uint8_t* scratch_for_current_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lock(g_mutex);
  ScratchSlot& slot = g_slot[dev];
  const unsigned long long ctx = attn_host::current_context_id();
  if (slot.addr && ctx != 0 && ctx == slot.ctx) return slot.addr;
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return nullptr;
  slot.addr = static_cast<uint8_t*>(p);
  // the lookup creates the primary context if there was none yet
  slot.ctx = attn_host::current_context_id();
  return slot.addr;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

extern "C" attn_status_t attn_fwd_splitkv_decode_noalloc(
    const attn_bf16_t* Q, const attn_bf16_t* Kc, const attn_bf16_t* Vc, attn_bf16_t* O,
    float* lse, int B, int Hq, int Hkv, int Lmax, int d, float scale, const int32_t* k_lens,
    void* stream) {
  if (B < 1 || Hq < 1 || Hkv < 1 || Lmax < 0 || Hq % Hkv != 0) return ATTN_ERR_INVALID;
  if (static_cast<long long>(B) * Hq > (1LL << 30) || Lmax > (1 << 30)) return ATTN_ERR_INVALID;
  if (!Q || !Kc || !Vc || !O || !k_lens) return ATTN_ERR_INVALID;
  if (!aligned16(Q) || !aligned16(Kc) || !aligned16(Vc) || !aligned16(O) ||
      (lse && !aligned16(lse)) || !aligned16(k_lens))
    return ATTN_ERR_INVALID;
  if (!(std::isfinite(scale) && scale > 0.f)) return ATTN_ERR_INVALID;
  if (d != 128 && d != 64) return ATTN_ERR_UNSUPPORTED;
  if (!attn_decode_impl::supported_group(Hq / Hkv)) return ATTN_ERR_UNSUPPORTED;
  if (!attn_decode_impl::supported_shape(B, Hkv, Lmax, 0)) return ATTN_ERR_UNSUPPORTED;
  if (kHeader + attn_decode_impl::partials_bytes(B, Hq, Hkv, Lmax, d) >
      static_cast<size_t>(ATTN_NOALLOC_SCRATCH_BYTES))
    return ATTN_ERR_CAPACITY;

  uint8_t* scratch = scratch_for_current_device();
  if (!scratch) return ATTN_ERR_CUDA;
  int dev_sms = 0, dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&dev_sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return ATTN_ERR_CUDA;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  // The status word must start at zero for each call; the partials need no
  // clearing (the combine reads only partials the split kernel wrote).
  if (cudaMemsetAsync(scratch, 0, kHeader, s) != cudaSuccess) return ATTN_ERR_CUDA;
  cudaError_t e = attn_decode_impl::launch(
      reinterpret_cast<const __nv_bfloat16*>(Q), reinterpret_cast<const __nv_bfloat16*>(Kc),
      reinterpret_cast<const __nv_bfloat16*>(Vc), reinterpret_cast<__nv_bfloat16*>(O), lse, B, Hq,
      Hkv, Lmax, d, scale, k_lens, reinterpret_cast<int*>(scratch), scratch + kHeader, dev_sms, s);
  return e == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}
