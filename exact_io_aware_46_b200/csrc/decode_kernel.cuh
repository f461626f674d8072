// decode_kernel.cuh -- split-KV decode (one query token per sequence).
//
// Decode is the "short query scans a long history" case of "FlashAttention and
// long context: three ledgers" (prefill vs decode): per step the whole cache
// row range [0, k_len) is read once and the arithmetic per byte is tiny
// (4 FLOP/B with 4 query heads per key/value head), so the kernels are bound by
// HBM bandwidth:
//
//  * split kernel (tensor cores; below): one CTA per (sequence, key/value
//    head, chunk of CH keys); the scores and the PV product of each 128-key
//    block run as small tcgen05 MMAs (16 heads padded) over a TMA-fed ring, so
//    the CUDA cores only form the exponentials and the kernel streams the
//    cache; every chunk writes its normalised output and log2-sum-exp as a
//    partial;
//  * combine kernel: merges a sequence's partials with the normalised rule of
//    the FlashAttention-2 tutorial, 2.1.3.  Writing each partial as
//    (O_c, LSE_c) with e^{LSE_c} = e^{m_c} l_c gives exactly that rule's
//    weights: O = sum_c e^{LSE_c - M} O_c / sum_c e^{LSE_c - M}.
#pragma once

#include "launch_cache.cuh"
#include "sm100.cuh"

namespace attn_bwd_impl {
// 3-D bf16 tensor map [heads][rows][d], boxes of 64 columns x box_rows rows,
// 128-byte swizzle (defined with the C entry points)
bool make_tmap_rows(CUtensorMap* m, const void* base, int d, int L, long long heads,
                    int box_rows);
}

namespace attn_decode_impl {
// 4-D bf16 tensor map of a paged cache [pages][kv heads][page rows][d] with the
// coordinate order (column, page row, kv head, page), boxes of 64 columns x
// box_rows rows, 128-byte swizzle (defined with the C entry points)
bool make_tmap_paged(CUtensorMap* m, const void* base, int d, int page, int Hkv, int n_pages,
                     int box_rows);

constexpr int CH = 2048;  // keys per split (measured on B200 against 1024, 3072, 4096 and 8192)

inline bool supported_group(int G) { return G == 1 || G == 2 || G == 4 || G == 8; }

inline int n_split_max(int Lmax) { return Lmax > 0 ? (Lmax + CH - 1) / CH : 1; }

inline size_t partials_bytes(int B, int Hq, int, int Lmax, int d) {
  const size_t n = static_cast<size_t>(B) * Hq * n_split_max(Lmax);
  size_t bytes = n * d * 4 + n * 4;
  return (bytes + 255) & ~static_cast<size_t>(255);
}

struct SplitParams {
  const __nv_bfloat16* Q;
  const __nv_bfloat16* K;
  const __nv_bfloat16* V;
  const int* k_lens;
  int* status;
  float* part_o;    // [B*Hq][nsm][D] normalised chunk outputs
  float* part_lse;  // [B*Hq][nsm] log2-sum-exp of the chunk (scaled scores)
  int B, Hq, Hkv, G, Lmax, nsm;
  float scale_log2;
  // paged cache (block_table != nullptr): K/V are [n_pages][Hkv][page][D] and
  // row r of sequence b lives in page block_table[b * max_blocks + r / page]
  const int* block_table;
  int max_blocks, page_log2, n_pages;
};

// The grid is (sequence x kv head, chunk position counted from the sequence's
// end): every sequence's last (partial, shorter) chunk is dispatched last, so
// the grid's tail is short.  Its second dimension limits the cache to 65535
// chunks; paged caches need pages of at least 8 rows (a page segment must
// start on a 1024-byte swizzle atom).  page_rows = 0 for a contiguous cache.
inline bool supported_shape(long long B, int Hkv, int Lmax, int page_rows) {
  return n_split_max(Lmax) <= 65535 && B * Hkv <= 0x7fffffffLL &&
         (page_rows == 0 || page_rows >= 8);
}

__device__ __forceinline__ int valid_klen(const int* k_lens, int b, int Lmax, int* status,
                                          bool report) {
  int kl = __ldg(k_lens + b);
  if (kl < 0 || kl > Lmax) {
    if (report) atomicOr(status, 1);
    kl = 0;
  }
  return kl;
}

// ---------------------------------------------------------------- tensor-core split kernel
//
// One CTA per chunk of CH keys of one sequence and kv head, the two products
// on the tensor core (d = 64 or 128, contiguous or paged cache): per block of
// 128 keys,
//     S^T = K Q^T     (M = 128 keys on the TMEM lanes, N = 16 query heads
//                      padded, K = d; both operands K-major in shared memory)
//     O^T += V^T P^T  (M = d = 128 lanes, N = 16 heads, K = 128 keys; V^T is
//                      the V tile read MN-major, P is written by the softmax
//                      threads as a 16-row K-major tile)
// so the CUDA cores only form the scores' exponentials (G per key) and the
// kernel streams the cache (measured on B200, B64 Hq32 Hkv8, cache 32768,
// k_len ~ U[1024, 32768]: 6902 GB/s at d = 128 and 4900 GB/s at d = 64,
// against 6400 and 4486 GB/s for an earlier split kernel that formed both
// products on the CUDA cores, timed in the same process).  Warp 0 loads K and
// V blocks with TMA (128-byte swizzle) into a ring of three 32 KB slots, warp
// 1 issues the MMAs, warps 2-5 (one key row, then one d index, per thread) run
// the online softmax of the three-ledgers page per block with the stale-max
// threshold and write the chunk's normalised partial.  The block chain (S, softmax, PV) is serial;
// with two CTAs per SM and the next block's K and V in flight during it, the
// copies are the limit.
namespace tc {

// 4-D tiled copy global -> shared; completion counted on `bar` in bytes.
__device__ __forceinline__ void tma_load_4d(const CUtensorMap* m, uint64_t* bar, void* dst, int c0,
                                            int c1, int c2, int c3) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5, %6}], [%2];" ::"r"(sm100::smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(m)), "r"(sm100::smem_u32(bar)), "r"(c0), "r"(c1), "r"(c2),
      "r"(c3)
      : "memory");
}

constexpr int BK = 128;        // keys per block
constexpr int NH = 16;         // query heads per group, padded (the MMA's N)
constexpr int NSLOT = 3;       // ring slots (one K or V block of 32 KB each)
constexpr int SLOT = BK * 128 * 2;  // 32 KB: two 128-row x 64-column panels
constexpr int PANEL = BK * 128;     // 16 KB
constexpr int HPANEL = NH * 128;    // 2 KB: a 16-row x 64-column panel
constexpr int OFF_RING = 0;
constexpr int OFF_Q = NSLOT * SLOT;            // Q tile, 2 panels
constexpr int OFF_P = OFF_Q + 2 * HPANEL;      // P tile, 2 panels
constexpr int OFF_RED = OFF_P + 2 * HPANEL;    // [2][4 warps][NH] block maxima, [4][NH] sums
constexpr int OFF_BAR = OFF_RED + 3 * 4 * NH * 4;
constexpr int SMEM_BYTES = OFF_BAR + 256 + 1024;  // barriers + alignment slack
constexpr int NTHREADS = 6 * 32;
constexpr uint32_t IDESC_S = sm100::idesc_bf16_f32(128, NH, false, false);
constexpr uint32_t IDESC_PV = sm100::idesc_bf16_f32(128, NH, true, false);
constexpr float RESCALE_THRESHOLD = 8.0f;  // log2 units

// PAGED: the cache is [pages][kv heads][page rows][d] behind a block table;
// a 128-key block is copied as page segments of min(page, 128) rows (4-D tensor
// map), and segments past the sequence's last page are addressed at page
// n_pages, out of range, so the copy fills them with zeros.
template <int D, bool PAGED>
__global__ void __launch_bounds__(NTHREADS, 2)
    split_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                 const SplitParams p) {
  // d = 64: K and V tiles are one 64-column panel; O^T = V^T P^T still runs at
  // M = 128 over the slot's two panels, and the second (zero-filled once) only
  // feeds lanes 64-127, which are never read
  static_assert(D == 128 || D == 64, "head dimension");
  constexpr int DP = D / 64;  // 64-column panels per K or V tile
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = sm100::smem_u32(smem_raw);
  uint8_t* smem = smem_raw + ((1024 - (raw_addr & 1023)) & 1023);
  const uint32_t sbase = sm100::smem_u32(smem);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + OFF_BAR);
  uint64_t* kv_full = bars;              // [NSLOT]
  uint64_t* kv_empty = bars + NSLOT;     // [NSLOT]
  uint64_t* s_full = bars + 2 * NSLOT;
  uint64_t* p_full = s_full + 1;
  uint64_t* o_full = s_full + 2;
  uint64_t* q_ready = s_full + 3;
  uint64_t* drain = s_full + 4;
  uint64_t* mx_bar = s_full + 5;   // [2]: the softmax warps' block maxima are in
  uint64_t* sum_bar = s_full + 7;  // the softmax warps' row sums are in
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(s_full + 8);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  float* red = reinterpret_cast<float*>(smem + OFF_RED);

  // grid (sequence x kv head, chunk position counted from the sequence's end)
  const int hkv = blockIdx.x % p.Hkv, b = blockIdx.x / p.Hkv;
  const int kl = valid_klen(p.k_lens, b, p.Lmax, p.status,
                            blockIdx.y == gridDim.y - 1 && hkv == 0 && threadIdx.x == 0);
  const int chunk = (kl + CH - 1) / CH - static_cast<int>(gridDim.y - blockIdx.y);
  if (chunk < 0) return;
  const int k0 = chunk * CH;
  const int rows = min(CH, kl - k0);
  const int nblk = (rows + BK - 1) / BK;
  const int warp = threadIdx.x >> 5;
  const int head_kv = b * p.Hkv + hkv;
  const int* bt = PAGED ? p.block_table + static_cast<size_t>(b) * p.max_blocks : nullptr;
  if constexpr (PAGED) {
    // every block-table entry of this chunk is checked before any copy; a
    // chunk with a bad entry reads nothing and contributes an empty partial
    bool bad_page = false;
    const int blk1 = (k0 + rows - 1) >> p.page_log2;
    for (int bb = (k0 >> p.page_log2) + static_cast<int>(threadIdx.x); bb <= blk1; bb += NTHREADS) {
      const int pg = __ldg(bt + bb);
      if (pg < 0 || pg >= p.n_pages) bad_page = true;
    }
    if (__syncthreads_or(bad_page)) {
      if (threadIdx.x == 0) atomicOr(p.status, ATTN_DEV_BAD_PAGE);
      for (int e = threadIdx.x; e < p.G * D; e += NTHREADS) {
        const size_t ph = (static_cast<size_t>(b) * p.Hq + hkv * p.G + e / D) * p.nsm + chunk;
        p.part_o[ph * D + e % D] = 0.f;
        if (e % D == 0) p.part_lse[ph] = -INFINITY;
      }
      return;
    }
  }

  if (threadIdx.x == 0) {
    for (int i = 0; i < NSLOT; ++i) {
      sm100::mbar_init(&kv_full[i], 1);
      sm100::mbar_init(&kv_empty[i], 1);
    }
    sm100::mbar_init(s_full, 1);
    sm100::mbar_init(p_full, 4);
    sm100::mbar_init(o_full, 1);
    sm100::mbar_init(q_ready, 4);
    sm100::mbar_init(drain, 1);
    sm100::mbar_init(&mx_bar[0], 4);
    sm100::mbar_init(&mx_bar[1], 4);
    sm100::mbar_init(sum_bar, 4);
    *abort_flag = 0;
    sm100::fence_barrier_init();
  }
  if (warp == 0 && sm100::lane_id() == 0) {
    sm100::prefetch_tmap(&tmK);
    sm100::prefetch_tmap(&tmV);
  }
  if (warp == 1) {
    sm100::tmem_alloc(tmem_slot, 32);
    sm100::tmem_relinquish();
  }
  sm100::tc_fence_before();
  __syncthreads();
  sm100::tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tS = tmem, tO = tmem + NH;  // S^T: columns 0-15, O^T: 16-31

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (sm100::lane_id() == 0) {
      int issued = 0;
      for (int u = 0; u < 2 * nblk; ++u) {
        const int slot = u % NSLOT;
        if (!sm100::mbar_wait(&kv_empty[slot], ((u / NSLOT) & 1) ^ 1, abort_flag, p.status, 21))
          break;
        sm100::mbar_arrive_expect_tx(&kv_full[slot], BK * D * 2);
        ++issued;
        const int row = k0 + (u >> 1) * BK;
        if constexpr (PAGED) {
          const int page = 1 << p.page_log2;
          const int br = page < BK ? page : BK;  // rows per segment
          const int last_blk = (kl - 1) >> p.page_log2;
          for (int sg = 0; sg < BK / br; ++sg) {
            const int r = row + sg * br;
            const int blk = r >> p.page_log2;
            const int pg = blk <= last_blk ? __ldg(bt + blk) : p.n_pages;
            for (int c = 0; c < DP; ++c)
              tma_load_4d((u & 1) ? &tmV : &tmK, &kv_full[slot],
                          smem + OFF_RING + slot * SLOT + c * PANEL + sg * br * 128, c * 64,
                          r & (page - 1), hkv, pg);
          }
        } else {
          for (int c = 0; c < DP; ++c)
            sm100::tma_load_3d((u & 1) ? &tmV : &tmK, &kv_full[slot],
                               smem + OFF_RING + slot * SLOT + c * PANEL, c * 64, row, head_kv);
        }
      }
      // the CTA must not exit while copies still land in its shared memory
      for (int u = issued - 1; u >= 0 && u >= issued - NSLOT; --u)
        sm100::mbar_wait_drain(&kv_full[u % NSLOT], (u / NSLOT) & 1);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    const bool leader = sm100::elect_one();
    auto commit = [&](uint64_t* bar) {
      if (leader) sm100::tc_commit(bar);
      __syncwarp();
    };
    const uint64_t qd = sm100::sdesc_sw128(sbase + OFF_Q, 16, 1024);
    const uint64_t pd = sm100::sdesc_sw128(sbase + OFF_P, 16, 1024);
    bool ok = sm100::mbar_wait(q_ready, 0, abort_flag, p.status, 22);
    for (int j = 0; j < nblk && ok; ++j) {
      const int uk = 2 * j, uv = 2 * j + 1;
      const int ks = uk % NSLOT, vs = uv % NSLOT;
      if (!(ok = sm100::mbar_wait(&kv_full[ks], (uk / NSLOT) & 1, abort_flag, p.status, 23))) break;
      sm100::tc_fence_after();
      if (leader) {
        // S^T = K Q^T: both K-major; K steps of 16 d (32 bytes) inside a panel
        const uint64_t kd = sm100::sdesc_sw128(sbase + OFF_RING + ks * SLOT, 16, 1024);
#pragma unroll
        for (int k = 0; k < D / 16; ++k)
          sm100::mma_ss(tS, kd + static_cast<uint64_t>(((k >> 2) * PANEL + (k & 3) * 32) >> 4),
                        qd + static_cast<uint64_t>(((k >> 2) * HPANEL + (k & 3) * 32) >> 4),
                        IDESC_S, k > 0 ? 1u : 0u);
      }
      commit(s_full);
      commit(&kv_empty[ks]);
      if (!(ok = sm100::mbar_wait(p_full, j & 1, abort_flag, p.status, 24))) break;
      if (!(ok = sm100::mbar_wait(&kv_full[vs], (uv / NSLOT) & 1, abort_flag, p.status, 25))) break;
      sm100::tc_fence_after();
      if (leader) {
        // O^T += V^T P^T: A = the V tile read MN-major (64-wide d panels 16 KB
        // apart, 8-key groups 1 KB apart), B = P K-major; K steps of 16 keys
        const uint64_t vd = sm100::sdesc_sw128(sbase + OFF_RING + vs * SLOT, PANEL, 1024);
#pragma unroll
        for (int k = 0; k < BK / 16; ++k)
          sm100::mma_ss(tO, vd + static_cast<uint64_t>((k * 2048) >> 4),
                        pd + static_cast<uint64_t>(((k >> 2) * HPANEL + (k & 3) * 32) >> 4),
                        IDESC_PV, (j > 0 || k > 0) ? 1u : 0u);
      }
      commit(&kv_empty[vs]);
    }
    commit(o_full);
    // every issued MMA must complete before the tensor memory is released
    commit(drain);
    sm100::mbar_wait_drain(drain, 0);
  } else {
    // ------------------------------------------------------------ softmax (warps 2-5)
    const int t = threadIdx.x - 64;              // 0..127
    const int q = warp & 3;                      // TMEM lane quarter of this warp
    const int r = q * 32 + sm100::lane_id();     // TMEM lane: key row of the block, then d
    const uint32_t lane_base = static_cast<uint32_t>(q * 32) << 16;
    const int G = p.G;
    // Q tile (16 rows of D / 8 16-byte chunks, heads >= G zero) and the
    // constant zero rows of P (16 chunks per row: 128 keys)
    for (int e = t; e < NH * (D / 8); e += 128) {
      const int g = e / (D / 8), c16 = e % (D / 8);
      uint4 v = make_uint4(0u, 0u, 0u, 0u);
      if (g < G)
        v = __ldg(reinterpret_cast<const uint4*>(
                      p.Q + (static_cast<size_t>(b) * p.Hq + hkv * G + g) * D) + c16);
      *reinterpret_cast<uint4*>(smem + OFF_Q + (c16 >> 3) * HPANEL + g * 128 +
                                (((c16 & 7) ^ (g & 7)) << 4)) = v;
    }
    for (int e = t; e < NH * 16; e += 128) {
      const int g = e >> 4, c16 = e & 15;
      if (g >= G)
        *reinterpret_cast<uint4*>(smem + OFF_P + (c16 >> 3) * HPANEL + g * 128 + ((c16 & 7) << 4)) =
            make_uint4(0u, 0u, 0u, 0u);
    }
    if constexpr (DP == 1) {  // the second panel of every ring slot: zeros
      for (int e = t; e < NSLOT * (PANEL / 16); e += 128)
        *reinterpret_cast<uint4*>(smem + OFF_RING + (e / (PANEL / 16)) * SLOT + PANEL +
                                  (e % (PANEL / 16)) * 16) = make_uint4(0u, 0u, 0u, 0u);
    }
    sm100::fence_proxy_async_smem();
    __syncwarp();
    if (sm100::lane_id() == 0) sm100::mbar_arrive(q_ready);

    float m_use[NH], l[NH];
#pragma unroll
    for (int h = 0; h < NH; ++h) {
      m_use[h] = -INFINITY;
      l[h] = 0.f;
    }
    // this thread's P entries: row h, key r -> panel r / 64, 16-byte chunk
    // (r % 64) / 8 swizzled by the row, element r % 8
    uint8_t* p_col = smem + OFF_P + (r >> 6) * HPANEL + ((r & 7) << 1);
    const int p_chunk = (r & 63) >> 3;
    bool ok = true;
    for (int j = 0; j < nblk && ok; ++j) {
      if (!(ok = sm100::mbar_wait(s_full, j & 1, abort_flag, p.status, 26))) break;
      sm100::tc_fence_after();
      uint32_t s[NH];
      sm100::tmem_ld16(tS + lane_base, s);
      sm100::tmem_ld_wait();
      const bool valid = j * BK + r < rows;
      float v[NH];
#pragma unroll
      for (int h = 0; h < NH; ++h)
        v[h] = (valid && h < G) ? __uint_as_float(s[h]) * p.scale_log2 : -INFINITY;
      // block maxima per head: within the warp, then across the four warps
      // (through shared memory and an mbarrier, so that every wait is bounded;
      // two buffers: a warp writes block j + 2's maxima only after all four
      // warps arrived for block j + 1, i.e. after they read block j's)
      float* rw = red + (j & 1) * 4 * NH;
#pragma unroll
      for (int h = 0; h < NH; ++h) {
        float m = v[h];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        if (sm100::lane_id() == h) rw[q * NH + h] = m;
      }
      __syncwarp();
      if (sm100::lane_id() == 0) sm100::mbar_arrive(&mx_bar[j & 1]);
      if (!(ok = sm100::mbar_wait(&mx_bar[j & 1], (j >> 1) & 1, abort_flag, p.status, 28))) break;
      bool need = false;
      float mb[NH];
#pragma unroll
      for (int h = 0; h < NH; ++h) {
        mb[h] = fmaxf(fmaxf(rw[h], rw[NH + h]), fmaxf(rw[2 * NH + h], rw[3 * NH + h]));
        need |= mb[h] > m_use[h] + RESCALE_THRESHOLD;
      }
      if (need) {  // uniform: every thread saw the same maxima
        float alpha[NH];
#pragma unroll
        for (int h = 0; h < NH; ++h) {
          const float mn = fmaxf(m_use[h], mb[h]);
          alpha[h] = (m_use[h] == -INFINITY) ? 0.f : sm100::ex2(m_use[h] - mn);
          m_use[h] = mn;
          l[h] *= alpha[h];
        }
        if (j > 0) {
          // O^T holds PV of the previous blocks (complete: this block's S^T was
          // issued after them); rescale this thread's row (one d index)
          uint32_t o[NH];
          sm100::tmem_ld16(tO + lane_base, o);
          sm100::tmem_ld_wait();
#pragma unroll
          for (int h = 0; h < NH; ++h) o[h] = __float_as_uint(__uint_as_float(o[h]) * alpha[h]);
          sm100::tmem_st16(tO + lane_base, o);
          sm100::tmem_st_wait();
        }
      }
#pragma unroll
      for (int h = 0; h < NH; ++h) {
        if (h < G) {
          const float pv = (v[h] == -INFINITY) ? 0.f : sm100::ex2(v[h] - m_use[h]);
          l[h] += pv;
          *reinterpret_cast<__nv_bfloat16*>(p_col + h * 128 + ((p_chunk ^ (h & 7)) << 4)) =
              __float2bfloat16_rn(pv);
        }
      }
      sm100::fence_proxy_async_smem();
      sm100::tc_fence_before();
      __syncwarp();
      if (sm100::lane_id() == 0) sm100::mbar_arrive(p_full);
    }
    // ---- partial of the chunk: l over the 128 key rows, O^T row d = r
    if (ok) ok = sm100::mbar_wait(o_full, 0, abort_flag, p.status, 27);
    float* rs = red + 2 * 4 * NH;
#pragma unroll
    for (int h = 0; h < NH; ++h) {
      float x = l[h];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
      if (sm100::lane_id() == h) rs[q * NH + h] = x;
    }
    __syncwarp();
    if (sm100::lane_id() == 0) sm100::mbar_arrive(sum_bar);
    if (ok) ok = sm100::mbar_wait(sum_bar, 0, abort_flag, p.status, 29);
    uint32_t o[NH];
    if (ok && !*abort_flag) {
      sm100::tc_fence_after();
      sm100::tmem_ld16(tO + lane_base, o);
      sm100::tmem_ld_wait();
    }
    const bool live = ok && !*abort_flag;
#pragma unroll
    for (int h = 0; h < NH; ++h) {
      if (h >= G) break;
      const float ls = rs[h] + rs[NH + h] + rs[2 * NH + h] + rs[3 * NH + h];
      const size_t ph = (static_cast<size_t>(b) * p.Hq + hkv * G + h) * p.nsm + chunk;
      const bool has = live && ls > 0.f;
      if (r < D) p.part_o[ph * D + r] = has ? __uint_as_float(o[h]) / ls : 0.f;
      if (r == 0) p.part_lse[ph] = has ? m_use[h] + log2f(ls) : -INFINITY;
    }
  }
  sm100::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    sm100::tc_fence_after();
    sm100::tmem_dealloc(tmem, 32);
  }
}

}  // namespace tc

struct CombineParams {
  const float* part_o;
  const float* part_lse;
  const int* k_lens;
  int* status;
  __nv_bfloat16* O;
  float* lse;
  int Hq, Lmax, nsm;
};

template <int D>
__global__ void __launch_bounds__(D) decode_combine_kernel(const CombineParams p) {
  const int bh = blockIdx.x;
  const int b = bh / p.Hq;
  const int kl = valid_klen(p.k_lens, b, p.Lmax, p.status, false);
  const int n = (kl + CH - 1) / CH;
  const float* lp = p.part_lse + static_cast<size_t>(bh) * p.nsm;
  float M = -INFINITY;
  for (int c = 0; c < n; ++c) M = fmaxf(M, lp[c]);
  float wsum = 0.f, acc = 0.f;
  if (M != -INFINITY) {
    const float* op = p.part_o + static_cast<size_t>(bh) * p.nsm * D + threadIdx.x;
    for (int c = 0; c < n; ++c) {
      const float w = (lp[c] == -INFINITY) ? 0.f : sm100::ex2(lp[c] - M);
      wsum += w;
      acc += w * op[static_cast<size_t>(c) * D];
    }
  }
  p.O[static_cast<size_t>(bh) * D + threadIdx.x] = __float2bfloat16_rn(wsum > 0.f ? acc / wsum : 0.f);
  if (threadIdx.x == 0 && p.lse)
    p.lse[bh] = wsum > 0.f ? (M + log2f(wsum)) * 0.69314718055994531f : -INFINITY;
}

// The split kernel and the combine.  Measured on B200
// (B64 Hq32 Hkv8 d128, cache 32768, k_len ~ U[1024, 32768], 64-row pages in a
// random order): the paged cache reads at 6951 GB/s, the same rate as the
// contiguous cache (the earlier CUDA-core split kernel: 6066-6171 GB/s).
template <int D, bool PAGED>
cudaError_t launch_tc(const SplitParams& sp, const CombineParams& cp, cudaStream_t s) {
  CUtensorMap tk, tv;
  const long long heads = static_cast<long long>(sp.B) * sp.Hkv;
  const int page = 1 << sp.page_log2;
  const int br = page < tc::BK ? page : tc::BK;
  const bool maps =
      PAGED ? make_tmap_paged(&tk, sp.K, D, page, sp.Hkv, sp.n_pages, br) &&
                  make_tmap_paged(&tv, sp.V, D, page, sp.Hkv, sp.n_pages, br)
            : attn_bwd_impl::make_tmap_rows(&tk, sp.K, D, sp.Lmax, heads, tc::BK) &&
                  attn_bwd_impl::make_tmap_rows(&tv, sp.V, D, sp.Lmax, heads, tc::BK);
  if (!maps) return attn_host::report(cudaErrorInvalidValue, "decode tensor maps");
  auto kernel = tc::split_kernel<D, PAGED>;
  cudaError_t e = attn_host::report(attn_host::set_smem(kernel, tc::SMEM_BYTES),
                                    "decode tensor-core kernel shared-memory attribute");
  if (e != cudaSuccess) return e;
  kernel<<<dim3(static_cast<unsigned>(sp.Hkv * sp.B), sp.nsm, 1), tc::NTHREADS, tc::SMEM_BYTES,
           s>>>(tk, tv, sp);
  if ((e = attn_host::report_launch(kernel, "decode tensor-core split kernel")) != cudaSuccess)
    return e;
  decode_combine_kernel<D><<<sp.B * sp.Hq, D, 0, s>>>(cp);
  return attn_host::report_launch(decode_combine_kernel<D>, "decode_combine_kernel");
}

// Paged cache description for launch(); Lmax is then max_blocks * page.
struct PagedKV {
  const int* block_table;  // device [B][max_blocks]
  int max_blocks, page_log2, n_pages;
};

inline cudaError_t launch(const __nv_bfloat16* Q, const __nv_bfloat16* K, const __nv_bfloat16* V,
                          __nv_bfloat16* O, float* lse, int B, int Hq, int Hkv, int Lmax, int d,
                          float scale, const int* k_lens, int* status, uint8_t* scratch, int,
                          cudaStream_t s, const PagedKV* paged = nullptr) {
  SplitParams sp;
  sp.block_table = paged ? paged->block_table : nullptr;
  sp.max_blocks = paged ? paged->max_blocks : 0;
  sp.page_log2 = paged ? paged->page_log2 : 0;
  sp.n_pages = paged ? paged->n_pages : 0;
  sp.Q = Q;
  sp.K = K;
  sp.V = V;
  sp.k_lens = k_lens;
  sp.status = status;
  sp.nsm = n_split_max(Lmax);
  const size_t n = static_cast<size_t>(B) * Hq * sp.nsm;
  sp.part_o = reinterpret_cast<float*>(scratch);
  sp.part_lse = reinterpret_cast<float*>(scratch + n * d * 4);
  sp.B = B;
  sp.Hq = Hq;
  sp.Hkv = Hkv;
  sp.G = Hq / Hkv;
  sp.Lmax = Lmax;
  sp.scale_log2 = scale * 1.4426950408889634f;
  CombineParams cp;
  cp.part_o = sp.part_o;
  cp.part_lse = sp.part_lse;
  cp.k_lens = k_lens;
  cp.status = status;
  cp.O = O;
  cp.lse = lse;
  cp.Hq = Hq;
  cp.Lmax = Lmax;
  cp.nsm = sp.nsm;
  // the caller checked supported_shape()
  if (d == 128) return paged ? launch_tc<128, true>(sp, cp, s) : launch_tc<128, false>(sp, cp, s);
  return paged ? launch_tc<64, true>(sp, cp, s) : launch_tc<64, false>(sp, cp, s);
}

}  // namespace attn_decode_impl
