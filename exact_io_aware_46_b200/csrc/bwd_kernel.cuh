// bwd_kernel.cuh -- attention backward by recomputation on sm_100a.
//
// "FlashAttention and long context: three ledgers" (online-softmax
// section) states the backward keeps only small per-row statistics and
// recomputes the score blocks it needs, trading compute for memory traffic.
// With the saved LSE (and D_i = sum_d dO_id O_id) every score tile is rebuilt
// as P = exp(S * scale - LSE); the gradients are the calculus of the
// definition:
//     dV = P^T dO ; dP = dO V^T ; dS = P o (dP - D) ;
//     dK = scale dS^T Q ; dQ = scale dS K.
//
// B200 design.  Three launches:
//  1. prep: D per query row, LSE in log2 units (+inf for rows without a
//     visible key or past Lq, so their P is exactly 0), and a zeroed fp32 dQ
//     accumulator; rows are padded to a multiple of 128 per head.
//  2. main (persistent, one CTA per SM): a work item is one 128-key tile of one
//     (batch, key/value head).  K and V stay in shared memory while the item
//     walks every 128-row query tile of every query head of the group that can
//     see the keys.  Per query tile the tensor core computes, with keys on the
//     128 TMEM lanes and every MMA at M = 128, N = 128,
//        S^T  = K Q^T          (SS)        dP^T = V dO^T        (SS)
//        dV  += P^T dO         (TS: P^T from TMEM, written by the softmax)
//        dQ^T = K^T dS^T       (SS, both operands MN-major)
//        dK  += dS^T Q         (SS: dS^T staged in shared memory)
//     dV and dK accumulate in TMEM across the item (256 columns); S^T/P^T and
//     dP^T take the other 256, and dQ^T reuses the dP^T columns once dS has
//     been formed.  Tensor memory holds one query tile at a time, so the
//     issue order S^T(t), dK(t-1), dP^T(t), dV(t), dQ^T(t), S^T(t+1), dK(t), ...
//     gives each hand-off one MMA group of cover: P(t) forms while dK(t-1) and
//     dP^T(t) run, dS(t) while dV(t) runs, and the drain of dQ^T(t) while
//     S^T(t+1) and dK(t) run.  Warps 0-7 form P and dS (one key row per thread,
//     two warps per row, 64 query rows each), warps 8-11 drain dQ^T into the
//     fp32 accumulator (d = 128: coalesced reductions and bulk reduce-adds;
//     d = 64: tensor reduce-adds), warp 12 feeds TMA, warp 13 issues MMAs.
//  3. convert: dQ = bf16(scale * accumulator).
#pragma once

#include "launch_cache.cuh"
#include "sm100.cuh"

namespace attn_bwd_impl {

constexpr int BN = 128;   // keys per work item (TMEM lanes)
constexpr int BMQ = 128;  // query rows per query tile
constexpr int NQS = 2;    // query-tile ring stages (Q with its log2-LSE and D); dO is single-buffered
constexpr int NSMX = 8;   // P/dS warps: 4 lane quarters x 2 halves of the query rows
constexpr int W_DRAIN = NSMX;        // warps 8-11: dQ drain
constexpr int W_LOAD = NSMX + 4;     // warp 12: TMA producer
constexpr int W_MMA = NSMX + 5;      // warp 13: MMA issuer
constexpr int NTHREADS = 32 * (NSMX + 6);
constexpr int NI = 4;                          // depth of the shared-memory item ring
constexpr int ITEM_READERS = NSMX + 4 + 1;     // warps that read each item: P/dS, drain, MMA
constexpr int PANEL = 16384;  // one 128-byte-swizzled panel: 128 rows x 64 bf16 columns
constexpr int DQ_ROWS = 32;   // query rows per dQ staging round (16 KB of fp32 at d = 128)

// Layout for head dimension DH (64 or 128): shared memory map (bytes; the
// swizzled panels are 1024-byte aligned; a 128-row tile is DH / 64 panels) and
// the instruction descriptors whose N is the head dimension.
template <int DH>
struct Cfg {
  static_assert(DH == 64 || DH == 128, "head dimension");
  static constexpr int PANELS = DH / 64;
  static constexpr int TILE = PANELS * PANEL;     // one 128-row bf16 tile
  static constexpr int OFF_K = 0;                 // [128 keys][d]
  static constexpr int OFF_V = TILE;
  static constexpr int OFF_Q = 2 * TILE;          // NQS stages of [128 rows][d]
  static constexpr int OFF_DO = OFF_Q + NQS * TILE;  // [128 rows][d]
  static constexpr int OFF_DS = OFF_DO + TILE;    // dS^T [128 keys][128 rows]: panels of 64 rows
  // d = 128: dQ^T (lanes = d) is staged row-major DQ_ROWS query rows at a time
  // for bulk reduce-adds; d = 64: the tile's dQ (lanes = query rows) is staged
  // as two 128-byte-swizzled boxes of 32 columns for tensor reduce-adds
  static constexpr bool STAGED_DQ = DH == 128;
  static constexpr int OFF_DQ = OFF_DS + 2 * PANEL;  // 1024-byte aligned
  static constexpr int DQ_STAGE = STAGED_DQ ? DQ_ROWS * DH * 4 : BMQ * DH * 4;
  static constexpr int OFF_LD = OFF_DQ + DQ_STAGE;  // lse2 [128], D [128]
  static constexpr int OFF_BAR = OFF_LD + NQS * 1024;
  static constexpr int SMEM_BYTES = OFF_BAR + 256 + 1024;  // barriers + alignment slack
  static_assert(SMEM_BYTES <= 232448, "dynamic shared memory limit");
  // dV += P^T dO and dK += dS^T Q (A K-major, B MN-major); dQ^T = K^T dS^T
  // (M = d = 128, N = 128 rows) or dQ = dS K (M = 128 rows, N = d = 64), both
  // operands MN-major
  static constexpr uint32_t IDESC_DV = sm100::idesc_bf16_f32(128, DH, false, true);
  static constexpr uint32_t IDESC_DQ = STAGED_DQ ? sm100::idesc_bf16_f32(128, BMQ, true, true)
                                                 : sm100::idesc_bf16_f32(128, DH, true, true);
};

// TMEM columns (512 allocated)
constexpr uint32_t S_COL = 0;     // S^T, overwritten by P^T (packed bf16) -- 128
constexpr uint32_t DP_COL = 128;  // dP^T, then dQ of the same tile -- 128 (DH of them for dQ)
constexpr uint32_t DV_COL = 256;  // DH columns
constexpr uint32_t DK_COL = 384;  // DH columns

constexpr uint32_t IDESC_S = sm100::idesc_bf16_f32(128, BMQ, false, false);

// Exponentials on the FMA pipe (polynomial exp2) for column pairs cp with
// (cp & 7) >= POLY_FROM: the 16384 exponentials of a tile take 1024 cycles on
// the special-function unit alone, more than the one MMA group (~690 cycles)
// that covers the forming of P.
constexpr int POLY_FROM = 5;

// 32-byte global store of eight 32-bit words; the address must be 32-byte aligned.
__device__ __forceinline__ void st_global_v8(void* p, const uint32_t* v) {
  asm volatile("st.global.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(p), "r"(v[0]),
               "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7])
               : "memory");
}

struct Args {
  const __nv_bfloat16 *Q, *K, *V, *O, *dO;
  const float* lse;
  __nv_bfloat16 *dQ, *dK, *dV;
  int B, Hq, Hkv, Lq, Lk, d;
  float scale;
  int causal;
  int window;  // > 0: sliding window (with causal)
  const int* k_lens;
  int* status;
  uint8_t* scratch;
  int sms;
};

inline int lq_pad(int Lq) { return ((Lq > 0 ? Lq : 1) + BMQ - 1) / BMQ * BMQ; }

inline size_t scratch_bytes(int B, int Hq, int, int Lq, int, int d) {
  const size_t rows = static_cast<size_t>(B) * Hq * lq_pad(Lq);
  size_t bytes = rows * d * 4 + rows * 8;
  return (bytes + 255) & ~static_cast<size_t>(255);
}

struct Params {
  float* dq_acc;       // [B*Hq][Lqp][d] fp32
  const float* lse2;   // [B*Hq][Lqp]
  const float* Dvec;   // [B*Hq][Lqp]
  __nv_bfloat16* dK;
  __nv_bfloat16* dV;
  const int* k_lens;
  int* status;
  int B, Hq, Hkv, G, Lq, Lk, Lqp;
  float scale, scale_log2;
  int causal;
  int window;  // > 0: a query row sees only its `window` latest keys
  int n_kv;     // ceil(Lk / 128)
  int n_qt;     // Lqp / BMQ
  int n_items;  // B * Hkv * n_kv
  int* sched;   // [0] next dynamic item, [1] finished CTAs (workspace header)
};

struct Item {
  int b, hkv, n, kv_len, i_lo, T;  // T = query tiles visited (over the group's heads)
};

// Item order: groups of KV_HEAD_GROUP (batch, kv head) pairs; inside a group
// the earliest key tiles first (they are seen by the most query rows, so the
// static round-robin starts with the heaviest items), heads interleaved.  The
// group's Q, dO and dQ accumulator (8 MB per head at L = 8192, d = 128) stay
// L2-resident while all of its key tiles stream past them; visiting one key
// tile of every head at a time did not fit L2 (52 % hit rate).
constexpr int KV_HEAD_GROUP = 4;

__device__ __forceinline__ Item get_item(const Params& p, int w, bool* bad) {
  Item it;
  const int BH = p.B * p.Hkv;
  const int per_group = KV_HEAD_GROUP * p.n_kv;
  const int grp = w / per_group;
  const int r = w % per_group;
  const int gsize = min(KV_HEAD_GROUP, BH - grp * KV_HEAD_GROUP);
  it.n = r / gsize;
  const int bh = grp * KV_HEAD_GROUP + r % gsize;
  it.b = bh / p.Hkv;
  it.hkv = bh % p.Hkv;
  int kl = p.Lk;
  if (p.k_lens) {
    kl = __ldg(p.k_lens + it.b);
    if (kl < 0 || kl > p.Lk) {
      if (bad) *bad = true;
      kl = 0;
    }
  }
  it.kv_len = kl;
  const int k0 = it.n * BN;
  it.i_lo = 0;
  it.T = 0;
  if (k0 >= kl || p.Lq == 0) return it;
  int r_min = 0;
  if (p.causal) r_min = max(0, k0 - (p.Lk - p.Lq));  // first row that sees key k0
  if (r_min >= p.Lq) return it;
  it.i_lo = r_min / BMQ;
  int i_end = (p.Lq + BMQ - 1) / BMQ;  // one past the last query tile
  if (p.window > 0) {
    // the last row that sees a key of this tile: i + off - W < k0 + BN - 1
    const int r_max = k0 + BN - 2 - (p.Lk - p.Lq) + p.window;
    if (r_max < r_min) return it;
    i_end = min(i_end, r_max / BMQ + 1);
  }
  it.T = p.G * (i_end - it.i_lo);
  return it;
}

// The t-th query tile an item visits: query head g of the group and query tile i.
__device__ __forceinline__ void tile_of(const Item& it, int t, int nq, int& g, int& i) {
  g = t / nq;
  i = it.i_lo + t % nq;
}

// Bulk reduce-add of `bytes` fp32 values from shared to global memory (the
// TMA unit performs the additions at L2), tracked by a bulk async-group.
__device__ __forceinline__ void bulk_reduce_add_f32(float* gdst, const void* ssrc, uint32_t bytes) {
  asm volatile(
      "cp.reduce.async.bulk.global.shared::cta.bulk_group.add.f32 [%0], [%1], %2;" ::"l"(
          reinterpret_cast<uint64_t>(gdst)),
      "r"(sm100::smem_u32(ssrc)), "r"(bytes)
      : "memory");
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
// Waits until the shared-memory sources of all committed bulk groups were read.
__device__ __forceinline__ void bulk_wait_read_all() {
  asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}
// Waits until all committed bulk groups completed (writes visible).
__device__ __forceinline__ void bulk_wait_all() {
  asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}

// acc[0] += a: one 4-byte reduction, performed at L2 (the 32 lanes of a warp
// cover 128 contiguous bytes, so the request is coalesced).
__device__ __forceinline__ void red_add_f32(float* acc, float a) {
  asm volatile("red.global.add.f32 [%0], %1;" ::"l"(acc), "f"(a) : "memory");
}


// Tensor reduce-add of one shared-memory box into global memory through the
// tensor map `m` at coordinates (c0, c1, c2); the TMA unit performs the
// additions at L2.  Tracked by the calling thread's bulk async-group.
__device__ __forceinline__ void tma_reduce_add_3d(const CUtensorMap* m, const void* ssrc, int c0,
                                                  int c1, int c2) {
  asm volatile(
      "cp.reduce.async.bulk.tensor.3d.global.shared::cta.add.tile.bulk_group"
      " [%0, {%2, %3, %4}], [%1];" ::"l"(reinterpret_cast<uint64_t>(m)),
      "r"(sm100::smem_u32(ssrc)), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}

__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes,
                                         uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          sm100::smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(sm100::smem_u32(bar))
      : "memory");
}

// ------------------------------------------------------------------ prep

template <int DH>
__global__ void __launch_bounds__(256) bwd_prep_kernel(const __nv_bfloat16* O,
                                                        const __nv_bfloat16* dO,
                                                        const float* lse, float* dq_acc,
                                                        float* lse2, float* Dv, int BH, int Lq,
                                                        int Lqp) {
  constexpr int EPL = DH / 32;  // elements per lane
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (warp >= BH * Lqp) return;
  const int bh = warp / Lqp, r = warp % Lqp;
  float acc = 0.f;
  if (r < Lq) {
    const size_t off = (static_cast<size_t>(bh) * Lq + r) * DH + lane * EPL;
    uint32_t a[EPL / 2], g[EPL / 2];
    if constexpr (EPL == 4) {
      const uint2 ta = *reinterpret_cast<const uint2*>(O + off);
      const uint2 tg = *reinterpret_cast<const uint2*>(dO + off);
      a[0] = ta.x; a[1] = ta.y; g[0] = tg.x; g[1] = tg.y;
    } else {
      a[0] = *reinterpret_cast<const uint32_t*>(O + off);
      g[0] = *reinterpret_cast<const uint32_t*>(dO + off);
    }
#pragma unroll
    for (int e = 0; e < EPL / 2; ++e)
      acc += __uint_as_float(a[e] << 16) * __uint_as_float(g[e] << 16) +
             __uint_as_float(a[e] & 0xFFFF0000u) * __uint_as_float(g[e] & 0xFFFF0000u);
  }
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  float* zrow = dq_acc + static_cast<size_t>(warp) * DH + lane * EPL;
  if constexpr (EPL == 4)
    *reinterpret_cast<float4*>(zrow) = make_float4(0.f, 0.f, 0.f, 0.f);
  else
    *reinterpret_cast<float2*>(zrow) = make_float2(0.f, 0.f);
  if (lane == 0) {
    Dv[warp] = acc;
    float l2 = INFINITY;
    if (r < Lq) {
      const float l = lse[static_cast<size_t>(bh) * Lq + r];
      l2 = (l == -INFINITY) ? INFINITY : l * 1.4426950408889634f;
    }
    lse2[warp] = l2;
  }
}

template <int DH>
__global__ void __launch_bounds__(256) bwd_dq_convert_kernel(const float* dq_acc,
                                                              __nv_bfloat16* dQ, int BH, int Lq,
                                                              int Lqp, float scale) {
  const size_t i = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x;  // 4 elements
  const size_t total = static_cast<size_t>(BH) * Lq * (DH / 4);
  if (i >= total) return;
  const size_t row = i / (DH / 4);
  const int c4 = static_cast<int>(i % (DH / 4));
  const int bh = static_cast<int>(row / Lq), r = static_cast<int>(row % Lq);
  const float4 v =
      reinterpret_cast<const float4*>(dq_acc + (static_cast<size_t>(bh) * Lqp + r) * DH)[c4];
  uint2 o;
  o.x = sm100::pack_bf16x2(v.x * scale, v.y * scale);
  o.y = sm100::pack_bf16x2(v.z * scale, v.w * scale);
  reinterpret_cast<uint2*>(dQ + row * DH)[c4] = o;
}

// ------------------------------------------------------------------ main

template <int DH>
__global__ void __launch_bounds__(NTHREADS, 1)
    bwd_main_kernel(const __grid_constant__ CUtensorMap tmQ,
                    const __grid_constant__ CUtensorMap tmdO,
                    const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV,
                    const __grid_constant__ CUtensorMap tmAcc, const Params p) {
  using C = Cfg<DH>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = sm100::smem_u32(smem_raw);
  uint8_t* smem = smem_raw + ((1024 - (raw_addr & 1023)) & 1023);
  const uint32_t sbase = sm100::smem_u32(smem);

  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* kv_full = bars + 0;
  uint64_t* kv_empty = bars + 1;
  uint64_t* q_full = bars + 2;     // [NQS]
  uint64_t* q_empty = bars + 4;    // [NQS]
  uint64_t* do_full = bars + 6;
  uint64_t* do_empty = bars + 7;
  uint64_t* s_full = bars + 8;
  uint64_t* p_full = bars + 9;
  uint64_t* dp_full = bars + 10;
  uint64_t* ds_full = bars + 11;
  uint64_t* dq_full = bars + 12;
  uint64_t* dq_empty = bars + 13;
  uint64_t* dkv_full = bars + 14;
  uint64_t* dkv_empty = bars + 15;
  uint64_t* drain = bars + 16;
  uint64_t* item_full = bars + 17;   // [NI]
  uint64_t* item_empty = bars + 21;  // [NI]
  int* item_ring = reinterpret_cast<int*>(bars + 25);  // [NI]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(item_ring + NI);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  if (threadIdx.x == 0) {
    sm100::mbar_init(kv_full, 1);
    sm100::mbar_init(kv_empty, 1);
    for (int s = 0; s < NQS; ++s) {
      sm100::mbar_init(&q_full[s], 1);
      sm100::mbar_init(&q_empty[s], 1);
    }
    sm100::mbar_init(do_full, 1);
    sm100::mbar_init(do_empty, 1);
    sm100::mbar_init(s_full, 1);
    sm100::mbar_init(p_full, NSMX);
    sm100::mbar_init(dp_full, 1);
    sm100::mbar_init(ds_full, NSMX);
    sm100::mbar_init(dq_full, 1);
    sm100::mbar_init(dq_empty, 4);
    sm100::mbar_init(dkv_full, 1);
    sm100::mbar_init(dkv_empty, NSMX);
    sm100::mbar_init(drain, 1);
    for (int i = 0; i < NI; ++i) {
      sm100::mbar_init(&item_full[i], 1);
      sm100::mbar_init(&item_empty[i], ITEM_READERS);
    }
    *abort_flag = 0;
    sm100::fence_barrier_init();
  }
  if (warp == W_LOAD && sm100::lane_id() == 0) {
    sm100::prefetch_tmap(&tmQ);
    sm100::prefetch_tmap(&tmdO);
    sm100::prefetch_tmap(&tmK);
    sm100::prefetch_tmap(&tmV);
    if constexpr (!C::STAGED_DQ) sm100::prefetch_tmap(&tmAcc);
  }
  if (warp == W_MMA) {
    sm100::tmem_alloc(tmem_slot, 512);
    sm100::tmem_relinquish();
  }
  sm100::tc_fence_before();
  __syncthreads();
  sm100::tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int off = p.Lk - p.Lq;  // bottom-right causal alignment
  // a consumer warp's view of the item ring: the k-th item of this CTA, or -1
  // at the end (one arrival per warp; the caller's whole warp calls this)
  auto next_item = [&](uint32_t k, int& w) -> bool {
    if (!sm100::mbar_wait(&item_full[k % NI], (k / NI) & 1, abort_flag, p.status)) return false;
    w = *reinterpret_cast<volatile int*>(&item_ring[k % NI]);
    __syncwarp();
    if (sm100::lane_id() == 0) sm100::mbar_arrive(&item_empty[k % NI]);
    return true;
  };
  if (warp == W_LOAD) {
    // ------------------------------------------------------------ TMA producer
    // per query tile: Q (+ its log2-LSE and D) into the two-stage ring, then dO
    // into its single buffer (free once dV of the previous tile has run)
    if (sm100::lane_id() == 0) {
      uint32_t tq = 0, ik = 0;
      int last_q[NQS] = {-1, -1}, last_do = -1;  // last tile whose copies were issued
      uint32_t kv_issued = 0;
      bool ok = true;
      for (; ok; ++ik) {
        // dynamic scheduling: the CTA's first item is its index, the others
        // come from the counter in the workspace (heaviest items first)
        if (!(ok = sm100::mbar_wait(&item_empty[ik % NI], ((ik / NI) & 1) ^ 1, abort_flag,
                                    p.status)))
          break;
        int w = (ik == 0) ? static_cast<int>(blockIdx.x)
                          : atomicAdd(p.sched, 1) + static_cast<int>(gridDim.x);
        if (w >= p.n_items) w = -1;
        *reinterpret_cast<volatile int*>(&item_ring[ik % NI]) = w;
        sm100::mbar_arrive(&item_full[ik % NI]);
        if (w < 0) break;
        const Item it = get_item(p, w, nullptr);
        if (!(ok = sm100::mbar_wait(kv_empty, (ik & 1) ^ 1, abort_flag, p.status))) break;
        sm100::mbar_arrive_expect_tx(kv_full, 2 * C::TILE);
        ++kv_issued;
        const int kvh = it.b * p.Hkv + it.hkv;
        for (int c = 0; c < C::PANELS; ++c) {
          sm100::tma_load_3d(&tmK, kv_full, smem + C::OFF_K + c * PANEL, c * 64, it.n * BN, kvh);
          sm100::tma_load_3d(&tmV, kv_full, smem + C::OFF_V + c * PANEL, c * 64, it.n * BN, kvh);
        }
        const int nq = it.T > 0 ? it.T / p.G : 0;
        for (int t = 0; t < it.T && ok; ++t, ++tq) {
          int g, i;
          tile_of(it, t, nq, g, i);
          const int slot = tq % NQS;
          const int qh = it.b * p.Hq + it.hkv * p.G + g;
          if (!(ok = sm100::mbar_wait(&q_empty[slot], ((tq / NQS) & 1) ^ 1, abort_flag,
                                      p.status)))
            break;
          sm100::mbar_arrive_expect_tx(&q_full[slot], C::TILE + 1024);
          for (int c = 0; c < C::PANELS; ++c)
            sm100::tma_load_3d(&tmQ, &q_full[slot], smem + C::OFF_Q + slot * C::TILE + c * PANEL,
                               c * 64, i * BMQ, qh);
          const size_t rowoff = static_cast<size_t>(qh) * p.Lqp + i * BMQ;
          bulk_g2s(smem + C::OFF_LD + slot * 1024, p.lse2 + rowoff, 512, &q_full[slot]);
          bulk_g2s(smem + C::OFF_LD + slot * 1024 + 512, p.Dvec + rowoff, 512, &q_full[slot]);
          last_q[slot] = static_cast<int>(tq);
          if (!(ok = sm100::mbar_wait(do_empty, (tq & 1) ^ 1, abort_flag, p.status))) break;
          sm100::mbar_arrive_expect_tx(do_full, C::TILE);
          for (int c = 0; c < C::PANELS; ++c)
            sm100::tma_load_3d(&tmdO, do_full, smem + C::OFF_DO + c * PANEL, c * 64, i * BMQ, qh);
          last_do = static_cast<int>(tq);
        }
      }
      // the CTA must not exit while tensor copies still land in its shared
      // memory, which an expired wait elsewhere could otherwise allow: wait
      // (bounded) for the last issued phase of every load barrier (in normal
      // operation the consumers have already waited for all of them)
      if (kv_issued > 0) sm100::mbar_wait_drain(kv_full, (kv_issued - 1) & 1);
      for (int sl = 0; sl < NQS; ++sl)
        if (last_q[sl] >= 0) sm100::mbar_wait_drain(&q_full[sl], (last_q[sl] / NQS) & 1);
      if (last_do >= 0) sm100::mbar_wait_drain(do_full, last_do & 1);
    }
  } else if (warp == W_MMA) {
    // ------------------------------------------------------------ MMA issuer
    // The whole warp runs the loop (warp-uniform values stay in uniform
    // registers) and one elected lane issues; descriptors are built once per
    // operand and stepped by constant offsets.  MMA issue is close to
    // synchronous, so scalar work between two MMAs idles the tensor pipe.
    const bool leader = sm100::elect_one();
    {
      uint32_t tq = 0, ik = 0;
      bool ok = true;
      const uint32_t kA = sbase + C::OFF_K, vA = sbase + C::OFF_V;
      const uint32_t doA = sbase + C::OFF_DO, dsA = sbase + C::OFF_DS;
      auto qA = [&](int slot) { return sbase + C::OFF_Q + slot * C::TILE; };
      auto commit = [&](uint64_t* bar) {
        if (leader) sm100::tc_commit(bar);
        __syncwarp();
      };
      // S^T (or dP^T) = A_keys[128 x d] * B_rows[128 x d]^T, both K-major
      auto issue_kmajor = [&](uint32_t dcol, uint32_t a, uint32_t b) {
        const uint64_t ad = sm100::sdesc_sw128(a, 16, 1024);
        const uint64_t bd = sm100::sdesc_sw128(b, 16, 1024);
        if (leader) {
#pragma unroll
          for (int k = 0; k < DH / 16; ++k) {
            const uint64_t o = static_cast<uint64_t>(((k >> 2) * PANEL + (k & 3) * 32) >> 4);
            sm100::mma_ss(tmem + dcol, ad + o, bd + o, IDESC_S, k > 0);
          }
        }
      };
      const uint64_t kd_mn = sm100::sdesc_sw128(kA, PANEL, 1024);   // K: MN-major B over d
      const uint64_t do_mn = sm100::sdesc_sw128(doA, PANEL, 1024);  // dO: MN-major B over d
      const uint64_t ds_k = sm100::sdesc_sw128(dsA, 16, 1024);      // dS^T: K-major A over rows
      const uint64_t ds_mn = sm100::sdesc_sw128(dsA, PANEL, 1024);  // dS: MN-major A over rows
      for (; ok; ++ik) {
        int w;
        if (!(ok = next_item(ik, w)) || w < 0) break;
        const Item it = get_item(p, w, nullptr);
        if (!(ok = sm100::mbar_wait(kv_full, ik & 1, abort_flag, p.status))) break;
        sm100::tc_fence_after();
        if (it.T == 0) {
          if (!(ok = sm100::mbar_wait(dkv_empty, (ik & 1) ^ 1, abort_flag, p.status))) break;
          commit(dkv_full);
          commit(kv_empty);
          continue;
        }
        {  // S^T of the item's first query tile
          const int slot = tq % NQS;
          if (!(ok = sm100::mbar_wait(&q_full[slot], (tq / NQS) & 1, abort_flag, p.status)))
            break;
          sm100::tc_fence_after();
          issue_kmajor(S_COL, kA, qA(slot));
          commit(s_full);
        }
        // Issue order, one MMA group each (dK of a tile is issued one tile late):
        //   S^T(t) | dK(t-1) | dP^T(t) | dV(t) [P(t)] | dQ^T(t) [dS(t)] | S^T(t+1) ...
        // P(t) forms while dK(t-1) and dP^T(t) run, dS(t) while dV(t) runs, and
        // the drain of dQ^T(t) has S^T(t+1) and dK(t) to hand the dP^T columns
        // back.  dS^T(t) is read by dQ^T(t) and dK(t) before dP^T(t+1) is
        // issued, so one shared-memory buffer serves every tile.
        auto issue_dk = [&](uint32_t tile, bool first) {
          const uint64_t q_mn = sm100::sdesc_sw128(qA(tile % NQS), PANEL, 1024);
          if (leader) {
#pragma unroll
            for (int k = 0; k < BMQ / 16; ++k)
              sm100::mma_ss(tmem + DK_COL, ds_k + ((((k >> 2) * PANEL) + (k & 3) * 32) >> 4),
                            q_mn + ((k * 2048) >> 4), C::IDESC_DV, (!first || k > 0) ? 1u : 0u);
          }
          commit(&q_empty[tile % NQS]);
        };
        for (int t = 0; t < it.T && ok; ++t) {
          const uint32_t cur = tq + t;
          const uint32_t par = cur & 1;
          if (t > 0) issue_dk(cur - 1, t == 1);
          // dP^T(t) = V dO^T: needs dO(t) and the dP^T columns back from the
          // drain of the previous tile's dQ^T
          if (!(ok = sm100::mbar_wait(do_full, par, abort_flag, p.status))) break;
          if (!(ok = sm100::mbar_wait(dq_empty, par ^ 1, abort_flag, p.status))) break;
          sm100::tc_fence_after();
          issue_kmajor(DP_COL, vA, doA);
          commit(dp_full);
          // dV += P^T dO : A = P^T (TMEM, packed bf16: query rows 0-63 in columns
          // 0-31, rows 64-127 from column 64 on), B = dO (MN-major)
          if (!(ok = sm100::mbar_wait(p_full, par, abort_flag, p.status))) break;
          if (t == 0 && !(ok = sm100::mbar_wait(dkv_empty, (ik & 1) ^ 1, abort_flag, p.status)))
            break;
          sm100::tc_fence_after();
          if (leader) {
#pragma unroll
            for (int k = 0; k < BMQ / 16; ++k)
              sm100::mma_ts(tmem + DV_COL, tmem + S_COL + (k >> 2) * 64 + (k & 3) * 8,
                            do_mn + ((k * 2048) >> 4), C::IDESC_DV, (t > 0 || k > 0) ? 1u : 0u);
          }
          commit(do_empty);
          // into the dP^T columns: d = 128, dQ^T = K^T dS^T (lanes = d; A = K^T,
          // B = dS^T, both MN-major); d = 64, dQ = dS K (lanes = query rows;
          // A = dS, B = K, both MN-major)
          if (!(ok = sm100::mbar_wait(ds_full, par, abort_flag, p.status))) break;
          sm100::tc_fence_after();
          if (leader) {
#pragma unroll
            for (int k = 0; k < BN / 16; ++k) {
              const uint64_t kk = kd_mn + ((k * 2048) >> 4), dd = ds_mn + ((k * 2048) >> 4);
              if constexpr (C::STAGED_DQ)
                sm100::mma_ss(tmem + DP_COL, kk, dd, C::IDESC_DQ, k > 0 ? 1u : 0u);
              else
                sm100::mma_ss(tmem + DP_COL, dd, kk, C::IDESC_DQ, k > 0 ? 1u : 0u);
            }
          }
          commit(dq_full);
          // S^T of the next query tile (P^T of this one was read by dV above)
          if (t + 1 < it.T) {
            const int ns = (cur + 1) % NQS;
            if (!(ok = sm100::mbar_wait(&q_full[ns], ((cur + 1) / NQS) & 1, abort_flag,
                                        p.status)))
              break;
            sm100::tc_fence_after();
            issue_kmajor(S_COL, kA, qA(ns));
            commit(s_full);
          }
        }
        if (!ok) break;
        issue_dk(tq + it.T - 1, it.T == 1);  // the item's last dK
        if (!ok) break;
        tq += it.T;
        commit(dkv_full);
        commit(kv_empty);
      }
      commit(drain);
      sm100::mbar_wait_drain(drain, 0);
    }
  } else if (warp < NSMX) {
    // ------------------------------------------------------------ P and dS
    // one key row per thread (= TMEM lane); the two warps of a lane quarter
    // take query rows [0, 64) and [64, 128) of the tile
    const int qd = warp & 3, hf = warp >> 2;
    const int kl_ = qd * 32 + sm100::lane_id();  // key row within the tile = TMEM lane
    const uint32_t lane_base = static_cast<uint32_t>(qd * 32) << 16;
    const uint32_t s_addr = tmem + lane_base + S_COL + 64 * hf;
    const uint32_t dp_addr = tmem + lane_base + DP_COL + 64 * hf;
    uint32_t tq = 0, ik = 0;
    bool ok = true;
    for (; ok; ++ik) {
      int w;
      if (!(ok = next_item(ik, w)) || w < 0) break;
      bool bad = false;
      const Item it = get_item(p, w, &bad);
      if (bad && threadIdx.x == 0) atomicOr(p.status, 1);
      const int key = it.n * BN + kl_;
      const int lim = it.kv_len - 1;  // last visible key (padding)
      const int nq = it.T > 0 ? it.T / p.G : 0;
      for (int t = 0; t < it.T && ok; ++t) {
        const uint32_t cur = tq + t;
        const int slot = cur % NQS;
        const uint32_t par = cur & 1;
        int g_unused, i;
        tile_of(it, t, nq, g_unused, i);
        const float* l2s = reinterpret_cast<const float*>(smem + C::OFF_LD + slot * 1024) + 64 * hf;
        const float* dsv = l2s + 128;
        // lse2 / D of this tile were delivered on q_full
        if (!(ok = sm100::mbar_wait(&q_full[slot], (cur / NQS) & 1, abort_flag, p.status)))
          break;
        if (!(ok = sm100::mbar_wait(s_full, par, abort_flag, p.status))) break;
        sm100::tc_fence_after();
        // P = exp2(S scale log2(e) - lse2), kept as packed bf16 pairs (the
        // precision dV uses; dS is formed from the same values)
        uint32_t pk[32];
        {
          // key visible to query row r0 + c iff key <= lim, c >= cmin and
          // (sliding window) c <= cmax
          const int r0 = i * BMQ + 64 * hf;
          const bool key_ok = key <= lim;
          const int cmin = p.causal ? key - r0 - off : -1;
          const int cmax = p.window > 0 ? key - off + p.window - 1 - r0 : 64;
          // whole half-tile visible: no per-element test (warp-uniform; usual case)
          const bool all_vis = __all_sync(0xffffffffu, key_ok && cmin <= 0 && cmax >= 63);
          const float4* l2v = reinterpret_cast<const float4*>(l2s);
          const float2 sl2x2 = make_float2(p.scale_log2, p.scale_log2);
#pragma unroll
          for (int h2 = 0; h2 < 2; ++h2) {  // 32 columns at a time (register pressure)
            uint32_t s[32];
            sm100::tmem_ld32(s_addr + 32 * h2, s);
            sm100::tmem_ld_wait();
            if (!all_vis) {
#pragma unroll
              for (int c = 0; c < 32; ++c) {
                const int cc = 32 * h2 + c;
                if (!key_ok || cc < cmin || cc > cmax) s[c] = __float_as_uint(-INFINITY);
              }
            }
#pragma unroll
            for (int c4 = 0; c4 < 8; ++c4) {
              const float4 lq = l2v[8 * h2 + c4];
              const float2 x0 = __ffma2_rn(
                  make_float2(__uint_as_float(s[4 * c4]), __uint_as_float(s[4 * c4 + 1])), sl2x2,
                  make_float2(-lq.x, -lq.y));
              const float2 x1 = __ffma2_rn(
                  make_float2(__uint_as_float(s[4 * c4 + 2]), __uint_as_float(s[4 * c4 + 3])),
                  sl2x2, make_float2(-lq.z, -lq.w));
              const int cp = 16 * h2 + 2 * c4;  // column pair index of x0
              float2 e0, e1;
              if ((cp & 7) >= POLY_FROM) {
                e0 = sm100::ex2_poly2(x0);
              } else {
                e0.x = sm100::ex2(x0.x);
                e0.y = sm100::ex2(x0.y);
              }
              if (((cp + 1) & 7) >= POLY_FROM) {
                e1 = sm100::ex2_poly2(x1);
              } else {
                e1.x = sm100::ex2(x1.x);
                e1.y = sm100::ex2(x1.y);
              }
              pk[cp] = sm100::pack_bf16x2(e0.x, e0.y);
              pk[cp + 1] = sm100::pack_bf16x2(e1.x, e1.y);
            }
          }
        }
        sm100::tmem_st32(s_addr, pk);
        sm100::tmem_st_wait();
        sm100::tc_fence_before();
        __syncwarp();
        if (sm100::lane_id() == 0) sm100::mbar_arrive(p_full);

        // dS = P o (dP - D), written K-major (row-contiguous per key) to panel hf
        if (!(ok = sm100::mbar_wait(dp_full, par, abort_flag, p.status))) break;
        sm100::tc_fence_after();
        uint8_t* line = smem + C::OFF_DS + hf * PANEL + kl_ * 128;
        const float4* dvv = reinterpret_cast<const float4*>(dsv);
#pragma unroll
        for (int h2 = 0; h2 < 2; ++h2) {
          uint32_t dp[32];
          sm100::tmem_ld32(dp_addr + 32 * h2, dp);
          sm100::tmem_ld_wait();
          uint32_t w[16];
#pragma unroll
          for (int c4 = 0; c4 < 8; ++c4) {
            const float4 dq = dvv[8 * h2 + c4];
            const int c = 32 * h2 + 4 * c4;
            const float2 p0 = make_float2(__uint_as_float(pk[c / 2] << 16),
                                          __uint_as_float(pk[c / 2] & 0xFFFF0000u));
            const float2 p1 = make_float2(__uint_as_float(pk[c / 2 + 1] << 16),
                                          __uint_as_float(pk[c / 2 + 1] & 0xFFFF0000u));
            const float2 d0 = __fmul2_rn(
                p0,
                __fadd2_rn(make_float2(__uint_as_float(dp[4 * c4]), __uint_as_float(dp[4 * c4 + 1])),
                           make_float2(-dq.x, -dq.y)));
            const float2 d1 = __fmul2_rn(
                p1,
                __fadd2_rn(make_float2(__uint_as_float(dp[4 * c4 + 2]),
                                       __uint_as_float(dp[4 * c4 + 3])),
                           make_float2(-dq.z, -dq.w)));
            w[2 * c4] = sm100::pack_bf16x2(d0.x, d0.y);
            w[2 * c4 + 1] = sm100::pack_bf16x2(d1.x, d1.y);
          }
          // 128-byte swizzle: 16-byte chunk q of line kl_ lands at q ^ (kl_ & 7)
#pragma unroll
          for (int q = 0; q < 4; ++q)
            *reinterpret_cast<uint4*>(line + (((4 * h2 + q) ^ (kl_ & 7)) << 4)) =
                make_uint4(w[4 * q], w[4 * q + 1], w[4 * q + 2], w[4 * q + 3]);
        }
        sm100::fence_proxy_async_smem();
        sm100::tc_fence_before();
        __syncwarp();
        if (sm100::lane_id() == 0) sm100::mbar_arrive(ds_full);
      }
      if (!ok) break;
      tq += it.T;
      // ---------------- epilogue: dV, dK (x scale) of this key row, this warp's
      // half of the columns
      if (!(ok = sm100::mbar_wait(dkv_full, ik & 1, abort_flag, p.status))) break;
      sm100::tc_fence_after();
      const bool live = key < p.Lk;
      const size_t orow = (static_cast<size_t>(it.b) * p.Hkv + it.hkv) * p.Lk + (live ? key : 0);
      // each thread writes its own key row, so a warp's store touches 32 rows: 32-byte
      // stores fill whole sectors (d = 128 only: measured on B200, causal B2 H16 L8192,
      // 1.3762-1.3793 vs 1.3823-1.3834 ms; at d = 64 the wider path cost a register spill)
      const bool wide =
          DH == 128 &&
          ((reinterpret_cast<uintptr_t>(p.dV) | reinterpret_cast<uintptr_t>(p.dK)) & 31) == 0;
#pragma unroll 1
      for (int m = 0; m < 2; ++m) {
        __nv_bfloat16* dst = (m == 0 ? p.dV : p.dK) + orow * DH + (DH / 2) * hf;
        const float f = (m == 0) ? 1.f : p.scale;
        const uint32_t col = ((m == 0) ? DV_COL : DK_COL) + (DH / 2) * hf;
#pragma unroll 1
        for (int c = 0; c < DH / 64; ++c) {
          uint32_t v[32];
          sm100::tmem_ld32(tmem + lane_base + col + c * 32, v);
          sm100::tmem_ld_wait();
          uint32_t o[16];
#pragma unroll
          for (int e = 0; e < 16; ++e)
            o[e] = it.T > 0 ? sm100::pack_bf16x2(__uint_as_float(v[2 * e]) * f,
                                                 __uint_as_float(v[2 * e + 1]) * f)
                            : 0u;
          if (live) {
            if (wide) {  // this key row's 64 bytes as two whole sectors
              st_global_v8(dst + c * 32, &o[0]);
              st_global_v8(dst + c * 32 + 16, &o[8]);
            } else {
              uint4* d4 = reinterpret_cast<uint4*>(dst + c * 32);
#pragma unroll
              for (int q = 0; q < 4; ++q)
                d4[q] = make_uint4(o[4 * q], o[4 * q + 1], o[4 * q + 2], o[4 * q + 3]);
            }
          }
        }
      }
      sm100::tc_fence_before();
      __syncwarp();
      if (sm100::lane_id() == 0) sm100::mbar_arrive(dkv_empty);
    }
  } else if (warp >= W_DRAIN && warp < W_LOAD) {
    // ------------------------------------------------------------ dQ drain
    // d = 128: dQ^T of a query tile (lanes = head-dimension index, columns =
    // the tile's 128 rows) is moved to registers.  Its first DQ_ROWS rows are
    // added into the fp32 accumulator with coalesced 4-byte reductions straight
    // from registers (no wait on the staging buffer, so the TMEM columns go
    // back to the MMA warp as soon as the rest is in registers); the other
    // rows are staged row-major in shared memory DQ_ROWS rows at a time, each
    // block added with one bulk reduce-add (its rows are contiguous there).
    // The staging buffer is reused once the previous reduce has read it.
    // Measured on B200 (causal B2 H16 L8192 d128, same-process A/B): all four
    // rounds staged 1.457-1.486 ms; the first round by reductions 1.342-1.379
    // ms (shipped); the last one instead 1.420-1.442 ms; the first two
    // 1.402 ms; the last three 1.650 ms.
    // d = 64: dQ (lanes = the tile's rows) goes to registers one row per thread;
    // the rows are staged as two boxes of 128 rows x 32 columns in the 128-byte
    // swizzle of the accumulator's tensor map (a thread's 16-byte chunk c of row
    // r lands at chunk c ^ (r & 7) of the row's 128-byte line, so the eight
    // threads of a quarter-warp hit distinct banks) and added with two tensor
    // reduce-adds.
    const int tid = threadIdx.x - 32 * W_DRAIN;  // = TMEM lane
    const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
    float* stage = reinterpret_cast<float*>(smem + C::OFF_DQ);
    uint32_t tq = 0;
    bool ok = true;
    for (uint32_t ik = 0; ok; ++ik) {
      int w;
      if (!(ok = next_item(ik, w)) || w < 0) break;
      const Item it = get_item(p, w, nullptr);
      const int nq = it.T > 0 ? it.T / p.G : 0;
      for (int t = 0; t < it.T && ok; ++t) {
        const uint32_t cur = tq + t;
        int g, i;
        tile_of(it, t, nq, g, i);
        const int qh = it.b * p.Hq + it.hkv * p.G + g;
        float* acc_rows = p.dq_acc + (static_cast<size_t>(qh) * p.Lqp + i * BMQ) * DH;
        if (!(ok = sm100::mbar_wait(dq_full, cur & 1, abort_flag, p.status))) break;
        sm100::tc_fence_after();
        if constexpr (C::STAGED_DQ) {
          // DQ_ROWS rows of the tile (fp32 values `v`, one per row, of this
          // thread's d column) through the staging buffer into the accumulator
          auto stage_round = [&](const uint32_t* v, int row0) {
            // the previous reduce must have finished reading the staging buffer
            if (tid == 0) bulk_wait_read_all();
            sm100::named_bar_sync(1, 128);
#pragma unroll
            for (int c = 0; c < DQ_ROWS; ++c) stage[c * DH + tid] = __uint_as_float(v[c]);
            sm100::fence_proxy_async_smem();
            sm100::named_bar_sync(1, 128);
            if (tid == 0) bulk_reduce_add_f32(acc_rows + row0 * DH, stage, DQ_ROWS * DH * 4);
          };
          // rows 0-63 to registers, the first 32 of them out by reductions,
          // rows 64-127 to registers: the columns go back to the MMA warp
          // with at most 96 values held
          uint32_t a[64], b[64];
          sm100::tmem_ld32(tmem + lane_base + DP_COL, *reinterpret_cast<uint32_t(*)[32]>(&a[0]));
          sm100::tmem_ld32(tmem + lane_base + DP_COL + 32,
                           *reinterpret_cast<uint32_t(*)[32]>(&a[32]));
          sm100::tmem_ld_wait();
#pragma unroll
          for (int c = 0; c < DQ_ROWS; ++c)
            red_add_f32(acc_rows + c * DH + tid, __uint_as_float(a[c]));
          sm100::tmem_ld32(tmem + lane_base + DP_COL + 64,
                           *reinterpret_cast<uint32_t(*)[32]>(&b[0]));
          sm100::tmem_ld32(tmem + lane_base + DP_COL + 96,
                           *reinterpret_cast<uint32_t(*)[32]>(&b[32]));
          sm100::tmem_ld_wait();
          sm100::tc_fence_before();
          __syncwarp();
          if (sm100::lane_id() == 0) sm100::mbar_arrive(dq_empty);
          stage_round(&a[32], 32);
          stage_round(&b[0], 64);
          stage_round(&b[32], 96);
        } else {
          uint32_t v[64];
          sm100::tmem_ld32(tmem + lane_base + DP_COL, *reinterpret_cast<uint32_t(*)[32]>(&v[0]));
          sm100::tmem_ld32(tmem + lane_base + DP_COL + 32,
                           *reinterpret_cast<uint32_t(*)[32]>(&v[32]));
          sm100::tmem_ld_wait();
          // the whole row has left TMEM: the columns are free for dP^T
          sm100::tc_fence_before();
          __syncwarp();
          if (sm100::lane_id() == 0) sm100::mbar_arrive(dq_empty);
          // the previous tile's reduces must have finished reading the staging boxes
          if (tid == 0) bulk_wait_read_all();
          sm100::named_bar_sync(1, 128);
          uint8_t* line = smem + C::OFF_DQ + tid * 128;
#pragma unroll
          for (int h = 0; h < 2; ++h)
#pragma unroll
            for (int c = 0; c < 8; ++c)
              *reinterpret_cast<uint4*>(line + h * (BMQ * 128) + ((c ^ (tid & 7)) << 4)) =
                  make_uint4(v[32 * h + 4 * c], v[32 * h + 4 * c + 1], v[32 * h + 4 * c + 2],
                             v[32 * h + 4 * c + 3]);
          sm100::fence_proxy_async_smem();
          sm100::named_bar_sync(1, 128);
          if (tid == 0) {
            tma_reduce_add_3d(&tmAcc, smem + C::OFF_DQ, 0, i * BMQ, qh);
            tma_reduce_add_3d(&tmAcc, smem + C::OFF_DQ + BMQ * 128, 32, i * BMQ, qh);
            asm volatile("cp.async.bulk.commit_group;" ::: "memory");
          }
        }
      }
      tq += it.T;
    }
    // the convert pass reads the accumulator after this kernel; the bulk
    // reduces must be complete before the CTA exits
    if (tid == 0) bulk_wait_all();
  }

  sm100::tc_fence_before();
  __syncthreads();
  if (warp == W_MMA) {
    sm100::tc_fence_after();
    sm100::tmem_dealloc(tmem, 512);
  }
  if (threadIdx.x == 0) {
    // the last CTA to finish re-arms the dynamic scheduler for the next launch
    __threadfence();
    if (atomicAdd(p.sched + 1, 1) == static_cast<int>(gridDim.x) - 1) {
      p.sched[0] = 0;
      p.sched[1] = 0;
      __threadfence();
    }
  }
}

// ------------------------------------------------------------------ host side

bool make_tmap_rows(CUtensorMap* m, const void* base, int d, int L, long long heads,
                    int box_rows);
// fp32 view [heads][Lqp][64] of the d = 64 dQ accumulator, boxes of 32 columns x
// 128 rows x 1 head, 128-byte swizzle (the staging layout of the drain)
bool make_tmap_acc64(CUtensorMap* m, float* base, int Lqp, long long heads);

template <int DH>
attn_status_t launch_d(const Args& a, cudaStream_t s) {
  using C = Cfg<DH>;
  Params p;
  p.B = a.B;
  p.Hq = a.Hq;
  p.Hkv = a.Hkv;
  p.G = a.Hq / a.Hkv;
  p.Lq = a.Lq;
  p.Lk = a.Lk;
  p.Lqp = lq_pad(a.Lq);
  p.scale = a.scale;
  p.scale_log2 = a.scale * 1.4426950408889634f;
  p.causal = a.causal;
  p.window = a.window;
  p.k_lens = a.k_lens;
  p.status = a.status;
  const size_t rows = static_cast<size_t>(a.B) * a.Hq * p.Lqp;
  p.dq_acc = reinterpret_cast<float*>(a.scratch);
  float* lse2 = reinterpret_cast<float*>(a.scratch + rows * DH * 4);
  float* Dv = lse2 + rows;
  p.lse2 = lse2;
  p.Dvec = Dv;
  p.dK = a.dK;
  p.dV = a.dV;
  p.n_kv = (a.Lk + BN - 1) / BN;
  p.n_qt = p.Lqp / BMQ;
  p.n_items = a.B * a.Hkv * p.n_kv;
  p.sched = a.status + 1;
  const int BH = a.B * a.Hq;

  // 1. prep
  if (a.Lq > 0) {
    const long long warps = static_cast<long long>(BH) * p.Lqp;
    bwd_prep_kernel<DH><<<static_cast<unsigned>((warps * 32 + 255) / 256), 256, 0, s>>>(
        a.O, a.dO, a.lse, p.dq_acc, lse2, Dv, BH, a.Lq, p.Lqp);
    if (attn_host::report_launch(bwd_prep_kernel<DH>, "bwd_prep_kernel") != cudaSuccess)
      return ATTN_ERR_CUDA;
  }
  // 2. main
  if (p.n_items > 0) {
    CUtensorMap tq, tdo, tk, tv, tacc;
    if (!make_tmap_rows(&tq, a.Q, DH, a.Lq, BH, BMQ) || !make_tmap_rows(&tdo, a.dO, DH, a.Lq, BH, BMQ) ||
        !make_tmap_rows(&tk, a.K, DH, a.Lk, static_cast<long long>(a.B) * a.Hkv, BN) ||
        !make_tmap_rows(&tv, a.V, DH, a.Lk, static_cast<long long>(a.B) * a.Hkv, BN) ||
        !(C::STAGED_DQ ? (tacc = tq, true) : make_tmap_acc64(&tacc, p.dq_acc, p.Lqp, BH))) {
      attn_host::report(cudaErrorInvalidValue, "bwd tensor maps");
      return ATTN_ERR_CUDA;
    }
    if (attn_host::report(attn_host::set_smem(bwd_main_kernel<DH>, C::SMEM_BYTES),
                          "bwd_main_kernel shared-memory attribute") != cudaSuccess)
      return ATTN_ERR_CUDA;
    const int grid = p.n_items < a.sms ? p.n_items : a.sms;
    bwd_main_kernel<DH><<<grid, NTHREADS, C::SMEM_BYTES, s>>>(tq, tdo, tk, tv, tacc, p);
    if (attn_host::report_launch(bwd_main_kernel<DH>, "bwd_main_kernel") != cudaSuccess)
      return ATTN_ERR_CUDA;
  }
  // 3. dQ
  if (a.Lq > 0) {
    const size_t n4 = static_cast<size_t>(BH) * a.Lq * (DH / 4);
    bwd_dq_convert_kernel<DH><<<static_cast<unsigned>((n4 + 255) / 256), 256, 0, s>>>(
        p.dq_acc, a.dQ, BH, a.Lq, p.Lqp, a.scale);
    if (attn_host::report_launch(bwd_dq_convert_kernel<DH>, "bwd_dq_convert_kernel") !=
        cudaSuccess)
      return ATTN_ERR_CUDA;
  }
  return ATTN_OK;
}

inline attn_status_t launch(const Args& a, cudaStream_t s) {
  if (a.d == 128) return launch_d<128>(a, s);
  if (a.d == 64) return launch_d<64>(a, s);
  return ATTN_ERR_UNSUPPORTED;
}

}  // namespace attn_bwd_impl
