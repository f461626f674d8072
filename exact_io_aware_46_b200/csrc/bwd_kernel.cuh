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
//     accumulator; rows are padded to a multiple of 64 per head.
//  2. main (persistent, one CTA per SM): a work item is one 128-key tile of one
//     (batch, key/value head).  K and V stay in shared memory while the item
//     walks every 64-row query tile of every query head of the group that can
//     see the keys.  Per query tile the tensor core computes, with keys on the
//     128 TMEM lanes,
//        S^T  = K Q^T          (SS)        dP^T = V dO^T        (SS)
//        dV  += P^T dO         (TS: P^T from TMEM, written by the softmax)
//        dK  += dS^T Q         (SS: dS^T staged in shared memory)
//        dQ^T = K^T dS^T       (SS, both operands MN-major)
//     dV and dK accumulate in TMEM across the item; S/dP are double-buffered
//     and dQ^T reuses the dP buffer once dS has been formed.  Warps 0-3 form
//     P and dS (one key row per thread), warps 4-7 drain dQ^T with fp32
//     reductions into the accumulator, warp 8 feeds TMA, warp 9 issues MMAs.
//  3. convert: dQ = bf16(scale * accumulator).
#pragma once

#include "launch_cache.cuh"
#include "sm100.cuh"

namespace attn_bwd_impl {

constexpr int BN = 128;  // keys per work item (TMEM lanes)
constexpr int BMQ = 64;  // query rows per query tile
constexpr int D = 128;   // head dimension handled by the main kernel
constexpr int NQS = 3;   // query/dO ring stages
constexpr int NTHREADS = 320;  // P/dS warpgroup, dQ warpgroup, load warp, MMA warp

// shared memory map (bytes); the swizzled panels are 1024-byte aligned
constexpr int OFF_K = 0;                              // [128 keys][d]: 2 panels of 16 KB
constexpr int OFF_V = 32768;
constexpr int OFF_QS = 65536;                         // stage s: Q (2 x 8 KB) then dO (2 x 8 KB)
constexpr int QS_BYTES = 32768;
constexpr int OFF_DS = OFF_QS + NQS * QS_BYTES;       // dS^T buffers [128 keys][64 rows], 16 KB each
constexpr int OFF_LD = OFF_DS + 2 * 16384;            // stage s: lse2 [64] then D [64]
constexpr int OFF_DQ = OFF_LD + NQS * 512;            // dQ tile staging [64 rows][128] fp32, 32 KB
constexpr int OFF_BAR = OFF_DQ + 32768;
constexpr int SMEM_BYTES = OFF_BAR + 512 + 1024;
static_assert(SMEM_BYTES <= 232448, "dynamic shared memory limit");

// TMEM columns
constexpr uint32_t S_COL0 = 0;      // S^T / P^T, 2 buffers x 64
constexpr uint32_t DP_COL0 = 128;   // dP^T, then dQ^T, 2 buffers x 64
constexpr uint32_t DV_COL = 256;
constexpr uint32_t DK_COL = 384;

constexpr uint32_t IDESC_S = sm100::idesc_bf16_f32(128, BMQ, false, false);
constexpr uint32_t IDESC_DV = sm100::idesc_bf16_f32(128, D, false, true);
constexpr uint32_t IDESC_DQ = sm100::idesc_bf16_f32(128, BMQ, true, true);

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
  float* dq_acc;       // [B*Hq][Lqp][D] fp32
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
  int n_qt;     // Lqp / 64
  int n_items;  // B * Hkv * n_kv
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

__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes,
                                         uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          sm100::smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(sm100::smem_u32(bar))
      : "memory");
}

// ------------------------------------------------------------------ prep

__global__ void __launch_bounds__(256) bwd_prep_kernel(const __nv_bfloat16* O,
                                                        const __nv_bfloat16* dO,
                                                        const float* lse, float* dq_acc,
                                                        float* lse2, float* Dv, int BH, int Lq,
                                                        int Lqp) {
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (warp >= BH * Lqp) return;
  const int bh = warp / Lqp, r = warp % Lqp;
  float acc = 0.f;
  if (r < Lq) {
    const size_t off = (static_cast<size_t>(bh) * Lq + r) * D + lane * 4;
    const uint2 a = *reinterpret_cast<const uint2*>(O + off);
    const uint2 g = *reinterpret_cast<const uint2*>(dO + off);
    acc = __uint_as_float(a.x << 16) * __uint_as_float(g.x << 16) +
          __uint_as_float(a.x & 0xFFFF0000u) * __uint_as_float(g.x & 0xFFFF0000u) +
          __uint_as_float(a.y << 16) * __uint_as_float(g.y << 16) +
          __uint_as_float(a.y & 0xFFFF0000u) * __uint_as_float(g.y & 0xFFFF0000u);
  }
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  reinterpret_cast<float4*>(dq_acc + static_cast<size_t>(warp) * D)[lane] =
      make_float4(0.f, 0.f, 0.f, 0.f);
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

__global__ void __launch_bounds__(256) bwd_dq_convert_kernel(const float* dq_acc,
                                                              __nv_bfloat16* dQ, int BH, int Lq,
                                                              int Lqp, float scale) {
  const size_t i = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x;  // 4 elements
  const size_t total = static_cast<size_t>(BH) * Lq * (D / 4);
  if (i >= total) return;
  const size_t row = i / (D / 4);
  const int c4 = static_cast<int>(i % (D / 4));
  const int bh = static_cast<int>(row / Lq), r = static_cast<int>(row % Lq);
  const float4 v =
      reinterpret_cast<const float4*>(dq_acc + (static_cast<size_t>(bh) * Lqp + r) * D)[c4];
  uint2 o;
  o.x = sm100::pack_bf16x2(v.x * scale, v.y * scale);
  o.y = sm100::pack_bf16x2(v.z * scale, v.w * scale);
  reinterpret_cast<uint2*>(dQ + row * D)[c4] = o;
}

// ------------------------------------------------------------------ main

__global__ void __launch_bounds__(NTHREADS, 1)
    bwd_main_kernel(const __grid_constant__ CUtensorMap tmQ,
                    const __grid_constant__ CUtensorMap tmdO,
                    const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, const Params p) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = sm100::smem_u32(smem_raw);
  uint8_t* smem = smem_raw + ((1024 - (raw_addr & 1023)) & 1023);
  const uint32_t sbase = sm100::smem_u32(smem);

  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + OFF_BAR);
  uint64_t* kv_full = bars + 0;
  uint64_t* kv_empty = bars + 1;
  uint64_t* qdo_full = bars + 2;    // [NQS]
  uint64_t* qdo_empty = bars + 5;   // [NQS]
  uint64_t* s_full = bars + 8;      // [2]
  uint64_t* p_full = bars + 10;     // [2]
  uint64_t* dp_full = bars + 12;    // [2]
  uint64_t* ds_full = bars + 14;    // [2]
  uint64_t* ds_empty = bars + 16;   // [2]
  uint64_t* dq_full = bars + 18;    // [2]
  uint64_t* dq_empty = bars + 20;   // [2]
  uint64_t* dkv_full = bars + 22;
  uint64_t* dkv_empty = bars + 23;
  uint64_t* drain = bars + 24;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 25);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  if (threadIdx.x == 0) {
    sm100::mbar_init(kv_full, 1);
    sm100::mbar_init(kv_empty, 1);
    for (int s = 0; s < NQS; ++s) {
      sm100::mbar_init(&qdo_full[s], 1);
      sm100::mbar_init(&qdo_empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      sm100::mbar_init(&s_full[b], 1);
      sm100::mbar_init(&p_full[b], 128);
      sm100::mbar_init(&dp_full[b], 1);
      sm100::mbar_init(&ds_full[b], 128);
      sm100::mbar_init(&ds_empty[b], 1);
      sm100::mbar_init(&dq_full[b], 1);
      sm100::mbar_init(&dq_empty[b], 128);
    }
    sm100::mbar_init(dkv_full, 1);
    sm100::mbar_init(dkv_empty, 128);
    sm100::mbar_init(drain, 1);
    *abort_flag = 0;
    sm100::fence_barrier_init();
  }
  if (warp == 8 && sm100::lane_id() == 0) {
    sm100::prefetch_tmap(&tmQ);
    sm100::prefetch_tmap(&tmdO);
    sm100::prefetch_tmap(&tmK);
    sm100::prefetch_tmap(&tmV);
  }
  if (warp == 9) {
    sm100::tmem_alloc(tmem_slot, 512);
    sm100::tmem_relinquish();
  }
  sm100::tc_fence_before();
  __syncthreads();
  sm100::tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int off = p.Lk - p.Lq;  // bottom-right causal alignment
  if (warp == 8) {
    // ------------------------------------------------------------ TMA producer
    if (sm100::lane_id() == 0) {
      uint32_t tq = 0, ik = 0;
      bool ok = true;
      for (int w = blockIdx.x; w < p.n_items && ok; w += gridDim.x, ++ik) {
        const Item it = get_item(p, w, nullptr);
        if (!(ok = sm100::mbar_wait(kv_empty, (ik & 1) ^ 1, abort_flag, p.status))) break;
        sm100::mbar_arrive_expect_tx(kv_full, 2 * BN * D * 2);
        const int kvh = it.b * p.Hkv + it.hkv;
        for (int c = 0; c < 2; ++c) {
          sm100::tma_load_3d(&tmK, kv_full, smem + OFF_K + c * 16384, c * 64, it.n * BN, kvh);
          sm100::tma_load_3d(&tmV, kv_full, smem + OFF_V + c * 16384, c * 64, it.n * BN, kvh);
        }
        const int nq = it.T > 0 ? it.T / p.G : 0;
        for (int t = 0; t < it.T && ok; ++t, ++tq) {
          const int g = t / nq, i = it.i_lo + t % nq;
          const int slot = tq % NQS;
          if (!(ok = sm100::mbar_wait(&qdo_empty[slot], ((tq / NQS) & 1) ^ 1, abort_flag,
                                      p.status)))
            break;
          sm100::mbar_arrive_expect_tx(&qdo_full[slot], QS_BYTES + 512);
          const int qh = it.b * p.Hq + it.hkv * p.G + g;
          uint8_t* st = smem + OFF_QS + slot * QS_BYTES;
          for (int c = 0; c < 2; ++c) {
            sm100::tma_load_3d(&tmQ, &qdo_full[slot], st + c * 8192, c * 64, i * BMQ, qh);
            sm100::tma_load_3d(&tmdO, &qdo_full[slot], st + 16384 + c * 8192, c * 64, i * BMQ,
                               qh);
          }
          const size_t rowoff = static_cast<size_t>(qh) * p.Lqp + i * BMQ;
          bulk_g2s(smem + OFF_LD + slot * 512, p.lse2 + rowoff, 256, &qdo_full[slot]);
          bulk_g2s(smem + OFF_LD + slot * 512 + 256, p.Dvec + rowoff, 256, &qdo_full[slot]);
        }
      }
    }
  } else if (warp == 9) {
    // ------------------------------------------------------------ MMA issuer
    // The whole warp runs the loop (warp-uniform values stay in uniform
    // registers) and one elected lane issues; descriptors are built once per
    // operand and stepped by constant offsets.  MMA issue is close to
    // synchronous, so scalar work between two MMAs idles the tensor pipe.
    const bool leader = sm100::elect_one();
    {
      uint32_t tq = 0, ik = 0;
      bool ok = true;
      const uint32_t kA = sbase + OFF_K, vA = sbase + OFF_V;
      auto qA = [&](int slot) { return sbase + OFF_QS + slot * QS_BYTES; };
      auto doA = [&](int slot) { return sbase + OFF_QS + slot * QS_BYTES + 16384; };
      auto dsA = [&](int b) { return sbase + OFF_DS + b * 16384; };
      auto commit = [&](uint64_t* bar) {
        if (leader) sm100::tc_commit(bar);
        __syncwarp();
      };
      // S^T (or dP^T) = A_keys[128 x d] * B_rows[64 x d]^T, both K-major
      auto issue_kmajor = [&](uint32_t dcol, uint32_t a, uint32_t b) {
        const uint64_t ad = sm100::sdesc_sw128(a, 16, 1024);
        const uint64_t bd = sm100::sdesc_sw128(b, 16, 1024);
        if (leader) {
#pragma unroll
          for (int k = 0; k < D / 16; ++k)
            sm100::mma_ss(tmem + dcol, ad + (((k >> 2) * 16384 + (k & 3) * 32) >> 4),
                          bd + (((k >> 2) * 8192 + (k & 3) * 32) >> 4), IDESC_S, k > 0);
        }
      };
      for (int w = blockIdx.x; w < p.n_items && ok; w += gridDim.x, ++ik) {
        const Item it = get_item(p, w, nullptr);
        if (!(ok = sm100::mbar_wait(kv_full, ik & 1, abort_flag, p.status))) break;
        sm100::tc_fence_after();
        if (it.T == 0) {
          if (!(ok = sm100::mbar_wait(dkv_empty, (ik & 1) ^ 1, abort_flag, p.status))) break;
          commit(dkv_full);
          commit(kv_empty);
          continue;
        }
        // Issue order per query tile t (buffers b = t & 1, nb = (t + 1) & 1):
        //   S(t+1) | dV(t) [P(t)] | dP(t+1) [dQ^T(t-1) drained] | dK(t), dQ^T(t) [dS(t)]
        // so each wait on another warp's signal has half an iteration of queued
        // tensor work in front of it.
        {
          const int slot = tq % NQS, b = tq & 1;
          if (!(ok = sm100::mbar_wait(&qdo_full[slot], (tq / NQS) & 1, abort_flag, p.status)))
            break;
          sm100::tc_fence_after();
          issue_kmajor(S_COL0 + b * 64, kA, qA(slot));
          commit(&s_full[b]);
          if (!(ok = sm100::mbar_wait(&dq_empty[b], ((tq >> 1) & 1) ^ 1, abort_flag, p.status)))
            break;
          sm100::tc_fence_after();
          issue_kmajor(DP_COL0 + b * 64, vA, doA(slot));
          commit(&dp_full[b]);
        }
        const uint64_t kd_mn = sm100::sdesc_sw128(kA, 16384, 1024);  // K as MN-major A (over d)
        for (int t = 0; t < it.T && ok; ++t) {
          const uint32_t cur = tq + t;
          const int slot = cur % NQS, b = cur & 1;
          const uint32_t u = cur >> 1;
          const uint32_t nx = cur + 1;
          const int ns = nx % NQS, nb = nx & 1;
          const bool more = t + 1 < it.T;
          if (more) {
            if (!(ok = sm100::mbar_wait(&qdo_full[ns], (nx / NQS) & 1, abort_flag, p.status)))
              break;
            sm100::tc_fence_after();
            issue_kmajor(S_COL0 + nb * 64, kA, qA(ns));
            commit(&s_full[nb]);
          }
          if (!(ok = sm100::mbar_wait(&p_full[b], u & 1, abort_flag, p.status))) break;
          sm100::tc_fence_after();
          if (t == 0) {
            if (!(ok = sm100::mbar_wait(dkv_empty, (ik & 1) ^ 1, abort_flag, p.status))) break;
            sm100::tc_fence_after();
          }
          const uint64_t do_mn = sm100::sdesc_sw128(doA(slot), 8192, 1024);
          const uint64_t q_mn = sm100::sdesc_sw128(qA(slot), 8192, 1024);
          const uint64_t ds_k = sm100::sdesc_sw128(dsA(b), 16, 1024);
          const uint64_t ds_mn = sm100::sdesc_sw128(dsA(b), 8192, 1024);
          // dV += P^T dO : A = P^T (TMEM, packed bf16), B = dO (MN-major)
          if (leader) {
#pragma unroll
            for (int k = 0; k < BMQ / 16; ++k)
              sm100::mma_ts(tmem + DV_COL, tmem + S_COL0 + b * 64 + k * 8, do_mn + ((k * 2048) >> 4),
                            IDESC_DV, (t > 0 || k > 0) ? 1u : 0u);
          }
          if (more) {
            if (!(ok = sm100::mbar_wait(&dq_empty[nb], ((nx >> 1) & 1) ^ 1, abort_flag,
                                        p.status)))
              break;
            sm100::tc_fence_after();
            issue_kmajor(DP_COL0 + nb * 64, vA, doA(ns));
            commit(&dp_full[nb]);
          }
          if (!(ok = sm100::mbar_wait(&ds_full[b], u & 1, abort_flag, p.status))) break;
          sm100::tc_fence_after();
          if (leader) {
            // dK += dS^T Q : A = dS^T (K-major over rows), B = Q (MN-major)
#pragma unroll
            for (int k = 0; k < BMQ / 16; ++k)
              sm100::mma_ss(tmem + DK_COL, ds_k + ((k * 32) >> 4), q_mn + ((k * 2048) >> 4),
                            IDESC_DV, (t > 0 || k > 0) ? 1u : 0u);
            // dQ^T = K^T dS^T : A = K (MN-major over d), B = dS^T (MN-major over rows)
#pragma unroll
            for (int k = 0; k < BN / 16; ++k)
              sm100::mma_ss(tmem + DP_COL0 + b * 64, kd_mn + ((k * 2048) >> 4),
                            ds_mn + ((k * 2048) >> 4), IDESC_DQ, k > 0 ? 1u : 0u);
          }
          commit(&dq_full[b]);
          commit(&ds_empty[b]);
          commit(&qdo_empty[slot]);
        }
        if (!ok) break;
        tq += it.T;
        commit(dkv_full);
        commit(kv_empty);
      }
      commit(drain);
      sm100::mbar_wait_drain(drain, 0);
    }
  } else if (warp < 4) {
    // ------------------------------------------------------------ P and dS (one key per thread)
    const int kl_ = threadIdx.x;  // key row within the tile = TMEM lane
    const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
    uint32_t tq = 0, ik = 0;
    bool ok = true;
    for (int w = blockIdx.x; w < p.n_items && ok; w += gridDim.x, ++ik) {
      bool bad = false;
      const Item it = get_item(p, w, &bad);
      if (bad && threadIdx.x == 0) atomicOr(p.status, 1);
      const int key = it.n * BN + kl_;
      const int lim = it.kv_len - 1;  // last visible key (padding)
      const int nq = it.T > 0 ? it.T / p.G : 0;
      for (int t = 0; t < it.T && ok; ++t) {
        const uint32_t cur = tq + t;
        const int slot = cur % NQS, b = cur & 1;
        const uint32_t u = cur >> 1;
        const int i = it.i_lo + t % nq;
        const float* l2s = reinterpret_cast<const float*>(smem + OFF_LD + slot * 512);
        const float* dsv = l2s + 64;
        // lse2 / D of this stage were delivered on qdo_full
        if (!(ok = sm100::mbar_wait(&qdo_full[slot], (cur / NQS) & 1, abort_flag, p.status)))
          break;
        if (!(ok = sm100::mbar_wait(&s_full[b], u & 1, abort_flag, p.status))) break;
        sm100::tc_fence_after();
        uint32_t s[64];
        sm100::tmem_ld32(tmem + lane_base + S_COL0 + b * 64, *reinterpret_cast<uint32_t(*)[32]>(&s[0]));
        sm100::tmem_ld32(tmem + lane_base + S_COL0 + b * 64 + 32,
                         *reinterpret_cast<uint32_t(*)[32]>(&s[32]));
        sm100::tmem_ld_wait();
        // key visible to query row r0 + c iff key <= lim_key, c >= cmin and
        // (sliding window) c <= cmax
        const int r0 = i * BMQ;
        const bool key_ok = key <= lim;
        const int cmin = p.causal ? key - r0 - off : -1;
        const int cmax = p.window > 0 ? key - off + p.window - 1 - r0 : BMQ;
        // whole tile visible: no per-element test (warp-uniform; usual case)
        const bool all_vis = __all_sync(0xffffffffu, key_ok && cmin <= 0 && cmax >= BMQ - 1);
        const float4* l2v = reinterpret_cast<const float4*>(l2s);
        const float2 sl2x2 = make_float2(p.scale_log2, p.scale_log2);
        float pr[64];
#pragma unroll
        for (int c4 = 0; c4 < 16; ++c4) {
          const float4 lq = l2v[c4];
          const float2 x0 = __ffma2_rn(
              make_float2(__uint_as_float(s[4 * c4]), __uint_as_float(s[4 * c4 + 1])), sl2x2,
              make_float2(-lq.x, -lq.y));
          const float2 x1 = __ffma2_rn(
              make_float2(__uint_as_float(s[4 * c4 + 2]), __uint_as_float(s[4 * c4 + 3])), sl2x2,
              make_float2(-lq.z, -lq.w));
          pr[4 * c4] = sm100::ex2(x0.x);
          pr[4 * c4 + 1] = sm100::ex2(x0.y);
          pr[4 * c4 + 2] = sm100::ex2(x1.x);
          pr[4 * c4 + 3] = sm100::ex2(x1.y);
        }
        if (!all_vis) {
#pragma unroll
          for (int c = 0; c < 64; ++c)
            if (!key_ok || c < cmin || c > cmax) pr[c] = 0.f;
        }
        uint32_t pk[32];
#pragma unroll
        for (int c = 0; c < 32; ++c) pk[c] = sm100::pack_bf16x2(pr[2 * c], pr[2 * c + 1]);
        sm100::tmem_st32(tmem + lane_base + S_COL0 + b * 64, pk);
        sm100::tmem_st_wait();
        sm100::tc_fence_before();
        sm100::mbar_arrive(&p_full[b]);

        if (!(ok = sm100::mbar_wait(&dp_full[b], u & 1, abort_flag, p.status))) break;
        sm100::tc_fence_after();
        sm100::tmem_ld32(tmem + lane_base + DP_COL0 + b * 64,
                         *reinterpret_cast<uint32_t(*)[32]>(&s[0]));
        sm100::tmem_ld32(tmem + lane_base + DP_COL0 + b * 64 + 32,
                         *reinterpret_cast<uint32_t(*)[32]>(&s[32]));
        sm100::tmem_ld_wait();
        const float4* dvv = reinterpret_cast<const float4*>(dsv);
#pragma unroll
        for (int c4 = 0; c4 < 16; ++c4) {
          const float4 dq = dvv[c4];
          const float2 d0 = __fmul2_rn(
              make_float2(pr[4 * c4], pr[4 * c4 + 1]),
              __fadd2_rn(make_float2(__uint_as_float(s[4 * c4]), __uint_as_float(s[4 * c4 + 1])),
                         make_float2(-dq.x, -dq.y)));
          const float2 d1 = __fmul2_rn(
              make_float2(pr[4 * c4 + 2], pr[4 * c4 + 3]),
              __fadd2_rn(make_float2(__uint_as_float(s[4 * c4 + 2]), __uint_as_float(s[4 * c4 + 3])),
                         make_float2(-dq.z, -dq.w)));
          pk[2 * c4] = sm100::pack_bf16x2(d0.x, d0.y);
          pk[2 * c4 + 1] = sm100::pack_bf16x2(d1.x, d1.y);
        }
        if (!(ok = sm100::mbar_wait(&ds_empty[b], (u & 1) ^ 1, abort_flag, p.status))) break;
        uint8_t* line = smem + OFF_DS + b * 16384 + kl_ * 128;
#pragma unroll
        for (int q = 0; q < 8; ++q)
          *reinterpret_cast<uint4*>(line + ((q ^ (kl_ & 7)) << 4)) =
              make_uint4(pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
        sm100::fence_proxy_async_smem();
        sm100::tc_fence_before();
        sm100::mbar_arrive(&ds_full[b]);
      }
      if (!ok) break;
      tq += it.T;
      // ---------------- epilogue: dV, dK (x scale) for this key row
      if (!(ok = sm100::mbar_wait(dkv_full, ik & 1, abort_flag, p.status))) break;
      sm100::tc_fence_after();
      const bool live = key < p.Lk;
      const size_t orow = (static_cast<size_t>(it.b) * p.Hkv + it.hkv) * p.Lk + (live ? key : 0);
#pragma unroll 1
      for (int m = 0; m < 2; ++m) {
        __nv_bfloat16* dst = (m == 0 ? p.dV : p.dK) + orow * D;
        const float f = (m == 0) ? 1.f : p.scale;
        const uint32_t col = (m == 0) ? DV_COL : DK_COL;
#pragma unroll 1
        for (int c = 0; c < D / 32; ++c) {
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
            uint4* d4 = reinterpret_cast<uint4*>(dst + c * 32);
#pragma unroll
            for (int q = 0; q < 4; ++q) d4[q] = make_uint4(o[4 * q], o[4 * q + 1], o[4 * q + 2], o[4 * q + 3]);
          }
        }
      }
      sm100::tc_fence_before();
      sm100::mbar_arrive(dkv_empty);
    }
  } else {
    // ------------------------------------------------------------ dQ drain (one d column per thread)
    // dQ^T of a query tile (lanes = head-dimension index, columns = 64 rows)
    // is staged row-major in shared memory and added into the fp32
    // accumulator with one 32 KB bulk reduce (the tile's rows are contiguous
    // there); the staging buffer is reused once the previous reduce has read it.
    const int dl = threadIdx.x - 128;  // TMEM lane = head-dimension index
    const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
    float* stage = reinterpret_cast<float*>(smem + OFF_DQ);
    uint32_t tq = 0;
    bool ok = true;
    for (int w = blockIdx.x; w < p.n_items && ok; w += gridDim.x) {
      const Item it = get_item(p, w, nullptr);
      const int nq = it.T > 0 ? it.T / p.G : 0;
      for (int t = 0; t < it.T && ok; ++t) {
        const uint32_t cur = tq + t;
        const int b = cur & 1;
        const uint32_t u = cur >> 1;
        const int g = t / nq, i = it.i_lo + t % nq;
        if (!(ok = sm100::mbar_wait(&dq_full[b], u & 1, abort_flag, p.status))) break;
        sm100::tc_fence_after();
        uint32_t v[64];
        sm100::tmem_ld32(tmem + lane_base + DP_COL0 + b * 64, *reinterpret_cast<uint32_t(*)[32]>(&v[0]));
        sm100::tmem_ld32(tmem + lane_base + DP_COL0 + b * 64 + 32,
                         *reinterpret_cast<uint32_t(*)[32]>(&v[32]));
        sm100::tmem_ld_wait();
        sm100::tc_fence_before();
        sm100::mbar_arrive(&dq_empty[b]);
        // the previous tile's reduce must have finished reading the staging buffer
        if (threadIdx.x == 128) bulk_wait_read_all();
        sm100::named_bar_sync(1, 128);
#pragma unroll
        for (int c = 0; c < 64; ++c) stage[c * D + dl] = __uint_as_float(v[c]);
        sm100::fence_proxy_async_smem();
        sm100::named_bar_sync(1, 128);
        if (threadIdx.x == 128) {
          const int qh = it.b * p.Hq + it.hkv * p.G + g;
          bulk_reduce_add_f32(p.dq_acc + (static_cast<size_t>(qh) * p.Lqp + i * BMQ) * D, stage,
                              BMQ * D * 4);
        }
      }
      tq += it.T;
    }
    // the convert pass reads the accumulator after this kernel; the reduces
    // must be complete before the CTA exits
    if (threadIdx.x == 128) bulk_wait_all();
  }

  sm100::tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    sm100::tc_fence_after();
    sm100::tmem_dealloc(tmem, 512);
  }
}

// ------------------------------------------------------------------ host side

bool make_tmap_rows(CUtensorMap* m, const void* base, int L, long long heads, int box_rows);

inline attn_status_t launch(const Args& a, cudaStream_t s) {
  if (a.d != D) return ATTN_ERR_UNSUPPORTED;
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
  float* lse2 = reinterpret_cast<float*>(a.scratch + rows * D * 4);
  float* Dv = lse2 + rows;
  p.lse2 = lse2;
  p.Dvec = Dv;
  p.dK = a.dK;
  p.dV = a.dV;
  p.n_kv = (a.Lk + BN - 1) / BN;
  p.n_qt = p.Lqp / BMQ;
  p.n_items = a.B * a.Hkv * p.n_kv;
  const int BH = a.B * a.Hq;

  // 1. prep
  if (a.Lq > 0) {
    const long long warps = static_cast<long long>(BH) * p.Lqp;
    bwd_prep_kernel<<<static_cast<unsigned>((warps * 32 + 255) / 256), 256, 0, s>>>(
        a.O, a.dO, a.lse, p.dq_acc, lse2, Dv, BH, a.Lq, p.Lqp);
    if (cudaGetLastError() != cudaSuccess) return ATTN_ERR_CUDA;
  }
  // 2. main
  if (p.n_items > 0) {
    CUtensorMap tq, tdo, tk, tv;
    if (!make_tmap_rows(&tq, a.Q, a.Lq, BH, BMQ) || !make_tmap_rows(&tdo, a.dO, a.Lq, BH, BMQ) ||
        !make_tmap_rows(&tk, a.K, a.Lk, static_cast<long long>(a.B) * a.Hkv, BN) ||
        !make_tmap_rows(&tv, a.V, a.Lk, static_cast<long long>(a.B) * a.Hkv, BN))
      return ATTN_ERR_CUDA;
    if (attn_host::set_smem(bwd_main_kernel, SMEM_BYTES) != cudaSuccess)
      return ATTN_ERR_CUDA;
    const int grid = p.n_items < a.sms ? p.n_items : a.sms;
    bwd_main_kernel<<<grid, NTHREADS, SMEM_BYTES, s>>>(tq, tdo, tk, tv, p);
    if (cudaGetLastError() != cudaSuccess) return ATTN_ERR_CUDA;
  }
  // 3. dQ
  if (a.Lq > 0) {
    const size_t n4 = static_cast<size_t>(BH) * a.Lq * (D / 4);
    bwd_dq_convert_kernel<<<static_cast<unsigned>((n4 + 255) / 256), 256, 0, s>>>(
        p.dq_acc, a.dQ, BH, a.Lq, p.Lqp, a.scale);
    if (cudaGetLastError() != cudaSuccess) return ATTN_ERR_CUDA;
  }
  return ATTN_OK;
}

}  // namespace attn_bwd_impl
