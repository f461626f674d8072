// fwd_kernel.cuh -- forward attention on sm_100a.
//
// Computes O = softmax((Q K^T + M) * scale) V and the per-row log-sum-exp with
// the online softmax of "FlashAttention and long context: three ledgers"
// (section "the key of FlashAttention is online softmax"): per query row keep
// the running max m, the sum l relative to m and the unnormalised output o;
// for each key/value tile rescale l and o by e^{m - m'} and add the tile's
// e^{S - m'} and e^{S - m'} V; finally O = o / l.  Tiles of Q, K and V are
// staged on chip (the tiling of the FlashAttention-2 tutorial, 2.1.2), so the
// score and probability tiles live only in tensor memory and registers.
//
// B200 design (not the A100/Hopper designs the pages describe):
//  * persistent CTAs, one per SM, walking a heaviest-first list of work items;
//    an item is a pair of 128-row query tiles of one (batch, head);
//  * warp 16 streams K and V tiles with TMA (128-byte swizzle) into a ring of
//    shared-memory slots; the two query tiles are loaded once per item;
//  * warp 17 owns tensor memory and one elected lane issues every tcgen05.mma:
//    S_t = Q_t K_j^T (both operands in shared memory) into TMEM, and
//    O_t += P_t V_j with P_t read from TMEM where the softmax wrote it over S_t;
//  * warps 0-7 and 8-15 are the softmax warps of query tile 0 and 1, so the
//    tensor core computes one tile's scores while the other tile's softmax
//    runs (ping-pong).  Two warps share each row (= TMEM lane) of a tile, one
//    per half of the key columns, and agree on the row max through shared
//    memory; two warps per scheduler and tile hide the latency of the
//    exponential chains that a single warp left exposed.
//  * a quarter of the exponentials (an eighth with 8-bit inputs or d = 64) run on the
//    FMA pipe (polynomial exp2), the rest on the special-function unit;
//  * the running max is kept in the log2 domain and is only moved when a row's
//    new max exceeds it by more than 8 (a factor 256): o and l only need a
//    common reference max, so a stale max is exact, and the O rescale in TMEM
//    becomes rare.
#pragma once

#include <climits>

#include "sm100.cuh"

namespace attn_fwd_impl {

constexpr int BM = 128;        // query rows per tile (= TMEM lanes)
constexpr int BN = 128;        // keys per key/value tile
constexpr int NSMX = 16;       // softmax warps: 2 tiles x 2 column halves x 4 lane quarters
constexpr int NTHREADS = 32 * NSMX + 64;  // + load warp + MMA warp
constexpr int W_LOAD = NSMX;
constexpr int W_MMA = NSMX + 1;
constexpr int CHUNK_BYTES = 128 * 128;  // one 128-row x 64-column bf16 swizzle panel
constexpr float RESCALE_THRESHOLD = 8.0f;  // log2 units

// EB: bytes per element of Q, K and V (2: bf16, 1: E4M3)
template <int D, int EB = 2>
struct Cfg {
  static constexpr int PANEL = 128 / EB;  // elements per 128-byte swizzle panel row
  static constexpr int CHUNKS = D / PANEL;
  static constexpr int KSTEP = 32 / EB;   // K elements per MMA instruction (32 bytes)
  static constexpr int TILE_BYTES = BM * D * EB;
  static constexpr int NS = (TILE_BYTES == 32768) ? 4 : 8;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_KV = 2 * TILE_BYTES;
  // row-max exchange [parity][tile][half][row] and row-sum exchange (same shape)
  static constexpr int OFF_RED = OFF_KV + NS * TILE_BYTES;
  static constexpr int OFF_LSUM = OFF_RED + 2 * 2 * 2 * BM * 4;
  static constexpr int OFF_BAR = OFF_LSUM + 2 * 2 * 2 * BM * 4;
  static constexpr int SMEM_BYTES = OFF_BAR + 512 + 1024;  // barriers, item ring + alignment slack
  // TMEM columns: S_0, S_1 (128 fp32 columns each), then O_0, O_1 (D columns
  // each).  At d = 128 the P of key half h (64 keys: packed bf16 pairs, or
  // E4M3 quads) overwrites the first 32 (16) of the 64 S columns that half h
  // was read from, so S_t(j+1) waits for PV_t(j).  At d = 64 (bf16) the O
  // tiles leave 128 columns free: P_t gets 64 of its own (half h at 32 h), and
  // S_t(j+1) is issued as soon as the softmax has read S_t(j), so the next
  // scores compute while this step's exponentials are formed.  Measured on
  // B200 (causal B4 H16 L4096 d64): 0.2171-0.2191 -> 0.2129-0.2130 ms; the
  // softmax warps' instruction throughput, not the wait for S, bounds d = 64.
  static constexpr bool SEP_P = D == 64 && EB == 2;
  __device__ static constexpr uint32_t s_col(int t) { return t * 128u; }
  __device__ static constexpr uint32_t o_col(int t) { return 256u + t * D; }
  __device__ static constexpr uint32_t p_col(int t) { return SEP_P ? 384u + 64u * t : t * 128u; }
  static constexpr uint32_t P_HALF = SEP_P ? 32u : 64u;  // columns between P's key halves
  static constexpr uint32_t IDESC_S = EB == 2 ? sm100::idesc_bf16_f32(128, BN, false, false)
                                               : sm100::idesc_e4m3_f32(128, BN, false, false);
  static constexpr uint32_t IDESC_PV = EB == 2 ? sm100::idesc_bf16_f32(128, D, false, true)
                                                : sm100::idesc_e4m3_f32(128, D, false, true);
};

struct Params {
  __nv_bfloat16* O;
  float* lse;
  const int* k_lens;
  int* status;  // device status word (workspace + 0)
  int* sched;   // [0] next dynamic item, [1] finished CTAs (workspace + 4)
  int B, Hq, Hkv, Lq, Lk;
  float scale_log2;  // scale * log2(e)
  int causal;
  int n_pairs;  // ceil(Lq / 256) (ceil(max_seqlen_q / 256) for packed sequences)
  int n_items;  // B * Hq * n_pairs
  // packed (variable-length) sequences: Q/O [total_q, Hq, D], K/V [total_k, Hkv, D],
  // sequence b = rows [cu_q[b], cu_q[b+1]) and [cu_k[b], cu_k[b+1]); lse [Hq, total_q].
  // nullptr for the batched layout.
  const int* cu_q;
  const int* cu_k;
  int total_q, total_k;
  int window;  // > 0: sliding window (with causal): a row sees its `window` latest keys
  // 8-bit inputs: one fp32 scale per 128-row tile of each head; a dequantised
  // row i is code * scale[head][i / 128].  nullptr for bf16 inputs.
  const float* q_scale;  // [B * Hq][n_qt]
  const float* k_scale;  // [B * Hkv][n_kt]
  const float* v_scale;  // [B * Hkv][n_kt]
  int n_qt, n_kt;
  // folding into an accumulator (ring attention): o_acc [B, Hq, Lq, D] fp32 and
  // lse [B, Hq, Lq] (in/out); O (bf16, may be nullptr) receives the merged O.
  float* o_acc;
  int merge_init;  // 1: the accumulator is overwritten instead of merged into
};

struct Item {
  int b, h, row0;  // row0: first query row of tile 0; tile 1 starts at row0 + BM
  int lq;          // query rows of this sequence
  int koff;        // Lk - Lq of this sequence (bottom-right causal alignment)
  int kv_len;      // visible keys
  int q_coord, k_coord;  // tensor-map row coordinate of the sequence's row 0
  int q_head, kv_head;   // tensor-map head coordinates
  size_t o_off;          // element offset of (row 0, head h) in O
  size_t o_rstride;      // elements between consecutive rows of O
  size_t lse_off;        // offset of row 0 in lse
  int n0, n1;    // one past the last key/value tile each query tile visits
  int lo0, lo1;  // first key/value tile each query tile visits (0 without a window)
  int jb, nmax;  // the item's key/value tiles: [jb, nmax)
};

// Kernel variants, fixed at compile time so that the plain batched forward
// carries none of the others' per-item state (measured: a single kernel with
// runtime switches ran the plain workload 7 % slower -- register spills in the
// MMA-issuing warp):
//   MODE_PLAIN   [B, H, L, d] tensors, optional causal mask and key padding;
//   MODE_WINDOW  the same with a sliding-window causal mask (p.window keys);
//   MODE_VARLEN  packed sequences [T, H, d] with cu_seqlens offsets;
//   MODE_FP8     the plain layout with E4M3 Q, K, V and per-tile scales;
//   MODE_MERGE   the plain layout, the result folded into an fp32 accumulator.
enum : int { MODE_PLAIN = 0, MODE_WINDOW = 1, MODE_VARLEN = 2, MODE_FP8 = 3, MODE_MERGE = 4 };

constexpr int DEV_BAD_SCALE = 8;  // device status bit: a scale that is not finite and > 0

constexpr int HEAD_GROUP = 8;  // heads whose items are interleaved (L2 reuse of their K/V)
constexpr int NI = 4;          // depth of the shared-memory item ring

__device__ __forceinline__ int tiles_for(const Params& p, const Item& it, int row0) {
  if (row0 >= it.lq) return 0;
  const int last = min(row0 + BM - 1, it.lq - 1);
  int hi = it.kv_len;
  if (p.causal) hi = min(hi, last + it.koff + 1);
  return hi <= 0 ? 0 : (hi + BN - 1) / BN;
}

// Item order: groups of HEAD_GROUP (batch, head) pairs; inside a group the
// latest query rows (heaviest under a causal mask) first, heads interleaved.
// Grouping keeps the concurrently streamed K/V within a few heads (L2-resident)
// while dynamic fetching keeps the heaviest-first property for load balance.
template <int D_OF_O, int MODE>
__device__ __forceinline__ Item get_item(const Params& p, int w, bool* bad) {
  Item it;
  const int BH = p.B * p.Hq;
  const int per_group = HEAD_GROUP * p.n_pairs;
  const int g = w / per_group;
  const int r = w % per_group;
  const int gsize = min(HEAD_GROUP, BH - g * HEAD_GROUP);
  const int pair = p.n_pairs - 1 - r / gsize;
  const int bh = g * HEAD_GROUP + r % gsize;
  it.b = bh / p.Hq;
  it.h = bh % p.Hq;
  it.row0 = pair * 2 * BM;
  const int kvh = it.h / (p.Hq / p.Hkv);
  if constexpr (MODE != MODE_VARLEN) {
    int kl = p.Lk;
    if (p.k_lens) {
      kl = __ldg(p.k_lens + it.b);
      if (kl < 0 || kl > p.Lk) {
        if (bad) *bad = true;
        kl = 0;
      }
    }
    it.lq = p.Lq;
    it.koff = p.Lk - p.Lq;
    it.kv_len = kl;
    it.q_coord = 0;
    it.k_coord = 0;
    it.q_head = it.b * p.Hq + it.h;
    it.kv_head = it.b * p.Hkv + kvh;
    it.o_off = 0;  // the epilogue addresses [B, H, L, d] directly in this layout
    it.o_rstride = D_OF_O;
    it.lse_off = 0;
  } else {
    const int q0 = __ldg(p.cu_q + it.b), q1 = __ldg(p.cu_q + it.b + 1);
    const int k0 = __ldg(p.cu_k + it.b), k1 = __ldg(p.cu_k + it.b + 1);
    // a malformed sequence (offsets decreasing, past the totals, or longer than
    // the stated maximum) is reported and skipped: nothing is read or written
    const bool ok = 0 <= q0 && q0 <= q1 && q1 <= p.total_q && q1 - q0 <= p.Lq && 0 <= k0 &&
                    k0 <= k1 && k1 <= p.total_k && k1 - k0 <= p.Lk;
    if (!ok && bad) *bad = true;
    it.lq = ok ? q1 - q0 : 0;
    it.kv_len = ok ? k1 - k0 : 0;
    it.koff = it.kv_len - it.lq;
    it.q_coord = ok ? q0 : 0;
    it.k_coord = ok ? k0 : 0;
    it.q_head = it.h;
    it.kv_head = kvh;
    it.o_off = (static_cast<size_t>(it.q_coord) * p.Hq + it.h) * D_OF_O;
    it.o_rstride = static_cast<size_t>(p.Hq) * D_OF_O;
    it.lse_off = static_cast<size_t>(it.h) * p.total_q + it.q_coord;
  }
  it.n0 = tiles_for(p, it, it.row0);
  it.n1 = tiles_for(p, it, it.row0 + BM);
  // sliding window: key tiles entirely below the first row's window are skipped
  it.lo0 = it.lo1 = 0;
  if constexpr (MODE == MODE_WINDOW) {
    const int f0 = it.row0 + it.koff - p.window + 1, f1 = f0 + BM;
    it.lo0 = f0 > 0 ? f0 / BN : 0;
    it.lo1 = f1 > 0 ? f1 / BN : 0;
    if (it.lo0 >= it.n0) it.n0 = it.lo0 = 0;  // no row of the tile sees a key
    if (it.lo1 >= it.n1) it.n1 = it.lo1 = 0;
  }
  it.nmax = max(it.n0, it.n1);
  it.jb = it.n0 > 0 ? it.lo0 : it.lo1;  // tile 1 never starts before tile 0
  return it;
}

// 32-byte global store / load of eight 32-bit words (one whole sector per lane);
// the address must be 32-byte aligned.
__device__ __forceinline__ void st_global_v8(void* p, const uint32_t* v) {
  asm volatile("st.global.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(p), "r"(v[0]),
               "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7])
               : "memory");
}
__device__ __forceinline__ void ld_global_v8(const void* p, uint32_t* v) {
  asm volatile("ld.global.v8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
               : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]),
                 "=r"(v[6]), "=r"(v[7])
               : "l"(p)
               : "memory");
}

// Polynomial (FMA-pipe) instead of MUFU exp2 for column pairs whose index
// cp = c / 2 satisfies cp % 8 >= 6 (bf16 at d = 128: a quarter of the
// exponentials) or cp % 8 == 7 (8-bit inputs, and d = 64: an eighth; at d = 64,
// causal B4 H16 L4096, an eighth 0.2007-0.2016 ms, a quarter 0.2038, three
// eighths 0.2140, a half 0.2304).  The softmax warps are issue-bound as
// much as MUFU-bound, so the best share is small.  Measured on B200 (causal
// B4 H16 L4096 d128): with one softmax warp per row 0 % 0.313 ms, 12.5 % 0.310
// ms, 25 % 0.325 ms, 50 % 0.349 ms; with two warps per row (this kernel)
// 12.5 % 0.2519-0.2540 ms, 25 % 0.2499-0.2509 ms, 37.5 % 0.2601-0.2621 ms;
// the 8-bit kernel, whose XU pipe also carries the E4M3 conversions, 12.5 %
// 0.2263 ms and 25 % 0.2304 ms.
template <int D, int EB>
__device__ __forceinline__ constexpr bool poly_pair(int cp) {
  return (EB == 2 && D == 128) ? (cp & 7) >= 6 : (cp & 7) == 7;
}

// S_t = Q_t K_j^T: 128 x 128 (keys) x D, both operands K-major SW128 panels.
// One base descriptor per operand; the K-steps (32 bytes each: 16 bf16 or 32
// E4M3 elements) add constant offsets (>> 4) to the start-address field.
// Inlined: an out-of-line call put its argument and descriptor set-up between
// consecutive MMAs.
template <int D, int EB>
__device__ __forceinline__ void issue_s_tile(uint32_t d_tmem, uint32_t q_smem, uint32_t k_smem) {
  using C = Cfg<D, EB>;
  const uint64_t qd = sm100::sdesc_sw128(q_smem, 16, 1024);
  const uint64_t kd = sm100::sdesc_sw128(k_smem, 16, 1024);
#pragma unroll
  for (int k = 0; k < D / C::KSTEP; ++k) {
    const uint64_t off = static_cast<uint64_t>(((k >> 2) * CHUNK_BYTES + (k & 3) * 32) >> 4);
    if constexpr (EB == 2)
      sm100::mma_ss(d_tmem, qd + off, kd + off, C::IDESC_S, k > 0 ? 1u : 0u);
    else
      sm100::mma_ss_f8(d_tmem, qd + off, kd + off, C::IDESC_S, k > 0 ? 1u : 0u);
  }
}

// O_t (+)= P_t V_j: A = P_t from TMEM (8 columns per instruction: 16 keys of
// packed bf16 or 32 keys of E4M3; keys 64..127 start 64 columns further on),
// B = V_j MN-major (LBO = next 128-byte panel of columns, SBO = next 8 keys);
// consecutive instructions start 16 (bf16) or 32 (E4M3) key rows further on.
template <int D, int EB>
__device__ __forceinline__ void issue_pv_tile(uint32_t o_tmem, uint32_t p_tmem, uint32_t v_smem,
                                              bool acc) {
  using C = Cfg<D, EB>;
  constexpr int KS = C::KSTEP;        // keys per instruction
  constexpr int PER_HALF = 64 / KS;   // instructions per 64-key half
  const uint64_t vd = sm100::sdesc_sw128(v_smem, CHUNK_BYTES, 1024);
#pragma unroll
  for (int k = 0; k < BN / KS; ++k) {
    const uint32_t a = p_tmem + (k / PER_HALF) * C::P_HALF + (k % PER_HALF) * 8;
    const uint64_t b = vd + static_cast<uint64_t>((k * KS * 128) >> 4);
    if constexpr (EB == 2)
      sm100::mma_ts(o_tmem, a, b, C::IDESC_PV, (acc || k > 0) ? 1u : 0u);
    else
      sm100::mma_ts_f8(o_tmem, a, b, C::IDESC_PV, (acc || k > 0) ? 1u : 0u);
  }
}

template <int D, int MODE>
__global__ void __launch_bounds__(NTHREADS, 1)
    fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
               const __grid_constant__ CUtensorMap tmV, const Params p) {
  constexpr int EB = MODE == MODE_FP8 ? 1 : 2;
  using C = Cfg<D, EB>;
  extern __shared__ uint8_t smem_raw[];
  // 1024-byte alignment for the 128-byte swizzle panels
  const uint32_t raw_addr = sm100::smem_u32(smem_raw);
  uint8_t* smem = smem_raw + ((1024 - (raw_addr & 1023)) & 1023);
  const uint32_t sbase = sm100::smem_u32(smem);

  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* kv_full = bars;
  uint64_t* kv_empty = bars + C::NS;
  uint64_t* q_full = bars + 2 * C::NS;
  uint64_t* q_empty = q_full + 1;
  uint64_t* s_full = q_full + 2;   // [2]
  uint64_t* p_full = q_full + 4;   // [2]
  uint64_t* o_full = q_full + 6;   // [2]
  uint64_t* o_empty = q_full + 8;  // [2]
  uint64_t* drain = q_full + 10;
  uint64_t* item_full = q_full + 11;   // [NI]
  uint64_t* item_empty = q_full + 11 + NI;  // [NI]
  uint64_t* s_free = q_full + 11 + 2 * NI;  // [2] (d = 64): the softmax has read S_t
  uint64_t* p_free = q_full + 13 + 2 * NI;  // [2] (d = 64): PV_t has read P_t
  int* item_ring = reinterpret_cast<int*>(q_full + 15 + 2 * NI);  // [NI]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(item_ring + NI);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;

  if (threadIdx.x == 0) {
    for (int i = 0; i < C::NS; ++i) {
      sm100::mbar_init(&kv_full[i], 1);
      sm100::mbar_init(&kv_empty[i], 1);
    }
    sm100::mbar_init(q_full, 1);
    sm100::mbar_init(q_empty, 1);
    for (int t = 0; t < 2; ++t) {
      sm100::mbar_init(&s_full[t], 1);
      sm100::mbar_init(&p_full[t], NSMX / 2);  // one arrival per softmax warp of the tile
      sm100::mbar_init(&o_full[t], 1);
      sm100::mbar_init(&o_empty[t], NSMX / 2);
      sm100::mbar_init(&s_free[t], NSMX / 2);  // one arrival per softmax warp of the tile
      sm100::mbar_init(&p_free[t], 1);
    }
    sm100::mbar_init(drain, 1);
    for (int i = 0; i < NI; ++i) {
      sm100::mbar_init(&item_full[i], 1);
      sm100::mbar_init(&item_empty[i], 1 + 32 * NSMX);  // the MMA thread + all softmax threads
    }
    *abort_flag = 0;
    sm100::fence_barrier_init();
  }
  if (warp == W_LOAD && sm100::lane_id() == 0) {
    sm100::prefetch_tmap(&tmQ);
    sm100::prefetch_tmap(&tmK);
    sm100::prefetch_tmap(&tmV);
  }
  if (warp == W_MMA) {
    sm100::tmem_alloc(tmem_slot, 512);
    sm100::tmem_relinquish();
  }
  sm100::tc_fence_before();
  __syncthreads();
  sm100::tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  // consumers' view of the item ring: the k-th item index, or -1 at the end
  auto next_item = [&](uint32_t k, int& w) -> bool {
    if (!sm100::mbar_wait(&item_full[k % NI], (k / NI) & 1, abort_flag, p.status)) return false;
    w = *reinterpret_cast<volatile int*>(&item_ring[k % NI]);
    sm100::mbar_arrive(&item_empty[k % NI]);
    return true;
  };

  if (warp == W_LOAD) {
    // ------------------------------------------------------------ scheduler + TMA producer
    if (sm100::lane_id() == 0) {
      uint32_t use = 0;     // K/V tile copies issued
      int q_issued = 0;     // Q copies issued (one per item)
      for (uint32_t k = 0;; ++k) {
        if (!sm100::mbar_wait(&item_empty[k % NI], ((k / NI) & 1) ^ 1, abort_flag, p.status))
          break;
        int w = (k == 0) ? static_cast<int>(blockIdx.x)
                         : atomicAdd(p.sched, 1) + static_cast<int>(gridDim.x);
        if (w >= p.n_items) w = -1;
        *reinterpret_cast<volatile int*>(&item_ring[k % NI]) = w;
        sm100::mbar_arrive(&item_full[k % NI]);
        if (w < 0) break;
        const Item it = get_item<D, MODE>(p, w, nullptr);
        if (!sm100::mbar_wait(q_empty, (k & 1) ^ 1, abort_flag, p.status)) break;
        sm100::mbar_arrive_expect_tx(q_full, 2 * C::TILE_BYTES);
        ++q_issued;
        const int qh = it.q_head;
        for (int t = 0; t < 2; ++t)
          for (int c = 0; c < C::CHUNKS; ++c)
            sm100::tma_load_3d(&tmQ, q_full,
                               smem + C::OFF_Q + t * C::TILE_BYTES + c * CHUNK_BYTES,
                               c * C::PANEL, it.q_coord + it.row0 + t * BM, qh);
        const int kvh = it.kv_head;
        bool ok = true;
        for (int j = it.jb; j < it.nmax && ok; ++j) {
          for (int kv = 0; kv < 2; ++kv, ++use) {
            const int slot = use % C::NS;
            if (!sm100::mbar_wait(&kv_empty[slot], ((use / C::NS) & 1) ^ 1, abort_flag,
                                  p.status)) {
              ok = false;
              break;
            }
            sm100::mbar_arrive_expect_tx(&kv_full[slot], C::TILE_BYTES);
            for (int c = 0; c < C::CHUNKS; ++c)
              sm100::tma_load_3d(kv == 0 ? &tmK : &tmV, &kv_full[slot],
                                 smem + C::OFF_KV + slot * C::TILE_BYTES + c * CHUNK_BYTES,
                                 c * C::PANEL, it.k_coord + j * BN, kvh);
          }
        }
        if (!ok) break;
      }
      // the CTA must not exit while tensor copies still land in its shared
      // memory, which an expired wait elsewhere could otherwise allow: wait
      // (bounded, ignoring the abort flag) for the last issued phase of every
      // load barrier; in normal operation the consumers already waited for them
      if (q_issued > 0) sm100::mbar_wait_drain(q_full, (q_issued - 1) & 1);
      for (uint32_t sl = 0; sl < C::NS && sl < use; ++sl) {
        const uint32_t last = sl + C::NS * ((use - 1 - sl) / C::NS);
        sm100::mbar_wait_drain(&kv_full[sl], (last / C::NS) & 1);
      }
    }
  } else if (warp == W_MMA) {
    // ------------------------------------------------------------ MMA issuer
    // The whole warp runs the loop so that its warp-uniform values (slots,
    // parities, descriptors) live in uniform registers; one elected lane
    // issues the tensor-core instructions.  Issue is close to synchronous (an
    // MMA is accepted about when the previous one starts), so any per-MMA
    // scalar work between them idles the tensor pipe: measured on B200,
    // lane-0-only code with out-of-line issue functions ran this kernel at
    // 0.306 ms (causal B4 H16 L4096 d128), inlined issue at 0.270 ms, and
    // this warp-wide form at 0.254 ms.
    const bool leader = sm100::elect_one();
    {
      uint32_t use = 0;
      uint32_t pc0 = 0, pc1 = 0;  // P tiles consumed per query tile
      bool ok = true;
      const uint32_t q_addr = sbase + C::OFF_Q;
      const uint32_t kv_addr = sbase + C::OFF_KV;

      auto commit = [&](uint64_t* b) {
        if (leader) sm100::tc_commit(b);
        __syncwarp();
      };
      auto issue_s = [&](int t, int slot) {
        if (leader)
          issue_s_tile<D, EB>(tmem + C::s_col(t), q_addr + t * C::TILE_BYTES,
                          kv_addr + slot * C::TILE_BYTES);
      };
      auto issue_pv = [&](int t, int slot, bool acc) {
        if (leader)
          issue_pv_tile<D, EB>(tmem + C::o_col(t), tmem + C::p_col(t),
                           kv_addr + slot * C::TILE_BYTES, acc);
      };
      // d = 64: S_t(n) may overwrite the S columns once the softmax has read
      // S_t(n - 1) (release n - 1 of s_free[t]); sc counts the S_t issued
      uint32_t sc[2] = {0u, 0u};
      auto s_slot_free = [&](int t) -> bool {
        if constexpr (C::SEP_P) {
          if (sc[t] > 0 &&
              !sm100::mbar_wait(&s_free[t], (sc[t] - 1) & 1, abort_flag, p.status))
            return false;
          ++sc[t];
        }
        return true;
      };

      for (uint32_t k = 0; ok; ++k) {
        int w;
        if (!(ok = sm100::mbar_wait(&item_full[k % NI], (k / NI) & 1, abort_flag, p.status))) break;
        w = *reinterpret_cast<volatile int*>(&item_ring[k % NI]);
        __syncwarp();
        if (leader) sm100::mbar_arrive(&item_empty[k % NI]);
        if (w < 0) break;
        const Item it = get_item<D, MODE>(p, w, nullptr);
        if (!(ok = sm100::mbar_wait(q_full, k & 1, abort_flag, p.status))) break;
        sm100::tc_fence_after();
        const uint32_t oe_par = (k & 1) ^ 1;
        const int jb = it.jb;
        const int lo[2] = {it.lo0, it.lo1};
        if (it.nmax > jb) {
          const int ks = use % C::NS;
          if (!(ok = sm100::mbar_wait(&kv_full[ks], (use / C::NS) & 1, abort_flag, p.status)))
            break;
          sm100::tc_fence_after();
          if (it.n0 > jb && lo[0] == jb) {
            ok = s_slot_free(0);
            if (!ok) break;
            issue_s(0, ks);
            commit(&s_full[0]);
          }
          if (it.n1 > jb && lo[1] == jb) {
            ok = s_slot_free(1);
            if (!ok) break;
            issue_s(1, ks);
            commit(&s_full[1]);
          }
          commit(&kv_empty[ks]);
        }
        // Q is free once the item's last S has run: release it then, so the next
        // item's Q loads while this item's last PV steps execute
        if (it.nmax - jb <= 1) commit(q_empty);
        for (int j = jb; j < it.nmax && ok; ++j) {
          const uint32_t vuse = use + 2 * (j - jb) + 1;
          const int vs = vuse % C::NS;
          const uint32_t kuse = vuse + 1;
          const int ks = kuse % C::NS;
          bool k_ready = false;
          if (!(ok = sm100::mbar_wait(&kv_full[vs], (vuse / C::NS) & 1, abort_flag, p.status)))
            break;
          sm100::tc_fence_after();
          // one query tile's step: O_t += P_t V_j, then S_t = Q_t K_{j+1}^T
          auto step = [&](int t, int n_t, uint32_t& pc, bool pv, bool sn) -> bool {
            auto do_pv = [&]() -> bool {
              if (lo[t] <= j && j < n_t) {
                if (j == lo[t] && !sm100::mbar_wait(&o_empty[t], oe_par, abort_flag, p.status))
                  return false;
                if (!sm100::mbar_wait(&p_full[t], pc & 1, abort_flag, p.status)) return false;
                ++pc;
                sm100::tc_fence_after();
                issue_pv(t, vs, j > lo[t]);
                if constexpr (C::SEP_P) commit(&p_free[t]);
                if (j == n_t - 1) commit(&o_full[t]);
              }
              return true;
            };
            auto do_s = [&]() -> bool {
              if (lo[t] <= j + 1 && j + 1 < n_t) {
                if (!k_ready) {
                  if (!sm100::mbar_wait(&kv_full[ks], (kuse / C::NS) & 1, abort_flag, p.status))
                    return false;
                  sm100::tc_fence_after();
                  k_ready = true;
                }
                if (!s_slot_free(t)) return false;
                sm100::tc_fence_after();
                issue_s(t, ks);
                commit(&s_full[t]);
              }
              return true;
            };
            return (!pv || do_pv()) && (!sn || do_s());
          };
          if constexpr (C::SEP_P) {
            // d = 64 (P has columns of its own): both tiles' next S go in as soon
            // as the softmax has read the current one, ahead of either PV, so
            // neither tile's softmax waits behind the other tile's P
            if (!(ok = step(0, it.n0, pc0, false, true) && step(1, it.n1, pc1, false, true) &&
                       step(0, it.n0, pc0, true, false) && step(1, it.n1, pc1, true, false)))
              break;
          } else {
            // P overwrites S: each tile's next S follows its PV
            if (!(ok = step(0, it.n0, pc0, true, true))) break;
            if (!(ok = step(1, it.n1, pc1, true, true))) break;
          }
          if (k_ready) commit(&kv_empty[ks]);
          commit(&kv_empty[vs]);
          if (j + 2 == it.nmax) commit(q_empty);  // S_t(nmax - 1) were the last S
        }
        if (!ok) break;
        if (it.n0 == 0) {
          if (!(ok = sm100::mbar_wait(&o_empty[0], oe_par, abort_flag, p.status))) break;
          commit(&o_full[0]);
        }
        if (it.n1 == 0) {
          if (!(ok = sm100::mbar_wait(&o_empty[1], oe_par, abort_flag, p.status))) break;
          commit(&o_full[1]);
        }
        use += 2 * (it.nmax - jb);
      }
      // all issued tensor-core work (and its commits) must land before TMEM is freed
      commit(drain);
      sm100::mbar_wait_drain(drain, 0);
    }
  } else {
    // ------------------------------------------------------------ softmax warps
    const int t = warp >> 3;          // query tile
    const int hf = (warp >> 2) & 1;   // key-column half: columns [64 hf, 64 hf + 64)
    const int qd = warp & 3;          // lane quarter
    const int r = qd * 32 + sm100::lane_id();  // row within the tile = TMEM lane
    const uint32_t lane_base = static_cast<uint32_t>(qd * 32) << 16;
    const uint32_t s_addr = tmem + lane_base + C::s_col(t) + 64 * hf;
    const uint32_t pw_addr = tmem + lane_base + C::p_col(t) + C::P_HALF * hf;  // this half's P
    constexpr int DH = D / 2;  // output columns this thread rescales and writes
    const uint32_t o_addr = tmem + lane_base + C::o_col(t) + DH * hf;
    float* red = reinterpret_cast<float*>(smem + C::OFF_RED);    // [2][2][2][BM]
    float* lsum_x = reinterpret_cast<float*>(smem + C::OFF_LSUM);  // [2][2][2][BM]
    const int bar_id = 1 + t * 4 + qd;  // named barrier of the two warps sharing these rows
    const float sl2 = p.scale_log2;
    uint32_t s_cnt = 0, e_cnt = 0;
    bool ok = true;

    for (uint32_t k = 0; ok; ++k) {
      int w;
      if (!(ok = next_item(k, w)) || w < 0) break;
      bool bad = false;
      const Item it = get_item<D, MODE>(p, w, &bad);
      if (bad && threadIdx.x == 0) atomicOr(p.status, 1);
      const int n_t = t ? it.n1 : it.n0;
      const int row0 = it.row0 + t * BM;
      const int row = row0 + r;
      const int diag = row + it.koff;  // last visible key under the causal mask
      float m_use = -INFINITY, l = 0.f;
      const int lo_t = t ? it.lo1 : it.lo0;
      // 8-bit inputs: the scores of tile j are S_acc * q_scale * k_scale[j], so
      // the log2-domain factor is per tile; V's per-tile scale is folded into P
      // through the exponent, relative to the item's largest V scale v_ref so
      // that P stays within the E4M3 range (at most 2^8 with the stale max)
      float sl2_t = sl2, v_ref = 1.f;
      const float* ks_row = nullptr;
      const float* vs_row = nullptr;
      if constexpr (MODE == MODE_FP8) {
        if (n_t > 0) {
          ks_row = p.k_scale + static_cast<size_t>(it.kv_head) * p.n_kt;
          vs_row = p.v_scale + static_cast<size_t>(it.kv_head) * p.n_kt;
          const float sq = __ldg(p.q_scale + static_cast<size_t>(it.q_head) * p.n_qt + row0 / BM);
          bool good = sq > 0.f && sq < INFINITY;
          float vm = 0.f;
          for (int jj = lo_t + sm100::lane_id(); jj < n_t; jj += 32) {
            const float kv = __ldg(ks_row + jj), vv = __ldg(vs_row + jj);
            good = good && kv > 0.f && kv < INFINITY && vv > 0.f && vv < INFINITY;
            vm = fmaxf(vm, vv);
          }
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) vm = fmaxf(vm, __shfl_xor_sync(0xffffffffu, vm, o));
          if (!__all_sync(0xffffffffu, good) && sm100::lane_id() == 0)
            atomicOr(p.status, DEV_BAD_SCALE);
          sl2_t = sl2 * sq;
          v_ref = vm;
        }
      }
      for (int j = lo_t; j < n_t; ++j) {
        float sl2j = sl2_t, u_j = 0.f, rv = 1.f;
        if constexpr (MODE == MODE_FP8) {
          const float skj = __ldg(ks_row + j), svj = __ldg(vs_row + j);
          sl2j = sl2_t * skj;
          rv = v_ref / svj;       // >= 1: P of this tile is stored as p / rv
          u_j = -sm100::lg2(rv);
        }
        const float2 sl2x2 = make_float2(sl2j, sl2j);
        if (!(ok = sm100::mbar_wait(&s_full[t], s_cnt & 1, abort_flag, p.status))) break;
        float* red_w = red + ((s_cnt & 1) * 4 + t * 2) * BM;
        ++s_cnt;
        sm100::tc_fence_after();
        uint32_t s[64];
        sm100::tmem_ld32(s_addr, *reinterpret_cast<uint32_t(*)[32]>(&s[0]));
        sm100::tmem_ld32(s_addr + 32, *reinterpret_cast<uint32_t(*)[32]>(&s[32]));
        sm100::tmem_ld_wait();
        if constexpr (C::SEP_P) {  // the scores are in registers: S_t's columns are free
          sm100::tc_fence_before();
          __syncwarp();
          if (sm100::lane_id() == 0) sm100::mbar_arrive(&s_free[t]);
        }

        const int k0 = j * BN + 64 * hf;
        // sliding window: keys at or below the last row's window edge may be masked
        const bool win_edge =
            MODE == MODE_WINDOW && k0 <= row0 + (BM - 1) + it.koff - p.window;
        const bool need_mask =
            (k0 + 64 > it.kv_len) || (p.causal && (k0 + 63 > row0 + it.koff)) || win_edge;
        if (need_mask) {
          const int lim = p.causal ? min(it.kv_len - 1, diag) : it.kv_len - 1;
          const int lo_key = MODE == MODE_WINDOW ? diag - p.window + 1 : INT_MIN;
#pragma unroll
          for (int c = 0; c < 64; ++c)
            if (k0 + c > lim || k0 + c < lo_key) s[c] = __float_as_uint(-INFINITY);
        }
        float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
        for (int c = 0; c < 64; c += 4) {
          mx0 = sm100::max3(mx0, __uint_as_float(s[c]), __uint_as_float(s[c + 1]));
          mx1 = sm100::max3(mx1, __uint_as_float(s[c + 2]), __uint_as_float(s[c + 3]));
        }
        // the row max over all 128 keys: exchange with the warp holding the other half
        red_w[hf * BM + r] = fmaxf(mx0, mx1);
        sm100::named_bar_sync(bar_id, 64);
        const float m_new = fmaxf(fmaxf(mx0, mx1), red_w[(hf ^ 1) * BM + r]) * sl2j;
        const bool need = m_new > m_use + RESCALE_THRESHOLD;
        if constexpr (C::SEP_P) {
          // O and P_t are written below: PV_t of the previous P must have completed
          // (this S was issued before it)
          if (s_cnt > 1) {
            if (!(ok = sm100::mbar_wait(&p_free[t], (s_cnt - 2) & 1, abort_flag, p.status))) break;
            sm100::tc_fence_after();
          }
        }
        if (__any_sync(0xffffffffu, need)) {
          const float m_upd = fmaxf(m_use, m_new);
          const float alpha = (m_use == -INFINITY) ? 0.f : sm100::ex2(m_use - m_upd);
          l *= alpha;
          if (j > lo_t) {
            // O holds PV of the previous tiles (complete: S of this tile was
            // committed after them); rescale this thread's half in place
#pragma unroll 1
            for (int c = 0; c < DH / 16; ++c) {
              uint32_t o[16];
              sm100::tmem_ld16(o_addr + c * 16, o);
              sm100::tmem_ld_wait();
#pragma unroll
              for (int e = 0; e < 16; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
              sm100::tmem_st16(o_addr + c * 16, o);
            }
          }
          m_use = m_upd;
        }
        const float m_sub = (m_use == -INFINITY) ? 0.f : m_use;
        const float2 negm = make_float2(u_j - m_sub, u_j - m_sub);
        float2 lsum = make_float2(0.f, 0.f);
        auto exp_pair = [&](int cp) -> float2 {
          const float2 x = __ffma2_rn(
              make_float2(__uint_as_float(s[2 * cp]), __uint_as_float(s[2 * cp + 1])), sl2x2,
              negm);
          float2 e;
          if (poly_pair<D, EB>(cp)) {
            e = sm100::ex2_poly2(x);
          } else {
            e.x = sm100::ex2(x.x);
            e.y = sm100::ex2(x.y);
          }
          lsum = __fadd2_rn(lsum, e);
          return e;
        };
        // exponentials in two 32-column chunks; each chunk's P is stored to
        // TMEM while the next chunk is computed
        if constexpr (EB == 2) {
#pragma unroll
          for (int q = 0; q < 2; ++q) {
#pragma unroll
            for (int cp = 16 * q; cp < 16 * q + 16; ++cp) {
              const float2 e = exp_pair(cp);
              s[cp] = sm100::pack_bf16x2(e.x, e.y);
            }
            sm100::tmem_st16(pw_addr + 16 * q, &s[16 * q]);
          }
        } else {
#pragma unroll
          for (int q = 0; q < 2; ++q) {
#pragma unroll
            for (int cw = 8 * q; cw < 8 * q + 8; ++cw) {
              const float2 e0 = exp_pair(2 * cw), e1 = exp_pair(2 * cw + 1);
              s[cw] = sm100::pack_e4m3x4(e0.x, e0.y, e1.x, e1.y);
            }
            sm100::tmem_st8(pw_addr + 8 * q, &s[8 * q]);
          }
        }
        l += (lsum.x + lsum.y) * rv;
        sm100::tmem_st_wait();
        sm100::tc_fence_before();
        __syncwarp();
        if (sm100::lane_id() == 0) sm100::mbar_arrive(&p_full[t]);
      }
      if (!ok) break;
      // ---------------- epilogue: O = o / l (bf16), LSE = ln(2) * (m + log2 l)
      if (!(ok = sm100::mbar_wait(&o_full[t], k & 1, abort_flag, p.status))) break;
      sm100::tc_fence_after();
      const bool live = row < it.lq;
      // folding: both warps of a row read the accumulator's LSE before the
      // row-sum exchange below, which orders the write of the new LSE after it
      float lse_a = -INFINITY;
      const size_t rix = (static_cast<size_t>(it.b) * p.Hq + it.h) * p.Lq + (live ? row : 0);
      if constexpr (MODE == MODE_MERGE)
        if (live && !p.merge_init) lse_a = p.lse[rix];
      if (n_t > 0) {
        float* lx = lsum_x + ((e_cnt & 1) * 4 + t * 2) * BM;
        ++e_cnt;
        lx[hf * BM + r] = l;
        sm100::named_bar_sync(bar_id, 64);
        l += lx[(hf ^ 1) * BM + r];
      }
      const float inv = (l > 0.f) ? v_ref / l : 0.f;  // v_ref: P of 8-bit inputs is relative to it
      if constexpr (MODE == MODE_MERGE) {
        // normalised merge rule in LSE form with (O_a, LSE_a) = the accumulator and
        // (O_b, LSE_b) = this result: LSE = ln(e^LSE_a + e^LSE_b),
        // O = e^(LSE_a - LSE) O_a + e^(LSE_b - LSE) O_b, with O_b = o / l
        const float lse_b = (l > 0.f) ? (m_use + log2f(l)) * 0.69314718055994531f : -INFINITY;
        const float mx = fmaxf(lse_a, lse_b);
        float wa = 0.f, wb = 0.f, lse_new = -INFINITY;
        if (mx != -INFINITY) {
          wa = (lse_a == -INFINITY) ? 0.f : expf(lse_a - mx);
          wb = (lse_b == -INFINITY) ? 0.f : expf(lse_b - mx);
          const float ws = wa + wb;
          lse_new = mx + logf(ws);
          wa /= ws;
          wb = wb / ws * inv;
        }
        float* arow = p.o_acc + rix * D + DH * hf;
        __nv_bfloat16* orow = p.O ? p.O + rix * D + DH * hf : nullptr;
        // 32-byte loads and stores when both rows start on 32-byte boundaries
        const bool wide = ((reinterpret_cast<uintptr_t>(p.o_acc) |
                            reinterpret_cast<uintptr_t>(p.O)) & 31) == 0;
#pragma unroll 1
        for (int c = 0; c < DH / 16; ++c) {
          uint32_t o[16];
          if (n_t > 0) {  // warp-uniform: the TMEM load is collective
            sm100::tmem_ld16(o_addr + c * 16, o);
            sm100::tmem_ld_wait();
          } else {
#pragma unroll
            for (int e = 0; e < 16; ++e) o[e] = 0u;
          }
          if (live) {
            float4* a4 = reinterpret_cast<float4*>(arow + c * 16);
            uint32_t res[16];  // fp32 bits
            if (wide) {  // 32-byte accesses: whole sectors of this thread's row
              if (wa != 0.f) {
                ld_global_v8(arow + c * 16, &res[0]);
                ld_global_v8(arow + c * 16 + 8, &res[8]);
              } else {
#pragma unroll
                for (int e = 0; e < 16; ++e) res[e] = 0u;
              }
            } else {
#pragma unroll
              for (int v = 0; v < 4; ++v) {
                const float4 a = (wa != 0.f) ? a4[v] : make_float4(0.f, 0.f, 0.f, 0.f);
                res[4 * v] = __float_as_uint(a.x);
                res[4 * v + 1] = __float_as_uint(a.y);
                res[4 * v + 2] = __float_as_uint(a.z);
                res[4 * v + 3] = __float_as_uint(a.w);
              }
            }
#pragma unroll
            for (int e = 0; e < 16; ++e)
              res[e] = __float_as_uint(wa * __uint_as_float(res[e]) + wb * __uint_as_float(o[e]));
            if (wide) {
              st_global_v8(arow + c * 16, &res[0]);
              st_global_v8(arow + c * 16 + 8, &res[8]);
            } else {
#pragma unroll
              for (int v = 0; v < 4; ++v)
                a4[v] = make_float4(__uint_as_float(res[4 * v]), __uint_as_float(res[4 * v + 1]),
                                    __uint_as_float(res[4 * v + 2]),
                                    __uint_as_float(res[4 * v + 3]));
            }
            if (orow) {
              uint32_t pk[8];
#pragma unroll
              for (int e = 0; e < 8; ++e)
                pk[e] = sm100::pack_bf16x2(__uint_as_float(res[2 * e]),
                                           __uint_as_float(res[2 * e + 1]));
              if (wide) {
                st_global_v8(orow + c * 16, pk);
              } else {
                uint4* dst = reinterpret_cast<uint4*>(orow + c * 16);
                dst[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
                dst[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
              }
            }
          }
        }
        if (live && hf == 0) p.lse[rix] = lse_new;
        sm100::tc_fence_before();
        __syncwarp();
        if (sm100::lane_id() == 0) sm100::mbar_arrive(&o_empty[t]);
        continue;
      }
      __nv_bfloat16* orow;
      if constexpr (MODE == MODE_VARLEN)
        orow = p.O + it.o_off + (live ? row : 0) * it.o_rstride + DH * hf;
      else
        orow = p.O + ((static_cast<size_t>(it.b) * p.Hq + it.h) * p.Lq + (live ? row : 0)) * D +
               DH * hf;
      // each thread writes its own row, so a warp's store touches 32 rows: 32-byte
      // stores fill whole sectors (measured on B200, causal B4 H16 L4096 d128:
      // the O stores alone cost ~6 % of the kernel with 16-byte stores)
      const bool o_v8 = (reinterpret_cast<uintptr_t>(p.O) & 31) == 0;
      if (n_t > 0) {
#pragma unroll 1
        for (int c = 0; c < DH / 32; ++c) {
          uint32_t o[32];
          sm100::tmem_ld32(o_addr + c * 32, o);
          sm100::tmem_ld_wait();
          uint32_t pk[16];
#pragma unroll
          for (int e = 0; e < 16; ++e)
            pk[e] = sm100::pack_bf16x2(__uint_as_float(o[2 * e]) * inv,
                                       __uint_as_float(o[2 * e + 1]) * inv);
          if (live) {
            if (o_v8) {  // a row's 64 bytes as two full sectors
              st_global_v8(orow + c * 32, &pk[0]);
              st_global_v8(orow + c * 32 + 16, &pk[8]);
            } else {
              uint4* dst = reinterpret_cast<uint4*>(orow + c * 32);
#pragma unroll
              for (int v = 0; v < 4; ++v)
                dst[v] = make_uint4(pk[4 * v], pk[4 * v + 1], pk[4 * v + 2], pk[4 * v + 3]);
            }
          }
        }
      } else if (live) {
        uint4* dst = reinterpret_cast<uint4*>(orow);
        for (int v = 0; v < DH / 8; ++v) dst[v] = make_uint4(0, 0, 0, 0);
      }
      if (live && p.lse && hf == 0)
        p.lse[MODE == MODE_VARLEN ? it.lse_off + row
                                  : (static_cast<size_t>(it.b) * p.Hq + it.h) * p.Lq + row] =
            (l > 0.f) ? (m_use + log2f(l)) * 0.69314718055994531f : -INFINITY;
      sm100::tc_fence_before();
      __syncwarp();
      if (sm100::lane_id() == 0) sm100::mbar_arrive(&o_empty[t]);
    }
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

}  // namespace attn_fwd_impl
