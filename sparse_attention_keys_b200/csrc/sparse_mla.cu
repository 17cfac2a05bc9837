// dsa_sparse_mla: sparse MQA-style latent attention over the selected positions.
//
// For each (b, t, head h): z_u = scale * q[h] . kv[idx_u] over the 576 features (512 latent +
// 64 rotary), p = softmax over the selected u, out[h] = sum_u p_u kv[idx_u][0:512]. This is the
// absorbed MQA decode of "DeepSeek-V3.2-Exp - Similarities" (absorbed MQA decode excerpt: latent and
// rotary score terms, index mask, softmax, latent-weighted sum) with the index mask replaced by a
// gather of the selected rows, and the sparse-attention steps of the dense-block page
// (S' = S m^2/sqrt 192, A = softmax, O = AV).
//
// Tensor cores (tcgen05, kind::f16, bf16 in / fp32 accumulate in TMEM). A 128-head x 512 fp32
// output accumulator alone would fill all 512 TMEM columns, so each (query, key split) runs on two
// CTAs that split the OUTPUT features: CTA c accumulates out[:, 256c:256c+256) (256 TMEM columns).
// Each CTA computes the full 576-feature score itself, so the pair never exchanges data (1.5x the
// Q K^T work of a single pass; exchanging 128 x 32 fp32 partial scores per tile through distributed
// shared memory measured slower than recomputing them).
//
// TMEM: O [0,256), three 32-column score buffers [256,352), and Q features 0..319 of all 128 heads
// as bf16 pairs [352,512) (the A operand of the first 20 K-steps of Q K^T; the last 16 read Q
// features 320..575 from shared memory). The probabilities of tile j overwrite the first 16
// columns of the score buffer they came from (the A operand of P V).
//
// MMA issue: one thread issues a tcgen05.mma no faster than about every 30 ns (measured on B200),
// while a 128x32x16 MMA with A in TMEM takes about 9 ns on the tensor pipe, so Q K^T (36 MMAs
// per tile) is issued by three warps, one per score buffer (tile j uses buffer j mod 3), with every
// descriptor a precomputed base plus a constant; a fourth warp issues P V (two 128x256x16 MMAs per
// tile). Each buffer cycles through Q K^T, softmax and P V; three buffers keep the tensor pipe busy
// while the softmax of another tile runs.
//
// Selected 1152-byte latent rows are gathered in 32-key tiles by four warps with 16-byte cp.async
// (warp-wide 512-byte requests, unselected slots zero-filled), straight into the 128B-swizzled
// operand layout, split over two rings: the four 64-feature blocks this CTA's P V reads ("V ring",
// 16 KB per tile, 5 slots, freed when P V of the tile completes) and the other five blocks ("rest
// ring", 20 KB, 4 slots, freed as soon as Q K^T of the tile completes). Freeing the rest early lets
// the gathers run about four tiles ahead of the tensor core instead of waiting for P V.
// One shared-memory block is both the K-major B operand of Q K^T (N = keys) and the MN-major B
// operand of P V (N = features).
// Per CTA: 4 softmax warps (thread = head = TMEM lane), 1 P V warp, 4 gather warps (the first also
// loads Q features 320..575 by TMA), 3 Q K^T warps. The running max is only moved (and O rescaled in
// TMEM) when it grows by more than 2^32. With several key splits per query, fp32 partials (O, max,
// sum) go to the caller's workspace and a second kernel merges them.
#include <cuda_bf16.h>
#include <math.h>

#include <algorithm>

#include "common.cuh"
#include "kernels.h"

namespace dsa {

namespace {

constexpr int kHeads = 128;                        // TMEM lanes = MMA M
constexpr int kDqk = 576;
constexpr int kDv = 512;
constexpr int kKeys = 32;                          // selected keys per tile (N of Q K^T)
constexpr int kRegions = 9;                        // 576 features = 9 blocks of 64 (128 B), 128B swizzle
constexpr int kQTmemRegions = 5;                   // Q features 0..319 live in TMEM
constexpr int kQRegion = kHeads * 128;             // 16 KB
constexpr int kQBytes = (kRegions - kQTmemRegions) * kQRegion;   // 64 KB: features 320..575
constexpr int kKvRegion = kKeys * 128;             // 4 KB: one 64-feature block of a tile

// Shared-memory rings for the two layouts. 128 heads (a CTA pair per (query, split)): the "V ring"
// holds the four 64-feature blocks of this CTA's output half, the "rest ring" the other half's
// four and the rotary block. 64 heads (one CTA per (query, split), the head-parallel shard): the V
// ring holds all eight latent blocks, the rest ring the rotary block.
template <int HEADS>
struct MlaCfg {
  static_assert(HEADS == 128 || HEADS == 64, "128 heads, or a 64-head shard");
  static constexpr int kVRegions = HEADS == 128 ? 4 : 8;
  static constexpr int kRestRegions = kRegions - kVRegions;
  static constexpr int kVSlotBytes = kVRegions * kKvRegion;
  static constexpr int kRestSlotBytes = kRestRegions * kKvRegion;
  static constexpr int kVSlots = HEADS == 128 ? 5 : 4;
  static constexpr int kRestSlots = 4;
  static constexpr int kOffV = kQBytes;
  static constexpr int kOffRest = kOffV + kVSlots * kVSlotBytes;
  static constexpr int kOffBar = kOffRest + kRestSlots * kRestSlotBytes;
  static constexpr int kSmemBytes = 1024 + kOffBar + 256;
  static constexpr int kCtasPerUnit = HEADS == 128 ? 2 : 1;   // CTAs per (query, split)
};
constexpr int kSBufs = 3;
constexpr int kStageRow = 256 + 4;                 // floats per staged output row (1040 B: conflict-free)
static_assert(MlaCfg<128>::kOffV + kHeads * kStageRow * 4 <= MlaCfg<128>::kOffBar, "output staging fits");
static_assert(MlaCfg<64>::kOffV + kHeads * kStageRow * 4 <= MlaCfg<64>::kOffBar, "output staging fits");
static_assert(MlaCfg<128>::kSmemBytes <= 232448 && MlaCfg<64>::kSmemBytes <= 232448, "shared memory per CTA");
constexpr int kSoftmaxWarps = 4, kPvWarp = 4, kGatherWarp = 5, kGatherWarps = 4, kQkWarp = 9, kQkWarps = kSBufs;
constexpr int kMlaThreads = (kSoftmaxWarps + 1 + kGatherWarps + kQkWarps) * 32;
constexpr int kMaxSlots = 2048;                    // selected slots per CTA (split chunk cap)
constexpr int kTmemCols = 512;
constexpr uint32_t kTmemO = 0, kTmemS = 256, kTmemQ = kTmemS + kSBufs * kKeys;   // S: three 32-column buffers
constexpr float kLog2e = 1.4426950408889634f;
// The running max moves (and O is rescaled in TMEM, 256 columns per thread) only when a tile's
// max exceeds it by more than 2^32: P then stays below 2^32 (bf16 keeps its relative precision at
// any magnitude), l below 2^43 and O far from the fp32 range, and a rescale, which stalls the
// warp that does it while the other softmax warps wait at the next barrier, becomes rare.
constexpr float kRescaleThreshold = 32.0f;         // log2 units
static_assert(kTmemQ + kQTmemRegions * 32 == kTmemCols, "TMEM budget");

struct MlaSplit {
  int nsplit;
  int chunk;     // selected slots per split (multiple of kKeys, at most kMaxSlots)
};

// Key splits per query. Each CTA pays a fixed pipeline fill (about four tiles' time: Q staging and
// the first gather) and the splits need a merge pass, so the count minimises an estimate in tile
// units: waves x (tiles per CTA + fill) + merge, with waves = ceil(CTAs / SMs).
MlaSplit choose_split(int64_t BT, int k, int sms, int ctas_per_unit, int heads) {
  constexpr double kFillTiles = 4.0, kMergeTiles = 2.0;
  constexpr double kMergeTilesPerMB = 0.15;          // partials written + read, ~1.2 us per tile at HBM rate
  const int n_min = (k + kMaxSlots - 1) / kMaxSlots;  // a split holds at most kMaxSlots slots
  const int n_max = std::min((k + kKeys - 1) / kKeys, n_min + 256);
  MlaSplit best{0, 0};
  double best_cost = 1e300;
  for (int n = n_min; n <= n_max; ++n) {
    int chunk = (k + n - 1) / n;
    chunk = (chunk + kKeys - 1) / kKeys * kKeys;     // <= kMaxSlots, a multiple of kKeys
    const int nsplit = (k + chunk - 1) / chunk;
    const int64_t ctas = BT * ctas_per_unit * nsplit;
    const double waves = (double)((ctas + sms - 1) / sms);
    double cost = waves * (chunk / kKeys + kFillTiles);
    if (nsplit > 1) cost += kMergeTiles + kMergeTilesPerMB * (double)BT * nsplit * heads * kDv * 8 / 1e6;
    if (cost < best_cost) {
      best_cost = cost;
      best.nsplit = nsplit;
      best.chunk = chunk;
    }
  }
  return best;
}

// byte offset of 16-byte chunk `c` of row `r` in a 128B-swizzled tile of 128-byte rows
__device__ __forceinline__ uint32_t sw128(int r, int c) { return (uint32_t)(r * 128 + ((c ^ (r & 7)) << 4)); }

// 2^x with the MUFU approximation (relative error ~2^-22; softmax weights only need bf16 accuracy)
__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

}  // namespace

struct MlaParams {
  const uint16_t* q;
  const uint16_t* kv;
  const int32_t* idx;
  int B, T, S_max, k;
  int heads;                 // query heads per row of q / out / lse (128, or a 64-head shard)
  int q_ready;               // q is complete before the launch: it may be staged before the wait
  int nsplit, chunk;
  float scale_log2;          // softmax_scale * log2(e)
  uint16_t* out;
  float* lse;
  float* part_o;             // [BT][nsplit][heads][512]   (nsplit > 1)
  float* part_ml;            // [BT][nsplit][heads][2]     running max (log2 domain), sum
  int* status;
  // paged latent cache: kv is a pool of num_pages pages of page_size rows, and logical position v of
  // sequence b lives in row block_table[b][v / page_size] * page_size + v % page_size
  const int32_t* block_table;  // [B][max_pages]
  int max_pages, page_size, page_shift;   // page_size = 1 << page_shift
  int64_t num_pages;
};

// Pool row of logical position v (PAGED: pg = block_table[b][v / page_size], read one tile ahead),
// or -1 for a slot that takes no part: padding (v < 0), v >= S_max, or a page id outside the pool.
template <bool PAGED>
__device__ __forceinline__ bool kv_valid(const MlaParams& p, int v, int pg) {
  return v >= 0 && v < p.S_max && (!PAGED || (pg >= 0 && (int64_t)pg < p.num_pages));
}
template <bool PAGED>
__device__ __forceinline__ int kv_row(const MlaParams& p, int v, int pg) {
  if (!kv_valid<PAGED>(p, v, pg)) return -1;
  return PAGED ? (pg << p.page_shift) + (v & (p.page_size - 1)) : v;
}

// Q K^T of one 32-key tile: 20 K-steps with Q from TMEM, then 16 with Q from shared memory. LAYOUT
// fixes which ring holds each 64-feature block (0 / 1: the output half of a CTA of a 128-head pair;
// 2: the 64-head shard, latent blocks in the V ring and the rotary block in the rest ring), so every
// B descriptor is a base plus a constant. *_lo: low descriptor words (start address >> 4 in bits
// 0-13) of the shared-memory bases; hi: the common high word of the K-major 128B-swizzle descriptors.
template <int LAYOUT>
__device__ __forceinline__ void issue_qk_tile(uint32_t d, uint32_t tq, uint32_t q_lo, uint32_t v_lo, uint32_t r_lo,
                                              uint32_t hi, uint32_t idesc) {
#pragma unroll
  for (int r = 0; r < kRegions; ++r) {
    const bool in_v = LAYOUT == 2 ? r < 8 : (r < 8 && (r >> 2) == LAYOUT);
    const int v_blk = LAYOUT == 2 ? r : (r & 3);
    const int r_blk = LAYOUT == 2 ? 0 : (r == 8 ? 4 : (r & 3));
    const uint32_t kb = in_v ? v_lo + (uint32_t)((v_blk * kKvRegion) >> 4) : r_lo + (uint32_t)((r_blk * kKvRegion) >> 4);
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
      const int ks = 4 * r + kk;
      if (r < kQTmemRegions) {
        if (ks == 0) mma_f16_ts_lo<0>(d, tq, kb, hi, idesc);
        else mma_f16_ts_lo<1>(d, tq + ks * 8, kb + kk * 2, hi, idesc);
      } else {
        mma_f16_ss_lo<1>(d, q_lo + (uint32_t)(((r - kQTmemRegions) * kQRegion) >> 4) + kk * 2, hi, kb + kk * 2, hi,
                         idesc);
      }
    }
  }
}

// HEADS = 128: two CTAs per (query, key split), CTA c owning output features [256c, 256c + 256).
// HEADS = 64 (a head-parallel shard of the 128 heads): one CTA per (query, key split). TMEM lanes
// 64..127 hold a copy of heads 0..63 (their Q rows are staged twice, so Q K^T writes every score
// row twice), and P V runs block-diagonally: lanes 0..63 write P into the first 16 columns of the
// score buffer and zeros into the last 16, lanes 64..127 the reverse, and four MMAs accumulate
// P V[:, 0:256] into lanes 0..63 and P V[:, 256:512] into lanes 64..127 of the same 256 O columns.
template <bool PAGED, int HEADS>
__global__ void __launch_bounds__(kMlaThreads, 1)
    sparse_mla_kernel(const __grid_constant__ CUtensorMap q_map, const MlaParams p) {
  using Cfg = MlaCfg<HEADS>;
  constexpr int kVRegions = Cfg::kVRegions, kVSlots = Cfg::kVSlots, kRestSlots = Cfg::kRestSlots;
  constexpr int kVSlotBytes = Cfg::kVSlotBytes, kRestSlotBytes = Cfg::kRestSlotBytes;
  constexpr int kOffV = Cfg::kOffV, kOffRest = Cfg::kOffRest, kOffBar = Cfg::kOffBar;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* q_sm = smem;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kOffBar);
  uint64_t* kv_full = bars;                         // [kRestSlots] gather (cp.async) -> Q K^T issuer
  uint64_t* rest_empty = bars + kRestSlots;         // [kRestSlots] Q K^T done -> gather
  uint64_t* v_empty = bars + 2 * kRestSlots;        // [kVSlots]    P V done -> gather
  uint64_t* s_full = v_empty + kVSlots;             // [kSBufs] Q K^T done -> softmax (per score buffer)
  uint64_t* p_full = s_full + kSBufs;               // [kSBufs] softmax (P in TMEM) -> P V issuer
  uint64_t* pv_done = p_full + kSBufs;              // [kSBufs] P V done -> Q K^T issuer, softmax (O rescale)
  uint64_t* q_full = pv_done + kSBufs;              // TMA (Q in smem) + softmax (Q in TMEM) -> Q K^T issuers
  uint64_t* o_full = q_full + 1;                    // last P V done -> epilogue
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_flag;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // 128 heads: this CTA's output features [256*half, 256*half + 256); 64 heads: one CTA per unit
  const int half = HEADS == 128 ? (int)(blockIdx.x & 1) : 0;
  const int unit = HEADS == 128 ? (int)(blockIdx.x >> 1) : (int)blockIdx.x;
  const int q_head = tid & (HEADS - 1);        // softmax thread: the query head of its TMEM lane
  const int split = unit % p.nsplit;
  const int64_t bt = unit / p.nsplit;
  const int b = (int)(bt / p.T);
  const int slot0 = split * p.chunk;
  const int nslots = max(0, min(p.k, slot0 + p.chunk) - slot0);
  const int ntiles = (nslots + kKeys - 1) / kKeys;
  const int32_t* idx_row = p.idx + bt * p.k + slot0;
  const uint32_t v_ring = smem_u32(smem + kOffV), rest_ring = smem_u32(smem + kOffRest);

  // Before the set-up barrier, hint each head's features 0..319 into L2 (softmax warps, staged into
  // TMEM below). A prefetch is only a hint, so it is safe even if the preceding kernel is still
  // writing Q; every actual read of Q (unless the caller stated that Q is complete before the
  // launch), and of the indices, comes after grid_dep_wait.
  if (warp < kSoftmaxWarps && ntiles > 0) {
    const char* qrow = reinterpret_cast<const char*>(p.q + (bt * HEADS + q_head) * kDqk);
#pragma unroll
    for (int i = 0; i < kQTmemRegions; ++i) asm volatile("prefetch.global.L2 [%0];" ::"l"(qrow + 128 * i));
  }

  if (tid == 0) {
    abort_flag = 0;
    for (int s = 0; s < kRestSlots; ++s) {
      mbar_init(&kv_full[s], kGatherWarps * 32);
      mbar_init(&rest_empty[s], 1);
    }
    for (int s = 0; s < kVSlots; ++s) mbar_init(&v_empty[s], 1);
    for (int i = 0; i < kSBufs; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&p_full[i], kSoftmaxWarps * 32);
      mbar_init(&pv_done[i], 1);
    }
    mbar_init(q_full, 1 + kSoftmaxWarps * 32);
    mbar_init(o_full, 1);
    fence_barrier_init();
  }
  if (warp == kPvWarp) {
    tmem_alloc(&tmem_base_sh, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_sh;
  grid_dep_launch();                                 // the next kernel may start its set-up

  if (warp >= kQkWarp) {
    // ------------------------------------------------------------------ Q K^T issuers
    // warp kQkWarp + e issues Q K^T of the tiles j = e (mod 3) into score buffer e: with one score
    // buffer per issuing thread, a buffer's softmax and P V overlap the other buffers' Q K^T
    const int e = warp - kQkWarp;
    if (lane == 0 && ntiles > e) {
      const uint32_t idesc_s = idesc_f32acc(1 /*BF16*/, 1, 128, kKeys, 0, 0);
      const uint64_t q_desc = sdesc_kmajor_sw128(smem_u32(q_sm));
      const uint32_t hi = (uint32_t)(q_desc >> 32), q_lo = (uint32_t)q_desc;
      const uint32_t v_lo0 = (uint32_t)sdesc_kmajor_sw128(v_ring), r_lo0 = (uint32_t)sdesc_kmajor_sw128(rest_ring);
      const uint32_t d = tmem + kTmemS + e * kKeys, tq = tmem + kTmemQ;
      bool ok = mbar_wait(q_full, 0, &abort_flag, p.status, DSA_SITE_MLA_Q);
      for (int j = e; ok && j < ntiles; j += kSBufs) {
        // score buffer e still holds P of tile j - 3 until its P V completes
        if (j >= kSBufs &&
            !mbar_wait(&pv_done[e], ((j / kSBufs) + 1) & 1, &abort_flag, p.status, DSA_SITE_MLA_P_EMPTY))
          break;
        if (!mbar_wait(&kv_full[j % kRestSlots], (j / kRestSlots) & 1, &abort_flag, p.status, DSA_SITE_MLA_KV_FULL))
          break;
        fence_proxy_async_smem();        // cp.async (generic proxy) writes -> MMA (async proxy) reads
        tc_fence_after();
        const uint32_t v_lo = v_lo0 + (uint32_t)(((j % kVSlots) * kVSlotBytes) >> 4);
        const uint32_t r_lo = r_lo0 + (uint32_t)(((j % kRestSlots) * kRestSlotBytes) >> 4);
        if (HEADS == 64) issue_qk_tile<2>(d, tq, q_lo, v_lo, r_lo, hi, idesc_s);
        else if (half == 0) issue_qk_tile<0>(d, tq, q_lo, v_lo, r_lo, hi, idesc_s);
        else issue_qk_tile<1>(d, tq, q_lo, v_lo, r_lo, hi, idesc_s);
        mma_commit(&s_full[e]);
        mma_commit(&rest_empty[j % kRestSlots]);
      }
    }
  } else if (warp >= kGatherWarp) {
    // ------------------------------------------------------------------ gather warps
    // gather warp w copies keys 8w..8w+7 of each tile; for every key, lane L copies the 16-byte
    // chunks L (block L/8), L+32 (block 4+L/8) and, for L < 8, L+64 (the rotary block)
    const int w = warp - kGatherWarp;
    if (!p.q_ready) grid_dep_wait();                 // Q may come from the preceding kernel
    if (w == 0 && lane == 0 && ntiles > 0) {
      prefetch_tensormap(&q_map);
      mbar_arrive_expect_tx(q_full, kQBytes);
      for (int r = kQTmemRegions; r < kRegions; ++r) {
        uint8_t* dst = q_sm + (r - kQTmemRegions) * kQRegion;
        tma_load_2d(dst, &q_map, q_full, 64 * r, (int32_t)(bt * HEADS));
        // 64 heads: the same 64 rows again into rows 64..127 (8 KB on: whole 8-row swizzle atoms)
        if (HEADS == 64) tma_load_2d(dst + 64 * 128, &q_map, q_full, 64 * r, (int32_t)(bt * HEADS));
      }
    }
    if (p.q_ready) grid_dep_wait();                  // the indices may come from the preceding kernel
    const uint16_t* kv_b = PAGED ? p.kv : p.kv + (int64_t)b * p.S_max * kDqk;
    const int32_t* pages = PAGED ? p.block_table + (int64_t)b * p.max_pages : nullptr;
    const uint32_t blk = (uint32_t)(lane >> 3) * kKvRegion;      // block of chunks L and L+32 in its ring slot
    auto load_idx = [&](int j) -> int {
      const int slot = j * kKeys + 8 * w + (lane & 7);
      return (j < ntiles && slot < nslots) ? __ldg(idx_row + slot) : -1;
    };
    auto load_page = [&](int v) -> int { return (v >= 0 && v < p.S_max) ? __ldg(pages + (v >> p.page_shift)) : -1; };
    // dense: indices one tile ahead; paged: indices two tiles ahead, their page ids one tile ahead
    int idx_next = load_idx(0);
    int pg_next = 0, idx_next2 = -1;
    if (PAGED) {
      idx_next2 = load_idx(1);
      pg_next = load_page(idx_next);
    }
    for (int j = 0; j < ntiles; ++j) {
      const int idx_cur = idx_next, pg_cur = pg_next;
      if (PAGED) {
        idx_next = idx_next2;
        idx_next2 = load_idx(j + 2);
        pg_next = load_page(idx_next);
      } else {
        idx_next = load_idx(j + 1);
      }
      const int row_cur = kv_row<PAGED>(p, idx_cur, pg_cur);
      // a selected position past the cache, or (paged) on a page outside the pool
      if (lane < 8 && idx_cur >= 0 && row_cur < 0) set_status(p.status, DSA_ERR_DEVICE_BOUNDS);
      if (j >= kRestSlots &&
          !__all_sync(0xffffffffu, mbar_wait(&rest_empty[j % kRestSlots], ((j / kRestSlots) + 1) & 1, &abort_flag,
                                             p.status, DSA_SITE_MLA_KV_EMPTY)))
        break;
      if (j >= kVSlots &&
          !__all_sync(0xffffffffu, mbar_wait(&v_empty[j % kVSlots], ((j / kVSlots) + 1) & 1, &abort_flag,
                                             p.status, DSA_SITE_MLA_KV_EMPTY)))
        break;
      const uint32_t v_slot = v_ring + (j % kVSlots) * kVSlotBytes;
      const uint32_t r_slot = rest_ring + (j % kRestSlots) * kRestSlotBytes;
      // latent blocks L/8 and 4 + L/8, and the rotary block
      const uint32_t d0 = HEADS == 64 ? v_slot + blk : (half == 0 ? v_slot : r_slot) + blk;
      const uint32_t d1 = HEADS == 64 ? v_slot + 4 * kKvRegion + blk : (half == 1 ? v_slot : r_slot) + blk;
      const uint32_t d2 = HEADS == 64 ? r_slot : r_slot + 4 * kKvRegion;
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        const int row = __shfl_sync(0xffffffffu, row_cur, kk);
        const bool ok = row >= 0;
        const uint32_t off = sw128(8 * w + kk, lane & 7);
        const uint16_t* src = kv_b + (int64_t)(ok ? row : 0) * kDqk + lane * 8;
        cp_async_16_zfill(d0 + off, src, ok);
        cp_async_16_zfill(d1 + off, src + 256, ok);
        if (lane < 8) cp_async_16_zfill(d2 + off, src + 512, ok);
      }
      cp_async_mbar_arrive(&kv_full[j % kRestSlots]);
    }
    cp_async_wait_all();
  } else if (warp == kPvWarp) {
    // ------------------------------------------------------------------ P V issuer
    if (lane == 0 && ntiles > 0) {
      const uint32_t idesc_pv = idesc_f32acc(1, 1, 128, 256, 0, 1 /*B MN-major*/);
      const uint64_t v_desc = sdesc_mnmajor_sw128(v_ring, kKvRegion, 1024);
      const uint32_t hi = (uint32_t)(v_desc >> 32), v_lo0 = (uint32_t)v_desc;
      for (int j = 0; j < ntiles; ++j) {
        if (!mbar_wait(&p_full[j % kSBufs], (j / kSBufs) & 1, &abort_flag, p.status, DSA_SITE_MLA_P_FULL)) break;
        tc_fence_after();
        const uint32_t v_lo = v_lo0 + (uint32_t)(((j % kVSlots) * kVSlotBytes) >> 4);
        const uint32_t a = tmem + kTmemS + (j % kSBufs) * kKeys;
        if (j == 0) mma_f16_ts_lo<0>(tmem + kTmemO, a, v_lo, hi, idesc_pv);
        else mma_f16_ts_lo<1>(tmem + kTmemO, a, v_lo, hi, idesc_pv);
        mma_f16_ts_lo<1>(tmem + kTmemO, a + 8, v_lo + (2048 >> 4), hi, idesc_pv);    // keys 16..31
        if (HEADS == 64) {       // the block-diagonal second half: P of lanes 64..127 times V[:, 256:512]
          mma_f16_ts_lo<1>(tmem + kTmemO, a + 16, v_lo + ((4 * kKvRegion) >> 4), hi, idesc_pv);
          mma_f16_ts_lo<1>(tmem + kTmemO, a + 24, v_lo + ((4 * kKvRegion + 2048) >> 4), hi, idesc_pv);
        }
        mma_commit(&pv_done[j % kSBufs]);
        mma_commit(&v_empty[j % kVSlots]);
      }
      mma_commit(o_full);
    }
  } else {
    // ------------------------------------------------------------------ softmax warps (thread = head)
    const int h = tid;
    const uint32_t t_row = tmem + ((uint32_t)(warp * 32) << 16);
    if (!p.q_ready) grid_dep_wait();                 // Q may come from the preceding kernel
    // Q features 0..319 of head h -> TMEM as bf16 pairs (feature f in column f/2)
    if (ntiles > 0) {
      // two batches of loads, each fully in flight before its TMEM stores (which order memory)
      const uint4* qrow = reinterpret_cast<const uint4*>(p.q + (bt * HEADS + q_head) * kDqk);
      auto stage = [&](int c0, int nc) {
        uint4 v[3 * 8];
#pragma unroll
        for (int i = 0; i < 3 * 8; ++i)
          if (i < nc * 8) v[i] = __ldg(qrow + 8 * c0 + i);
#pragma unroll
        for (int c = 0; c < 3; ++c) {
          if (c < nc) {
            uint32_t buf[32];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              buf[4 * i] = v[8 * c + i].x; buf[4 * i + 1] = v[8 * c + i].y;
              buf[4 * i + 2] = v[8 * c + i].z; buf[4 * i + 3] = v[8 * c + i].w;
            }
            tmem_st32(t_row + kTmemQ + (c0 + c) * 32, buf);
          }
        }
      };
      static_assert(kQTmemRegions == 5, "Q staging batches");
      stage(0, 3);
      stage(3, 2);
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(q_full);
    }
    if (p.q_ready) grid_dep_wait();                  // the indices (earlier kernels); outputs written below
    float m = -INFINITY, l = 0.f;
    bool ok = true;
    // slot j * 32 + lane of the next tile (paged: also the slot two tiles ahead and the next tile's page id)
    const int32_t* pages = PAGED ? p.block_table + (int64_t)b * p.max_pages : nullptr;
    auto load_page = [&](int v) -> int { return (v >= 0 && v < p.S_max) ? __ldg(pages + (v >> p.page_shift)) : -1; };
    int v_next = lane < nslots ? __ldg(idx_row + lane) : -1;
    int pg_next = 0, v_next2 = -1;
    if (PAGED) {
      v_next2 = kKeys + lane < nslots ? __ldg(idx_row + kKeys + lane) : -1;
      pg_next = load_page(v_next);
    }
#pragma unroll 1
    for (int j = 0; ok && j < ntiles; ++j) {
      const uint32_t s_col = kTmemS + (j % kSBufs) * kKeys;
      const int v_cur = v_next, pg_cur = pg_next;
      if (PAGED) {
        v_next = v_next2;
        const int sn = (j + 2) * kKeys + lane;
        v_next2 = sn < nslots ? __ldg(idx_row + sn) : -1;
        pg_next = load_page(v_next);
      } else {
        const int sn = (j + 1) * kKeys + lane;
        v_next = sn < nslots ? __ldg(idx_row + sn) : -1;
      }
      const uint32_t vmask = __ballot_sync(0xffffffffu, kv_valid<PAGED>(p, v_cur, pg_cur));
      if (!__all_sync(0xffffffffu, mbar_wait(&s_full[j % kSBufs], (j / kSBufs) & 1, &abort_flag, p.status,
                                             DSA_SITE_MLA_S_FULL))) {
        ok = false;
        break;
      }
      tc_fence_after();
      uint32_t r0[32];
      tmem_ld32(t_row + s_col, r0);
      tmem_ld_wait();
      float z[kKeys];
#pragma unroll
      for (int i = 0; i < kKeys; ++i) z[i] = ((vmask >> i) & 1u) ? __uint_as_float(r0[i]) * p.scale_log2 : -INFINITY;
      float t4[4];
#pragma unroll
      for (int g = 0; g < 4; ++g)
        t4[g] = fmaxf(fmaxf(fmaxf(z[8 * g], z[8 * g + 1]), fmaxf(z[8 * g + 2], z[8 * g + 3])),
                      fmaxf(fmaxf(z[8 * g + 4], z[8 * g + 5]), fmaxf(z[8 * g + 6], z[8 * g + 7])));
      const float mx = fmaxf(fmaxf(t4[0], t4[1]), fmaxf(t4[2], t4[3]));
      float m_new = m, alpha = 1.f;
      if (mx > m + kRescaleThreshold) {
        m_new = mx;
        alpha = (m == -INFINITY) ? 0.f : fast_exp2(m - m_new);
      }
      uint32_t pk[kKeys / 2];
      float rs8[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int i = 0; i < kKeys; i += 2) {
        const float e0 = (m_new == -INFINITY) ? 0.f : fast_exp2(z[i] - m_new);
        const float e1 = (m_new == -INFINITY) ? 0.f : fast_exp2(z[i + 1] - m_new);
        rs8[(i >> 1) & 7] += e0 + e1;
        pk[i / 2] = pack_bf16(e0, e1);
      }
      l = l * alpha + (((rs8[0] + rs8[1]) + (rs8[2] + rs8[3])) + ((rs8[4] + rs8[5]) + (rs8[6] + rs8[7])));
      // O rescale: P V of every earlier tile must be done first (P V of tile j - 1 completes last)
      const bool rescale = (m != -INFINITY) && (m_new != m);
      if (__any_sync(0xffffffffu, rescale)) {
        if (j >= 1 && !__all_sync(0xffffffffu, mbar_wait(&pv_done[(j - 1) % kSBufs], ((j - 1) / kSBufs) & 1, &abort_flag,
                                                         p.status, DSA_SITE_MLA_P_EMPTY))) {
          ok = false;
          break;
        }
        tc_fence_after();
        const float a = rescale ? alpha : 1.f;
#pragma unroll 1
        for (int c = 0; c < 8; ++c) {
          uint32_t o[32];
          tmem_ld32(t_row + kTmemO + c * 32, o);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * a);
          tmem_st32(t_row + kTmemO + c * 32, o);
        }
      }
      m = m_new;
      if (HEADS == 128) {
        tmem_st16(t_row + s_col, pk);            // P over the scores it came from
      } else {                                   // the block-diagonal P of the 64-head shard
        uint32_t pz[2 * (kKeys / 2)];
        const bool low = warp < 2;               // lanes 0..63
#pragma unroll
        for (int i = 0; i < kKeys / 2; ++i) {
          pz[i] = low ? pk[i] : 0u;
          pz[kKeys / 2 + i] = low ? 0u : pk[i];
        }
        tmem_st32(t_row + s_col, pz);
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(&p_full[j % kSBufs]);
    }
    // ---- epilogue: O row (this CTA's 256 output features) / l
    const bool have_o = ntiles > 0 && ok &&
                        __all_sync(0xffffffffu, mbar_wait(o_full, 0, &abort_flag, p.status, DSA_SITE_MLA_O_FULL));
    if (have_o) tc_fence_after();
    // Each thread stages its head's row of this CTA's 256 output features (bf16 output, or the fp32
    // partial of a key split) in the now idle KV rings, then one bulk copy (TMA engine) per row
    // writes it out: the row is contiguous in global memory.
    const bool final_out = p.nsplit == 1;
    // 128 heads: lane h is head h, features of this CTA's half; 64 heads: lane h is head h mod 64,
    // features [256 * (h / 64), + 256)
    const int o_half = HEADS == 128 ? half : (h >> 6);
    const float scale = final_out ? (l > 0.f ? 1.f / l : 0.f) : 1.f;
    uint8_t* srow = smem + kOffV + h * kStageRow * 4;
#pragma unroll 1
    for (int c = 0; c < 8; c += 2) {
      uint32_t o[2][32];
      if (have_o) {
        tmem_ld32(t_row + kTmemO + c * 32, o[0]);
        tmem_ld32(t_row + kTmemO + (c + 1) * 32, o[1]);
        tmem_ld_wait();
      } else {
#pragma unroll
        for (int i = 0; i < 32; ++i) o[0][i] = o[1][i] = 0u;
      }
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        const int f0 = (c + hh) * 32;                 // first feature of this 32-column chunk
        if (final_out) {
          uint4* dst = reinterpret_cast<uint4*>(srow + f0 * 2);
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const uint32_t* v = &o[hh][8 * i];
            dst[i] = make_uint4(pack_bf16(__uint_as_float(v[0]) * scale, __uint_as_float(v[1]) * scale),
                                pack_bf16(__uint_as_float(v[2]) * scale, __uint_as_float(v[3]) * scale),
                                pack_bf16(__uint_as_float(v[4]) * scale, __uint_as_float(v[5]) * scale),
                                pack_bf16(__uint_as_float(v[6]) * scale, __uint_as_float(v[7]) * scale));
          }
        } else {
          uint4* dst = reinterpret_cast<uint4*>(srow + f0 * 4);
#pragma unroll
          for (int i = 0; i < 8; ++i) dst[i] = make_uint4(o[hh][4 * i], o[hh][4 * i + 1], o[hh][4 * i + 2], o[hh][4 * i + 3]);
        }
      }
    }
    fence_proxy_async_smem();                          // the row's generic writes -> the bulk copy's reads
    if (final_out) {
      bulk_store_s2g(p.out + (bt * HEADS + q_head) * kDv + 256 * o_half, smem_u32(srow), 256 * 2);
      if (p.lse && o_half == 0)
        p.lse[bt * HEADS + q_head] = l > 0.f ? (m + log2f(l)) * 0.6931471805599453f : -INFINITY;
    } else {
      const int64_t prow = (bt * p.nsplit + split) * HEADS + q_head;
      bulk_store_s2g(p.part_o + prow * kDv + 256 * o_half, smem_u32(srow), 256 * 4);
      if (o_half == 0) *reinterpret_cast<float2*>(p.part_ml + prow * 2) = make_float2(m, l);
    }
    bulk_commit();
    bulk_wait_all();                                   // shared memory stays valid until the copy is done
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kPvWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// Merge the key-split partials: one warp per (query, head), 16 output features per lane. The
// splits' (max, sum) pairs are read one per lane and reduced across the warp; the partial O rows
// are then streamed four splits at a time so that their loads overlap.
__global__ void __launch_bounds__(256) sparse_mla_combine_kernel(const MlaParams p, int64_t rows) {
  const int64_t wid = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  grid_dep_wait();                                   // the partials come from the preceding kernel
  grid_dep_launch();
  if (wid >= rows) return;
  const int64_t bt = wid / p.heads;
  const int head = (int)(wid - bt * p.heads);
  const float2* ml = reinterpret_cast<const float2*>(p.part_ml);
  auto ml_of = [&](int s) { return __ldg(ml + (bt * p.nsplit + s) * p.heads + head); };
  float m_all = -INFINITY;
  for (int s = lane; s < p.nsplit; s += 32) m_all = fmaxf(m_all, ml_of(s).x);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m_all = fmaxf(m_all, __shfl_xor_sync(0xffffffffu, m_all, o));
  auto weight = [&](float m) { return m == -INFINITY ? 0.f : exp2f(m - m_all); };
  float l_all = 0.f;
  for (int s = lane; s < p.nsplit; s += 32) {
    const float2 v = ml_of(s);
    l_all += v.y * weight(v.x);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) l_all += __shfl_xor_sync(0xffffffffu, l_all, o);
  float acc[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) acc[i] = 0.f;
  for (int s0 = 0; s0 < p.nsplit; s0 += 4) {
    float4 v[4][4];
    float wgt[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int s = s0 + u;
      wgt[u] = 0.f;
      if (s < p.nsplit) {
        wgt[u] = weight(ml_of(s).x);
        const float4* src =
            reinterpret_cast<const float4*>(p.part_o + ((bt * p.nsplit + s) * p.heads + head) * kDv + lane * 16);
#pragma unroll
        for (int i = 0; i < 4; ++i) v[u][i] = __ldcs(src + i);
      }
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      if (wgt[u] == 0.f) continue;       // split with no selected key (or beyond nsplit)
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        acc[4 * i] += v[u][i].x * wgt[u]; acc[4 * i + 1] += v[u][i].y * wgt[u];
        acc[4 * i + 2] += v[u][i].z * wgt[u]; acc[4 * i + 3] += v[u][i].w * wgt[u];
      }
    }
  }
  const float inv = l_all > 0.f ? 1.f / l_all : 0.f;
  uint32_t packed[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) packed[i] = pack_bf16(acc[2 * i] * inv, acc[2 * i + 1] * inv);
  uint4* dst = reinterpret_cast<uint4*>(p.out + (bt * p.heads + head) * kDv + lane * 16);
  dst[0] = make_uint4(packed[0], packed[1], packed[2], packed[3]);
  dst[1] = make_uint4(packed[4], packed[5], packed[6], packed[7]);
  if (p.lse && lane == 0)
    p.lse[bt * p.heads + head] = l_all > 0.f ? (m_all + log2f(l_all)) * 0.6931471805599453f : -INFINITY;
}

static MlaSplit split_for(int64_t BT, int k, int heads) {
  return choose_split(BT, k, dsa_host::device_sm_count(), heads == 128 ? MlaCfg<128>::kCtasPerUnit : MlaCfg<64>::kCtasPerUnit,
                      heads);
}

size_t sparse_mla_workspace_size(int B, int T, int k, int heads) {
  const int64_t BT = (int64_t)B * T;
  const MlaSplit s = split_for(BT, k, heads);
  if (s.nsplit <= 1) return 0;
  return (size_t)BT * s.nsplit * heads * (kDv + 2) * sizeof(float);
}

template <bool PAGED, int HEADS>
static int launch_mla(const uint16_t* q, MlaParams p, cudaStream_t stream, void* workspace, size_t ws_bytes) {
  using Cfg = MlaCfg<HEADS>;
  const int64_t BT = (int64_t)p.B * p.T;
  if (BT == 0) return DSA_OK;
  p.heads = HEADS;
  const MlaSplit s = split_for(BT, p.k, HEADS);
  p.nsplit = s.nsplit; p.chunk = s.chunk;
  if (s.nsplit > 1) {
    const size_t need = (size_t)BT * s.nsplit * HEADS * (kDv + 2) * sizeof(float);
    if (workspace == nullptr || ws_bytes < need) return DSA_ERR_WORKSPACE;
    p.part_o = static_cast<float*>(workspace);
    p.part_ml = p.part_o + (size_t)BT * s.nsplit * HEADS * kDv;
  }
  static uint64_t configured[dsa_host::kMaxSetupDevices] = {};
  if (dsa_host::needs_setup(configured, nullptr)) {
    if (cudaFuncSetAttribute(sparse_mla_kernel<PAGED, HEADS>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             Cfg::kSmemBytes) != cudaSuccess)
      return DSA_ERR_CUDA;
    dsa_host::mark_setup(configured);
  }
  const int64_t grid = BT * s.nsplit * Cfg::kCtasPerUnit;
  if (grid > 0x7fffffff) return DSA_ERR_INVALID_ARG;
  CUtensorMap q_map;                               // Q rows of HEADS heads, boxes of 64 features
  if (!dsa_host::encode_tensor_map_2d(&q_map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, (void*)q, kDqk,
                                      (uint64_t)BT * HEADS, kDqk * 2, 64, HEADS, CU_TENSOR_MAP_SWIZZLE_128B))
    return DSA_ERR_CUDA;
  int rc = dsa_host::launch(sparse_mla_kernel<PAGED, HEADS>, dim3((unsigned)grid), dim3(kMlaThreads), Cfg::kSmemBytes,
                            stream, q_map, p);
  if (rc != DSA_OK || s.nsplit == 1) return rc;
  const int64_t rows = BT * HEADS;
  return dsa_host::launch(sparse_mla_combine_kernel, dim3((unsigned)((rows + 7) / 8)), dim3(256), 0, stream, p, rows);
}

int launch_sparse_mla(const uint16_t* q, const uint16_t* kv, const int32_t* idx, int B, int T,
                      int S_max, int k, int heads, float softmax_scale, uint16_t* out, float* lse,
                      void* workspace, size_t ws_bytes, bool q_ready, cudaStream_t stream, int* status) {
  MlaParams p{};
  p.q_ready = q_ready ? 1 : 0;
  p.q = q; p.kv = kv; p.idx = idx; p.B = B; p.T = T; p.S_max = S_max; p.k = k;
  p.scale_log2 = softmax_scale * kLog2e;
  p.out = out; p.lse = lse; p.status = status;
  if (heads == 64) return launch_mla<false, 64>(q, p, stream, workspace, ws_bytes);
  return launch_mla<false, 128>(q, p, stream, workspace, ws_bytes);
}

int launch_sparse_mla_paged(const uint16_t* q, const uint16_t* kv_pool, int64_t num_pages,
                            const int32_t* block_table, int max_pages, int page_size, const int32_t* idx, int B,
                            int T, int k, float softmax_scale, uint16_t* out, float* lse, void* workspace,
                            size_t ws_bytes, cudaStream_t stream, int* status) {
  MlaParams p{};
  p.q = q; p.kv = kv_pool; p.idx = idx; p.B = B; p.T = T; p.S_max = max_pages * page_size; p.k = k;
  p.scale_log2 = softmax_scale * kLog2e;
  p.out = out; p.lse = lse; p.status = status;
  p.block_table = block_table; p.max_pages = max_pages; p.page_size = page_size; p.num_pages = num_pages;
  p.page_shift = __builtin_ctz((unsigned)page_size);
  return launch_mla<true, 128>(q, p, stream, workspace, ws_bytes);
}

}  // namespace dsa
