// dsa_index_scores: lightning-indexer scores on the FP8 tensor cores (tcgen05, kind::f8f6f4).
//
// Computes I[b,t,s] = k_scale[b,s] * sum_j w'[b,t,j] * ReLU(q8[b,t,j,:] . k8[b,s,:]) for every
// visible s (s <= q_pos, s < kv_len), w' = w * 64^-0.5 * q_scale * softmax_scale: the fp8_index
// call and weight fold of Indexer.forward ("DeepSeek-V3.2-Exp - Rotate first features",
// Indexer.forward excerpt) and S^I of the lightning-indexer steps (dense-block page).
//
// Tile: the MMA's M = 128 keys (A = K-cache rows, K-major, 128 B each = one 128B-swizzle atom
// row), N = NQ queries x 64 heads (B = the queries' FP8 head rows), K = 128 (4 MMAs of K=32).
// Each TMEM lane then holds one key and its N (query, head) dot products, so the ReLU and the
// weighted head-sum are an in-thread reduction over TMEM columns and the [T, 64, S] tensor of
// per-head products never leaves the SM. The CTA keeps its NQ queries resident and streams
// 16 KB key tiles through a TMA ring (one warp), one thread issues the MMAs into a ring of TMEM
// accumulators (two of 256 columns with four queries, four of 64 with one), and the epilogue warps
// (four per TMEM lane quadrant with four queries, one query each)
// drain TMEM while the next tile multiplies; each thread keeps eight independent partial sums so the
// head-sum is not one serial FMA chain.
// Key tiles above the causal diagonal of the CTA's queries are never loaded.
#include <algorithm>

#include "common.cuh"
#include "kernels.h"

namespace dsa {

namespace {

constexpr int kKeysPerTile = 128;
constexpr int kTileBytes = kKeysPerTile * 128;      // 16 KB of e4m3 keys
// epilogue warps: 4 per TMEM lane quadrant with 4 queries per CTA (one query each), 1 with one query
constexpr int epi_warps(int nq) { return nq >= 4 ? 16 : 4; }
constexpr int threads_for(int nq) { return (epi_warps(nq) + 2) * 32; }   // + TMA warp + MMA warp

template <int NQ>
struct ScoresCfg {
  static constexpr int N = NQ * 64;                 // MMA N: (query, head) columns
  static constexpr int kStages = NQ >= 4 ? 6 : 4;
  static constexpr int kAcc = NQ >= 4 ? 2 : 4;      // TMEM accumulators (ring)
  static constexpr int kQBytes = N * 128;
  static constexpr int kTmemCols = kAcc * N;
  static constexpr int kSmemBytes = 1024 /*align slack*/ + kQBytes + kStages * kTileBytes + 1024;
};

struct ScoresParams {
  const float* q_scale;
  const float* w;
  const float* k_scale;
  const int32_t* q_pos;
  const int32_t* kv_len;
  float* scores;
  int64_t ld;
  int B, T, S_max;
  int groups;          // query groups per sequence = ceil(T / NQ)
  int ksplit;          // CTAs sharing one query group's key tiles
  int tiles_per_split;
  float wscale;        // 64^-0.5 * softmax_scale
  uint32_t flags;
  int* status;
  // paged K-cache (block_table == nullptr: dense [B][S_max] rows)
  const int32_t* block_table;   // [B][max_pages]
  int max_pages, page_size, page_shift;   // page_size = 1 << page_shift
  int64_t num_pages;
};

// Pool row of sequence b's logical position s in a paged K-cache, or -1 if its page id is out of
// range (S_max = max_pages * page_size bounds s).
__device__ __forceinline__ int64_t paged_row(const ScoresParams& p, int b, int s) {
  const int pg = __ldg(p.block_table + (int64_t)b * p.max_pages + (s >> p.page_shift));
  return (pg >= 0 && pg < p.num_pages) ? ((int64_t)pg << p.page_shift) + (s & (p.page_size - 1)) : -1;
}

}  // namespace

template <int NQ, bool PAGED>
__global__ void __launch_bounds__(threads_for(NQ), 1)
    index_scores_kernel(const __grid_constant__ CUtensorMap qmap,
                        const __grid_constant__ CUtensorMap kmap, const ScoresParams p) {
  using Cfg = ScoresCfg<NQ>;
  constexpr int N = Cfg::N;
  constexpr int STAGES = Cfg::kStages;
  constexpr int kEpiWarps = epi_warps(NQ);
  constexpr int kThreads = threads_for(NQ);

  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* q_smem = smem;                                   // [N rows][128 B], 128B swizzle
  uint8_t* k_smem = smem + Cfg::kQBytes;                    // STAGES x [128 rows][128 B]
  uint64_t* bars = reinterpret_cast<uint64_t*>(k_smem + STAGES * kTileBytes);
  uint64_t* full = bars;                                    // [STAGES] TMA -> MMA
  uint64_t* empty = bars + STAGES;                          // [STAGES] MMA -> TMA
  constexpr int kAcc = Cfg::kAcc;
  uint64_t* acc_full = bars + 2 * STAGES;                   // [kAcc]   MMA -> epilogue
  uint64_t* acc_empty = acc_full + kAcc;                    // [kAcc]   epilogue -> MMA
  uint64_t* q_full = acc_empty + kAcc;
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_flag;
  __shared__ __align__(16) float wq[NQ][64];
  __shared__ int nvalid[NQ];
  __shared__ int ntiles_sh;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // Heavy (late, long-context) query groups first so the causal tail is short.
  const int unit = blockIdx.x / p.ksplit;
  const int split = blockIdx.x - unit * p.ksplit;
  const int b = unit / p.groups;
  const int g = p.groups - 1 - (unit - b * p.groups);
  const int t0 = g * NQ;

  if (threadIdx.x == 0) {
    abort_flag = 0;
    for (int s = 0; s < STAGES; ++s) { mbar_init(&full[s], 1); mbar_init(&empty[s], 1); }
    for (int a = 0; a < kAcc; ++a) { mbar_init(&acc_full[a], 1); mbar_init(&acc_empty[a], kEpiWarps * 32); }
    mbar_init(q_full, 1);
    fence_barrier_init();
  }
  if (warp == kEpiWarps + 1) {           // MMA warp owns the TMEM allocation
    tmem_alloc(&tmem_base_sh, Cfg::kTmemCols);
    tmem_relinquish();
  }
  grid_dep_wait();                       // q_scale, w and the caches come from earlier kernels
  grid_dep_launch();
  for (int i = threadIdx.x; i < NQ * 64; i += kThreads) {   // folded head weights
    const int q = i >> 6, j = i & 63;
    const int t = t0 + q;
    float v = 0.f;
    if (t < p.T) {
      const int64_t o = ((int64_t)b * p.T + t) * 64 + j;
      v = __fmul_rn(__fmul_rn(p.w[o], p.q_scale[o]), p.wscale);
    }
    wq[q][j] = v;
  }
  if (threadIdx.x < NQ) {
    const int t = t0 + threadIdx.x;
    int n = 0;
    if (t < p.T) n = max(0, min(min(p.q_pos[(int64_t)b * p.T + t] + 1, p.kv_len[b]), p.S_max));
    nvalid[threadIdx.x] = n;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (threadIdx.x == 0) {
    int nmax = 0;
    for (int q = 0; q < NQ; ++q) nmax = max(nmax, nvalid[q]);
    ntiles_sh = (nmax + kKeysPerTile - 1) / kKeysPerTile;
  }
  __syncthreads();
  const uint32_t tmem_base = tmem_base_sh;
  const int kt_begin = split * p.tiles_per_split;
  const int kt_end = min(ntiles_sh, kt_begin + p.tiles_per_split);
  const int my_tiles = max(0, kt_end - kt_begin);

  if (warp == kEpiWarps) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0 && my_tiles > 0) {
      prefetch_tensormap(&qmap);
      prefetch_tensormap(&kmap);
      mbar_arrive_expect_tx(q_full, Cfg::kQBytes);
      tma_load_2d(q_smem, &qmap, q_full, 0, (b * p.T + t0) * 64);
      // paged: each tile is two 64-row boxes from their pages (looked up one tile ahead); a half
      // past S_max or on an invalid page loads from an out-of-range row, i.e. zeros
      auto half_rows = [&](int i, int32_t (&r)[2]) {
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          const int ks0 = (kt_begin + i) * kKeysPerTile + 64 * hh;
          int64_t row = -1;
          if (i < my_tiles && ks0 < p.S_max) row = paged_row(p, b, ks0);
          r[hh] = row >= 0 ? (int32_t)row : (int32_t)(p.num_pages * p.page_size);
        }
      };
      int32_t rows_next[2] = {0, 0};
      if (PAGED) half_rows(0, rows_next);
      for (int i = 0; i < my_tiles; ++i) {
        const int s = i % STAGES;
        int32_t rows[2] = {rows_next[0], rows_next[1]};
        if (PAGED) half_rows(i + 1, rows_next);
        if (i >= STAGES && !mbar_wait(&empty[s], ((i / STAGES) + 1) & 1, &abort_flag, p.status, DSA_SITE_SCORES_K_EMPTY)) break;
        mbar_arrive_expect_tx(&full[s], kTileBytes);
        if (PAGED) {
          tma_load_2d(k_smem + s * kTileBytes, &kmap, &full[s], 0, rows[0]);
          tma_load_2d(k_smem + s * kTileBytes + kTileBytes / 2, &kmap, &full[s], 0, rows[1]);
        } else {
          tma_load_2d(k_smem + s * kTileBytes, &kmap, &full[s], 0, b * p.S_max + (kt_begin + i) * kKeysPerTile);
        }
      }
    }
  } else if (warp == kEpiWarps + 1) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0 && my_tiles > 0) {
      constexpr uint32_t idesc = idesc_f32acc(0 /*E4M3*/, 0 /*E4M3*/, 128, N, 0, 0);
      const uint32_t q_addr = smem_u32(q_smem);
      bool ok = mbar_wait(q_full, 0, &abort_flag, p.status, DSA_SITE_SCORES_Q);
      for (int i = 0; ok && i < my_tiles; ++i) {
        const int s = i % STAGES, a = i % kAcc;
        if (i >= kAcc && !mbar_wait(&acc_empty[a], ((i / kAcc) + 1) & 1, &abort_flag, p.status, DSA_SITE_SCORES_ACC_EMPTY)) break;
        if (!mbar_wait(&full[s], (i / STAGES) & 1, &abort_flag, p.status, DSA_SITE_SCORES_K_FULL)) break;
        tc_fence_after();
        const uint32_t k_addr = smem_u32(k_smem + s * kTileBytes);
        const uint32_t d_tmem = tmem_base + a * N;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          mma_f8f6f4_ss(d_tmem, sdesc_kmajor_sw128(k_addr + kk * 32), sdesc_kmajor_sw128(q_addr + kk * 32),
                        idesc, kk > 0 ? 1u : 0u);
        }
        mma_commit(&empty[s]);       // the K stage may be refilled once these MMAs have read it
        mma_commit(&acc_full[a]);    // accumulator a is ready for the epilogue
      }
    }
  } else {
    // ------------------------------------------------------------------ epilogue (warps 0-15)
    // warp w reads TMEM lane quadrant w % 4 (one key per thread) for query w / 4
    const int quad = warp & 3;
    constexpr int QPW = 1;                             // queries per epilogue warp
    const int q_lo = warp >> 2;
    const bool active = q_lo < NQ;                     // NQ = 1: one warp per quadrant
    const int row_in_tile = quad * 32 + lane;          // TMEM lane = key within the tile
    const float* ks_row = p.k_scale + (int64_t)b * p.S_max;
    // k_scale of this thread's key in tile i, one tile ahead; paged: its page id two tiles ahead
    // (-2: no key in that tile) and the scale one tile ahead (-1: the page is outside the pool)
    auto tile_key = [&](int i) { return (kt_begin + i) * kKeysPerTile + row_in_tile; };
    auto has_key = [&](int i) { return active && i < my_tiles && tile_key(i) < p.S_max; };
    auto load_pg = [&](int i) -> int {
      return has_key(i) ? __ldg(p.block_table + (int64_t)b * p.max_pages + (tile_key(i) >> p.page_shift)) : -2;
    };
    auto load_ks = [&](int i, int pg) -> float {
      if (!PAGED) return has_key(i) ? __ldg(ks_row + tile_key(i)) : 0.f;
      if (pg == -2) return 0.f;
      if (pg < 0 || pg >= p.num_pages) return -1.f;
      return __ldg(p.k_scale + ((int64_t)pg << p.page_shift) + (tile_key(i) & (p.page_size - 1)));
    };
    int pg_next = PAGED ? load_pg(1) : 0;
    float ks_next = load_ks(0, PAGED ? load_pg(0) : 0);
    for (int i = 0; i < my_tiles; ++i) {
      const int a = i % kAcc;
      const float ks = ks_next;
      ks_next = load_ks(i + 1, pg_next);               // one tile ahead
      if (PAGED) pg_next = load_pg(i + 2);             // two tiles ahead
      if (!__all_sync(0xffffffffu, mbar_wait(&acc_full[a], (i / kAcc) & 1, &abort_flag, p.status, DSA_SITE_SCORES_ACC_FULL))) break;
      tc_fence_after();
      if (active) {
        const int key = (kt_begin + i) * kKeysPerTile + row_in_tile;
#pragma unroll
        for (int qq = 0; qq < QPW; ++qq) {
          const int q = q_lo + qq;
          uint32_t r0[32], r1[32];
          const uint32_t taddr = tmem_base + ((uint32_t)(quad * 32) << 16) + a * N + q * 64;
          tmem_ld32(taddr, r0);
          tmem_ld32(taddr + 32, r1);
          tmem_ld_wait();
          // eight partial sums, as four packed pairs: head j accumulates into sum j mod 8 with one
          // lane of a paired fma.rn.f32x2 (each lane rounds exactly as fmaf)
          uint64_t acc2[4] = {0ull, 0ull, 0ull, 0ull};
          const float4* w4 = reinterpret_cast<const float4*>(&wq[q][0]);
#pragma unroll
          for (int jj = 0; jj < 8; ++jj) {
            const float4 wa = w4[2 * jj], wb = w4[2 * jj + 1];
            const float ww[8] = {wa.x, wa.y, wa.z, wa.w, wb.x, wb.y, wb.z, wb.w};
#pragma unroll
            for (int u = 0; u < 8; u += 2) {
              const int j = 8 * jj + u;
              const float v0 = fmaxf(__uint_as_float(j < 32 ? r0[j] : r1[j - 32]), 0.f);
              const float v1 = fmaxf(__uint_as_float(j + 1 < 32 ? r0[j + 1] : r1[j + 1 - 32]), 0.f);
              acc2[u / 2] = fma_f32x2(ww[u], ww[u + 1], v0, v1, acc2[u / 2]);
            }
          }
          float acc[8];
#pragma unroll
          for (int u = 0; u < 4; ++u) unpack_f32x2(acc2[u], acc[2 * u], acc[2 * u + 1]);
          const float tot = ((acc[0] + acc[1]) + (acc[2] + acc[3])) + ((acc[4] + acc[5]) + (acc[6] + acc[7]));
          const int t = t0 + q;
          if (t < p.T) {
            float* dst = p.scores + ((int64_t)b * p.T + t) * p.ld;
            if (key < nvalid[q]) {
              if (!PAGED || ks >= 0.f) dst[key] = tot * ks;
              else set_status(p.status, DSA_ERR_DEVICE_BOUNDS);   // visible key on an invalid page
            }
            else if ((p.flags & DSA_FILL_MASKED) && key < p.S_max) dst[key] = -INFINITY;
          }
        }
      }
      tc_fence_before();
      mbar_arrive(&acc_empty[a]);
    }
    if ((p.flags & DSA_FILL_MASKED) && warp < 4) {   // tiles of this split above the causal limit
      const int kt_stop = min((p.S_max + kKeysPerTile - 1) / kKeysPerTile, kt_begin + p.tiles_per_split);
      for (int kt = max(kt_begin, kt_end); kt < kt_stop; ++kt) {
        const int key = kt * kKeysPerTile + row_in_tile;
        if (key >= p.S_max) continue;
        for (int q = 0; q < NQ; ++q) {
          const int t = t0 + q;
          if (t < p.T) p.scores[((int64_t)b * p.T + t) * p.ld + key] = -INFINITY;
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kEpiWarps + 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, Cfg::kTmemCols);
  }
}

template <int NQ, bool PAGED>
static int launch_scores_nq(const uint8_t* q8, const uint8_t* k8, const ScoresParams& base,
                            cudaStream_t stream) {
  using Cfg = ScoresCfg<NQ>;
  CUtensorMap qmap, kmap;
  if (!dsa_host::encode_tensor_map_2d(&qmap, CU_TENSOR_MAP_DATA_TYPE_UINT8, (void*)q8, 128,
                                      (uint64_t)base.B * base.T * 64, 128, 128, NQ * 64,
                                      CU_TENSOR_MAP_SWIZZLE_128B) ||
      !dsa_host::encode_tensor_map_2d(&kmap, CU_TENSOR_MAP_DATA_TYPE_UINT8, (void*)k8, 128,
                                      base.block_table ? (uint64_t)base.num_pages * base.page_size
                                                       : (uint64_t)base.B * base.S_max,
                                      128, 128, base.block_table ? kKeysPerTile / 2 : kKeysPerTile,
                                      CU_TENSOR_MAP_SWIZZLE_128B))
    return DSA_ERR_CUDA;
  ScoresParams p = base;
  p.groups = (base.T + NQ - 1) / NQ;
  const int tiles_max = (base.S_max + kKeysPerTile - 1) / kKeysPerTile;
  const int64_t units = (int64_t)base.B * p.groups;
  // one wave: as many CTAs as fit on the device at once (key splits share a query group's tiles)
  static uint64_t configured[dsa_host::kMaxSetupDevices] = {};
  static int occupancy[dsa_host::kMaxSetupDevices] = {};
  int dev = 0;
  if (dsa_host::needs_setup(configured, &dev) && dev < dsa_host::kMaxSetupDevices) {
    // all of the unified L1 / shared storage as shared memory, so that as many CTAs as the shared
    // memory allows are resident
    if (cudaFuncSetAttribute(index_scores_kernel<NQ, PAGED>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             Cfg::kSmemBytes) != cudaSuccess ||
        cudaFuncSetAttribute(index_scores_kernel<NQ, PAGED>, cudaFuncAttributePreferredSharedMemoryCarveout,
                             cudaSharedmemCarveoutMaxShared) != cudaSuccess)
      return DSA_ERR_CUDA;
    const int per_sm = dsa_host::resident_ctas_per_sm((const void*)index_scores_kernel<NQ, PAGED>, threads_for(NQ),
                                                      Cfg::kSmemBytes, Cfg::kTmemCols);
    if (per_sm < 1) return DSA_ERR_CUDA;
    occupancy[dev] = per_sm;
    dsa_host::mark_setup(configured);
  }
  const int64_t target =
      (int64_t)(dev < dsa_host::kMaxSetupDevices ? std::max(1, occupancy[dev]) : 1) * dsa_host::device_sm_count();
  int ksplit = (int)std::max<int64_t>(1, target / units);
  ksplit = max(1, min(ksplit, tiles_max));
  p.ksplit = ksplit;
  p.tiles_per_split = (tiles_max + ksplit - 1) / ksplit;
  p.ksplit = (tiles_max + p.tiles_per_split - 1) / p.tiles_per_split;
  const int64_t grid = units * p.ksplit;
  if (grid > 0x7fffffff) return DSA_ERR_INVALID_ARG;
  if (dev >= dsa_host::kMaxSetupDevices && cudaFuncSetAttribute(index_scores_kernel<NQ, PAGED>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        Cfg::kSmemBytes) != cudaSuccess)
    return DSA_ERR_CUDA;
  return dsa_host::launch(index_scores_kernel<NQ, PAGED>, dim3((unsigned)grid), dim3(threads_for(NQ)),
                          Cfg::kSmemBytes, stream, qmap, kmap, p);
}

int launch_index_scores(const uint8_t* q8, const float* q_scale, const float* w, const uint8_t* k8,
                        const float* k_scale, const int32_t* q_pos, const int32_t* kv_len, int B,
                        int T, int S_max, float softmax_scale, float* scores, int64_t ld,
                        uint32_t flags, cudaStream_t stream, int* status) {
  ScoresParams p{};
  p.q_scale = q_scale; p.w = w; p.k_scale = k_scale; p.q_pos = q_pos; p.kv_len = kv_len;
  p.scores = scores; p.ld = ld; p.B = B; p.T = T; p.S_max = S_max;
  p.wscale = 0.125f * softmax_scale;   // 64^-0.5 (n_heads**-0.5 in Indexer.forward)
  p.flags = flags; p.status = status;
  if (T >= 4) return launch_scores_nq<4, false>(q8, k8, p, stream);
  return launch_scores_nq<1, false>(q8, k8, p, stream);
}

int launch_index_scores_paged(const uint8_t* q8, const float* q_scale, const float* w, const uint8_t* k8_pool,
                              const float* k_scale_pool, int64_t num_pages, const int32_t* block_table,
                              int max_pages, int page_size, const int32_t* q_pos, const int32_t* kv_len, int B,
                              int T, float softmax_scale, float* scores, int64_t ld, uint32_t flags,
                              cudaStream_t stream, int* status) {
  ScoresParams p{};
  p.q_scale = q_scale; p.w = w; p.k_scale = k_scale_pool; p.q_pos = q_pos; p.kv_len = kv_len;
  p.scores = scores; p.ld = ld; p.B = B; p.T = T; p.S_max = max_pages * page_size;
  p.wscale = 0.125f * softmax_scale;
  p.flags = flags; p.status = status;
  p.block_table = block_table; p.max_pages = max_pages; p.page_size = page_size; p.num_pages = num_pages;
  p.page_shift = __builtin_ctz((unsigned)page_size);
  if (T >= 4) return launch_scores_nq<4, true>(q8, k8_pool, p, stream);
  return launch_scores_nq<1, true>(q8, k8_pool, p, stream);
}

}  // namespace dsa
