// dsa_index_topk: the decode indexer's scores and their top-k in one launch; the scores never
// leave the SMs.
//
// Computes, per query row, the same selection as dsa_index_scores followed by dsa_topk (the
// fp8_index call, the causal mask and topk(min(index_topk, end_pos)) of Indexer.forward, "DeepSeek-
// V3.2-Exp - Rotate first features"; S^I and top_2048 of the lightning-indexer steps on the dense-
// block page), with the scores in fp32 bit for bit as dsa_index_scores makes them.
//
// A row's key tiles are split over a thread-block cluster of C CTAs (C = 1..8, CTA r taking tiles
// [r * tps, r * tps + tps)). Each CTA scores its tiles exactly as the index-scores kernel does
// (TMA ring of 128-key FP8 tiles, tcgen05 kind::f8f6f4 into TMEM, ReLU-weighted head sum in the
// epilogue) but keeps each score, as an order-preserving key, in shared memory. Then the cluster
// runs the radix select of the top-k kernel on the row spread over its CTAs: each CTA builds the
// histogram of its own keys (partial radix histograms per CTA), adds its non-zero bins into every
// CTA's copy of the row's histogram with distributed-shared-memory reductions, and after a cluster
// barrier every CTA picks the same digit. Digits 1 and 2 (bits 31..21, 20..10) always run; a third
// (bits 9..0) only when several keys share the k-th key's first 22 bits and it is not the smallest
// of them. A last exchange of per-CTA counts orders the selection by position across the cluster.
#include <algorithm>

#include "common.cuh"
#include "kernels.h"

namespace dsa {

namespace {

constexpr int kTile = 128;                          // keys per tile (MMA M)
constexpr int kTileBytes = kTile * 128;             // 16 KB of e4m3 keys
constexpr int kN = 64;                              // MMA N: the query's 64 heads
constexpr int kStages = 4, kAcc = 4;
constexpr int kEpiWarps = 4, kTmaWarp = 4, kMmaWarp = 5;
constexpr int kThreads = 192;                       // 4 epilogue warps + TMA warp + MMA warp
constexpr int kWarps = kThreads / 32;
constexpr int kQBytes = kN * 128;                   // 8 KB: the query's e4m3 head rows
constexpr int kTmemCols = kAcc * kN;
constexpr int kMaxTps = 32;                         // tiles per CTA (the keys of one CTA: 4096)
constexpr int kRegionWords = kMaxTps * kTile / 32 * 36;   // transposed keys: position p at p + 4 (p / 32)
// after the scores the stage ring holds the select's working set (words)
constexpr int kH1 = 0, kS1 = 2048, kH2 = 4096, kS2 = 6144, kH3 = 8192, kS3 = 9216, kStage = 10240;
static_assert((kStage + kMaxTps * kTile) * 4 <= kStages * kTileBytes, "select working set fits in the ring");
constexpr int kOffQ = 0, kOffRing = kQBytes, kOffRegion = kOffRing + kStages * kTileBytes;
constexpr int kOffBar = kOffRegion + kRegionWords * 4;
constexpr int kSmemBytes = 1024 + kOffBar + 256;

struct IndexTopkParams {
  const float* q_scale;
  const float* w;
  const float* k_scale;
  const int32_t* q_pos;
  const int32_t* kv_len;
  int32_t* idx;
  int B, T, S_max, k;
  int C;                // CTAs per row (the cluster)
  int tps;              // key tiles per CTA
  float wscale;         // 64^-0.5 * softmax_scale
  int* status;
};

__device__ __forceinline__ uint32_t order_key_f(float f) {
  uint32_t u = __float_as_uint(f);
  if ((u << 1) == 0) u = 0;                       // -0 and +0 compare equal
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ void red_add_if(uint32_t* hist, uint32_t bin, bool pred) {
  asm volatile("{\n\t.reg .pred p;\n\tsetp.ne.u32 p, %1, 0;\n\t@p red.shared.add.u32 [%0], 1;\n\t}" ::"r"(
                   smem_u32(hist + bin)),
               "r"((uint32_t)pred)
               : "memory");
}

// += v on the word at shared::cluster address `a` (another CTA's shared memory, or this one's)
__device__ __forceinline__ void red_cluster_add(uint32_t a, uint32_t v) {
  asm volatile("red.shared::cluster.add.u32 [%0], %1;" ::"r"(a), "r"(v) : "memory");
}
__device__ __forceinline__ void st_cluster(uint32_t a, uint32_t v) {
  asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(a), "r"(v) : "memory");
}
__device__ __forceinline__ uint32_t ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ uint32_t mapa_rank(uint32_t a, uint32_t r) {
  uint32_t o;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(o) : "r"(a), "r"(r));
  return o;
}
__device__ __forceinline__ void cluster_barrier() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// Exclusive prefix, in thread order, of one value per thread of the CTA; *total gets the sum. One
// barrier; `tot` (kWarps words) must not be reused before another barrier.
__device__ __forceinline__ uint32_t cta_excl_scan(uint32_t v, uint32_t* tot, uint32_t* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t incl = v;
#pragma unroll
  for (int d = 1; d < 32; d <<= 1) {
    const uint32_t o = __shfl_up_sync(0xffffffffu, incl, d);
    if (lane >= d) incl += o;
  }
  if (lane == 31) tot[warp] = incl;
  __syncthreads();
  const uint32_t wt = lane < kWarps ? tot[lane] : 0u;
  uint32_t ws = wt;
#pragma unroll
  for (int d = 1; d < kWarps; d <<= 1) {
    const uint32_t o = __shfl_up_sync(0xffffffffu, ws, d);
    if (lane >= d) ws += o;
  }
  const uint32_t warp_before = __shfl_sync(0xffffffffu, ws - wt, warp);
  *total = __shfl_sync(0xffffffffu, ws, kWarps - 1);
  return warp_before + incl - v;
}

// The bin of the row histogram `hist` (NB bins) holding the target-th largest key: sel[0] = bin,
// sel[1] = the target's rank inside it (1-based), sel[2] = the bin's count. Ends with a barrier.
template <int NB>
__device__ __forceinline__ void pick_bin(const uint32_t* hist, uint32_t target, uint32_t* tot, uint32_t* sel) {
  constexpr int C = (NB + kThreads - 1) / kThreads;
  const int top = NB - 1 - (int)threadIdx.x * C;   // this thread's bins: top, top - 1, ..., top - C + 1
  uint32_t h[C];
  uint32_t local = 0;
#pragma unroll
  for (int j = 0; j < C; ++j) {
    h[j] = top - j >= 0 ? hist[top - j] : 0u;
    local += h[j];
  }
  uint32_t total;
  uint32_t before = cta_excl_scan(local, tot, &total);
  if (before < target && target <= before + local) {
#pragma unroll
    for (int j = 0; j < C; ++j) {
      if (before + h[j] >= target) {
        sel[0] = (uint32_t)(top - j);
        sel[1] = target - before;
        sel[2] = h[j];
        break;
      }
      before += h[j];
    }
  }
  __syncthreads();
}

// Adds this CTA's histogram `h` (NB bins, local) into the row histogram `s` of every CTA of the
// cluster (non-zero bins only), then waits for the whole cluster: `s` is then the row's histogram.
template <int NB>
__device__ __forceinline__ void merge_hist(const uint32_t* h, uint32_t* s, int C) {
  __syncthreads();
  const uint32_t s_addr = smem_u32(s);
  for (int b = threadIdx.x; b < NB; b += kThreads) {
    const uint32_t v = h[b];
    if (v == 0u) continue;
    for (int r = 0; r < C; ++r) red_cluster_add(mapa_rank(s_addr + 4u * b, (uint32_t)r), v);
  }
  cluster_barrier();
}

// A launch of `kernel` as a grid of thread-block clusters of `cluster_x` CTAs along x, with
// programmatic stream serialization like every other launch of the library.
template <typename... KArgs, typename... Args>
int launch_clusters(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream, int cluster_x,
                    Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = (unsigned)cluster_x;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...) == cudaSuccess ? DSA_OK : DSA_ERR_CUDA;
}

}  // namespace

template <int KPT>
__global__ void __launch_bounds__(kThreads, 2)
    index_topk_kernel(const __grid_constant__ CUtensorMap qmap, const __grid_constant__ CUtensorMap kmap,
                      const IndexTopkParams p) {
  static_assert(KPT % 4 == 0 && KPT <= kMaxTps, "keys per thread");
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* q_smem = smem + kOffQ;
  uint8_t* k_smem = smem + kOffRing;
  uint32_t* ring = reinterpret_cast<uint32_t*>(k_smem);   // the select's working set, after the scores
  uint32_t* region = reinterpret_cast<uint32_t*>(smem + kOffRegion);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kOffBar);
  uint64_t* full = bars;                            // [kStages] TMA -> MMA
  uint64_t* empty = bars + kStages;                 // [kStages] MMA -> TMA
  uint64_t* acc_full = bars + 2 * kStages;          // [kAcc]    MMA -> epilogue
  uint64_t* acc_empty = acc_full + kAcc;            // [kAcc]    epilogue -> MMA
  uint64_t* q_full = acc_empty + kAcc;
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_flag;
  __shared__ __align__(16) float wq[64];
  __shared__ int nvalid_sh;
  __shared__ uint32_t tots[5][kWarps];
  __shared__ uint32_t sel[3];
  __shared__ uint32_t cnt[8][2];                    // per CTA of the cluster: (above, equal) counts

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, tid = threadIdx.x;
  const int C = p.C;
  const int rank = (int)ctarank();
  const int64_t row = blockIdx.x / C;               // (b, t)
  const int b = (int)(row / p.T);
  const int kt_begin = rank * p.tps;

  if (tid == 0) {
    abort_flag = 0;
    for (int s = 0; s < kStages; ++s) { mbar_init(&full[s], 1); mbar_init(&empty[s], 1); }
    for (int a = 0; a < kAcc; ++a) { mbar_init(&acc_full[a], 1); mbar_init(&acc_empty[a], kEpiWarps * 32); }
    mbar_init(q_full, 1);
    fence_barrier_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(&tmem_base_sh, kTmemCols);
    tmem_relinquish();
  }
  grid_dep_wait();                                  // q_scale, w and the caches come from earlier kernels
  grid_dep_launch();
  for (int j = tid; j < 64; j += kThreads) {        // folded head weights
    const int64_t o = row * 64 + j;
    wq[j] = __fmul_rn(__fmul_rn(p.w[o], p.q_scale[o]), p.wscale);
  }
  if (tid == 0) nvalid_sh = max(0, min(min(p.q_pos[row] + 1, p.kv_len[b]), p.S_max));
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = tmem_base_sh;
  const int n = nvalid_sh;                          // visible keys of the row
  const int ntiles = (n + kTile - 1) / kTile;
  const int kt_end = min(ntiles, kt_begin + p.tps);
  const int my_tiles = max(0, kt_end - kt_begin);
  const int n_loc = max(0, min(n - kt_begin * kTile, my_tiles * kTile));   // this CTA's visible keys

  if (warp == kTmaWarp) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0 && my_tiles > 0) {
      prefetch_tensormap(&qmap);
      prefetch_tensormap(&kmap);
      mbar_arrive_expect_tx(q_full, kQBytes);
      tma_load_2d(q_smem, &qmap, q_full, 0, (int32_t)(row * 64));
      for (int i = 0; i < my_tiles; ++i) {
        const int s = i % kStages;
        if (i >= kStages && !mbar_wait(&empty[s], ((i / kStages) + 1) & 1, &abort_flag, p.status,
                                       DSA_SITE_SCORES_K_EMPTY))
          break;
        mbar_arrive_expect_tx(&full[s], kTileBytes);
        tma_load_2d(k_smem + s * kTileBytes, &kmap, &full[s], 0, b * p.S_max + (kt_begin + i) * kTile);
      }
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0 && my_tiles > 0) {
      constexpr uint32_t idesc = idesc_f32acc(0 /*E4M3*/, 0 /*E4M3*/, 128, kN, 0, 0);
      const uint32_t q_addr = smem_u32(q_smem);
      bool ok = mbar_wait(q_full, 0, &abort_flag, p.status, DSA_SITE_SCORES_Q);
      for (int i = 0; ok && i < my_tiles; ++i) {
        const int s = i % kStages, a = i % kAcc;
        if (i >= kAcc && !mbar_wait(&acc_empty[a], ((i / kAcc) + 1) & 1, &abort_flag, p.status,
                                    DSA_SITE_SCORES_ACC_EMPTY))
          break;
        if (!mbar_wait(&full[s], (i / kStages) & 1, &abort_flag, p.status, DSA_SITE_SCORES_K_FULL)) break;
        tc_fence_after();
        const uint32_t k_addr = smem_u32(k_smem + s * kTileBytes);
        const uint32_t d_tmem = tmem_base + a * kN;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_f8f6f4_ss(d_tmem, sdesc_kmajor_sw128(k_addr + kk * 32), sdesc_kmajor_sw128(q_addr + kk * 32), idesc,
                        kk > 0 ? 1u : 0u);
        mma_commit(&empty[s]);
        mma_commit(&acc_full[a]);
      }
    }
  } else {
    // ------------------------------------------------------------------ epilogue (warps 0-3)
    // warp w reads TMEM lane quadrant w: thread = key within the tile. Each score goes to this
    // CTA's transposed key array at local position 128 i + row_in_tile.
    const int row_in_tile = warp * 32 + lane;
    const float* ks_row = p.k_scale + (int64_t)b * p.S_max;
    auto key_of = [&](int i) { return (kt_begin + i) * kTile + row_in_tile; };
    float ks_next = my_tiles > 0 && key_of(0) < p.S_max ? __ldg(ks_row + key_of(0)) : 0.f;
    for (int i = 0; i < my_tiles; ++i) {
      const int a = i % kAcc;
      const float ks = ks_next;
      ks_next = (i + 1 < my_tiles && key_of(i + 1) < p.S_max) ? __ldg(ks_row + key_of(i + 1)) : 0.f;
      if (!__all_sync(0xffffffffu, mbar_wait(&acc_full[a], (i / kAcc) & 1, &abort_flag, p.status,
                                             DSA_SITE_SCORES_ACC_FULL)))
        break;
      tc_fence_after();
      uint32_t r0[32], r1[32];
      const uint32_t taddr = tmem_base + ((uint32_t)(warp * 32) << 16) + a * kN;
      tmem_ld32(taddr, r0);
      tmem_ld32(taddr + 32, r1);
      tmem_ld_wait();
      // the head sum exactly as the index-scores kernel forms it (eight partial sums in packed pairs)
      uint64_t acc2[4] = {0ull, 0ull, 0ull, 0ull};
      const float4* w4 = reinterpret_cast<const float4*>(wq);
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
      const int pos = i * kTile + row_in_tile;      // local position
      region[pos + 4 * (pos >> 5)] = order_key_f(tot * ks);
      tc_fence_before();
      mbar_arrive(&acc_empty[a]);
    }
  }

  // ---------------------------------------------------------------- the row's selection
  tc_fence_before();
  __syncthreads();                                  // every score is in `region`; the ring is free
  int32_t* out = p.idx + row * (int64_t)p.k;
  const int k = p.k;
  // Every CTA of the cluster takes the same branches below and the same cluster barriers (the
  // conditions are the row's, identical in all of them), also after a bounded wait gave up: a
  // barrier.cluster has no time limit. The status word then says that the selection is void.
  if (n <= k) {                                     // everything visible is selected
    for (int i = tid; i < p.tps * kTile; i += kThreads) {
      const int pos = kt_begin * kTile + i;
      if (pos < n) out[pos] = pos;
    }
    if (rank == 0)
      for (int i = n + tid; i < k; i += kThreads) out[i] = -1;
  } else {
    uint32_t* h1 = ring + kH1;
    uint32_t* s1 = ring + kS1;
    uint32_t* h2 = ring + kH2;
    uint32_t* s2 = ring + kS2;
    uint32_t* h3 = ring + kH3;
    uint32_t* s3 = ring + kS3;
    int32_t* stage = reinterpret_cast<int32_t*>(ring + kStage);
    for (int i = tid; i < kStage; i += kThreads) ring[i] = 0u;
    // thread t owns local positions [t KPT, t KPT + KPT): its keys, read from the transposed array
    const int p0 = tid * KPT;
    const int nv = max(0, min(KPT, n_loc - p0));
    uint32_t key[KPT];
#pragma unroll
    for (int c = 0; c < KPT / 4; ++c) {
      uint4 kk = make_uint4(0u, 0u, 0u, 0u);
      const int pc = p0 + 4 * c;
      if (4 * c < nv) kk = *reinterpret_cast<const uint4*>(region + pc + 4 * (pc >> 5));
      key[4 * c] = kk.x;
      key[4 * c + 1] = kk.y;
      key[4 * c + 2] = kk.z;
      key[4 * c + 3] = kk.w;
    }
    const uint32_t valid = nv >= 32 ? 0xffffffffu : ((1u << nv) - 1u);
    __syncthreads();
    cluster_barrier();                              // every CTA's row histograms are zero
    // digit 1 (bits 31..21) over this CTA's keys, then over the row
#pragma unroll
    for (int i = 0; i < KPT; ++i) red_add_if(h1, key[i] >> 21, i < nv);
    merge_hist<2048>(h1, s1, C);
    pick_bin<2048>(s1, (uint32_t)k, tots[0], sel);
    const uint32_t d1 = sel[0];
    uint32_t rem = sel[1];
    uint32_t m_gt = 0, m_on = 0;
#pragma unroll
    for (int i = 0; i < KPT; ++i) {
      const uint32_t dg = key[i] >> 21;
      m_gt |= (uint32_t)(dg > d1) << i;
      m_on |= (uint32_t)(dg == d1) << i;
    }
    m_gt &= valid;
    m_on &= valid;
    // digit 2 (bits 20..10) over the keys on digit 1
#pragma unroll
    for (int i = 0; i < KPT; ++i) red_add_if(h2, (key[i] >> 10) & 2047u, (m_on >> i) & 1u);
    merge_hist<2048>(h2, s2, C);
    pick_bin<2048>(s2, rem, tots[1], sel);
    const uint32_t pre22 = (d1 << 11) | sel[0];
    rem = sel[1];
    const uint32_t n_on = sel[2];
    {
      uint32_t m2 = 0;
#pragma unroll
      for (int i = 0; i < KPT; ++i) {
        const uint32_t pfx = key[i] >> 10;
        m_gt |= (uint32_t)(((m_on >> i) & 1u) && pfx > pre22) << i;
        m2 |= (uint32_t)(((m_on >> i) & 1u) && pfx == pre22) << i;
      }
      m_on = m2;
    }
    uint32_t m_eq = 0, need_eq = 0;
    if (rem == n_on) {
      m_gt |= m_on;                                 // the k-th key is the smallest on its 22-bit prefix
    } else {
      // digit 3 (bits 9..0) over the keys on the first 22 bits
#pragma unroll
      for (int i = 0; i < KPT; ++i) red_add_if(h3, key[i] & 1023u, (m_on >> i) & 1u);
      merge_hist<1024>(h3, s3, C);
      pick_bin<1024>(s3, rem, tots[2], sel);
      const uint32_t thr = (pre22 << 10) | sel[0];
      need_eq = sel[1];                             // keys equal to the k-th that are selected
#pragma unroll
      for (int i = 0; i < KPT; ++i) {
        m_gt |= (uint32_t)(((m_on >> i) & 1u) && key[i] > thr) << i;
        m_eq |= (uint32_t)(((m_on >> i) & 1u) && key[i] == thr) << i;
      }
    }
    // position order: within the CTA by thread, across the cluster by rank
    uint32_t total;
    const uint32_t before = cta_excl_scan(((uint32_t)__popc(m_gt) << 16) | (uint32_t)__popc(m_eq), tots[3], &total);
    if (tid < C) {                                  // this CTA's counts, into every CTA's table
      const uint32_t a = smem_u32(&cnt[rank][0]);
      st_cluster(mapa_rank(a, (uint32_t)tid), total >> 16);
      st_cluster(mapa_rank(a + 4u, (uint32_t)tid), total & 0xFFFFu);
    }
    cluster_barrier();
    uint32_t g_pre = 0, e_pre = 0;
    for (int r = 0; r < rank; ++r) {
      g_pre += cnt[r][0];
      e_pre += cnt[r][1];
    }
    const uint32_t e_here = total & 0xFFFFu;
    const uint32_t need_here = min(e_here, need_eq > e_pre ? need_eq - e_pre : 0u);
    const uint32_t base = g_pre + min(e_pre, need_eq);   // selected keys before this CTA's
    const uint32_t gb = before >> 16, eb = before & 0xFFFFu;
    uint32_t m_sel = m_gt;
    {
      uint32_t m = m_eq;
      for (uint32_t r = eb; m && r < need_here; ++r) {
        m_sel |= m & (0u - m);
        m &= m - 1u;
      }
    }
    const uint32_t out_here = (total >> 16) + need_here;   // this CTA's selected keys
    uint32_t r = gb + min(eb, need_here);
    for (uint32_t m = m_sel; m; m &= m - 1u) stage[r++] = kt_begin * kTile + p0 + __ffs(m) - 1;
    __syncthreads();
    for (uint32_t i = tid; i < out_here; i += kThreads) out[base + i] = stage[i];
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

int launch_index_topk(const uint8_t* q8, const float* q_scale, const float* w, const uint8_t* k8,
                      const float* k_scale, const int32_t* q_pos, const int32_t* kv_len, int B, int T,
                      int S_max, float softmax_scale, int k, int32_t* idx, cudaStream_t stream, int* status) {
  const int64_t units = (int64_t)B * T;
  const int tiles_max = (S_max + kTile - 1) / kTile;
  if (tiles_max > 8 * kMaxTps) return DSA_ERR_INVALID_ARG;
  IndexTopkParams p{};
  p.q_scale = q_scale; p.w = w; p.k_scale = k_scale; p.q_pos = q_pos; p.kv_len = kv_len; p.idx = idx;
  p.B = B; p.T = T; p.S_max = S_max; p.k = k;
  p.wscale = 0.125f * softmax_scale;                // 64^-0.5 (n_heads**-0.5 in Indexer.forward)
  p.status = status;
  // CTAs per row: enough that a CTA holds at most kMaxTps tiles, and as many more (powers of two, at
  // most 8) as still fill one wave of resident CTAs
  static uint64_t configured[dsa_host::kMaxSetupDevices] = {};
  static int occupancy[dsa_host::kMaxSetupDevices] = {};
  int dev = 0;
  const bool fresh = dsa_host::needs_setup(configured, &dev);
  const bool tracked = dev >= 0 && dev < dsa_host::kMaxSetupDevices;
  int per_sm = tracked ? occupancy[dev] : 0;
  if (fresh || !tracked) {
    // all of the unified L1 / shared storage as shared memory: two CTAs per SM
    const void* fns[] = {(const void*)index_topk_kernel<8>, (const void*)index_topk_kernel<16>,
                         (const void*)index_topk_kernel<32>};
    for (const void* f : fns)
      if (cudaFuncSetAttribute(f, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes) != cudaSuccess ||
          cudaFuncSetAttribute(f, cudaFuncAttributePreferredSharedMemoryCarveout, cudaSharedmemCarveoutMaxShared) !=
              cudaSuccess)
        return DSA_ERR_CUDA;
    per_sm = dsa_host::resident_ctas_per_sm((const void*)index_topk_kernel<32>, kThreads, kSmemBytes, kTmemCols);
    if (per_sm < 1) return DSA_ERR_CUDA;
    if (tracked) {
      occupancy[dev] = per_sm;
      dsa_host::mark_setup(configured);
    }
  }
  const int64_t slots = (int64_t)std::max(1, per_sm) * dsa_host::device_sm_count();
  int C = 1;
  while ((C * kMaxTps) < tiles_max) C *= 2;
  while (C < 8 && units * (2 * C) <= slots) C *= 2;
  p.C = C;
  p.tps = (tiles_max + C - 1) / C;
  const int64_t grid = units * C;
  if (grid > 0x7fffffff) return DSA_ERR_INVALID_ARG;
  CUtensorMap qmap, kmap;
  if (!dsa_host::encode_tensor_map_2d(&qmap, CU_TENSOR_MAP_DATA_TYPE_UINT8, (void*)q8, 128, (uint64_t)units * 64, 128,
                                      128, kN, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !dsa_host::encode_tensor_map_2d(&kmap, CU_TENSOR_MAP_DATA_TYPE_UINT8, (void*)k8, 128, (uint64_t)B * S_max, 128,
                                      128, kTile, CU_TENSOR_MAP_SWIZZLE_128B))
    return DSA_ERR_CUDA;
  if (p.tps <= 8)
    return launch_clusters(index_topk_kernel<8>, dim3((unsigned)grid), dim3(kThreads), kSmemBytes, stream, C,
                                    qmap, kmap, p);
  if (p.tps <= 16)
    return launch_clusters(index_topk_kernel<16>, dim3((unsigned)grid), dim3(kThreads), kSmemBytes, stream, C,
                                    qmap, kmap, p);
  return launch_clusters(index_topk_kernel<32>, dim3((unsigned)grid), dim3(kThreads), kSmemBytes, stream, C,
                                  qmap, kmap, p);
}

}  // namespace dsa
