// Producers and output projection of the sparse MLA in its absorbed (MQA) form.
//
//   q_absorb   q[t][h][0:512]   = sum_d q_nope[t][h][d] * w_uk[h][d][0:512]        (bf16 MMA, fp32 acc)
//              q[t][h][512:576] = interleaved RoPE_64 of q_pe[t][h] at pos[t]
//   kv_entry   cache[dst][0:512] = kv[t];  cache[dst][512:576] = interleaved RoPE_64 of k_pe[t]
//   out_absorb x[t][h][0:128]   = sum_c o[t][h][c] * w_uv[h][0:128][c]
//
// "DeepSeek-V3.2-Exp - Similarities" page, MQA-decode excerpt: q_nope is multiplied into the latent
// space by wkv_b[:, :qk_nope_head_dim], scores combine the latent and rotary caches, and the
// latent-weighted sum is projected by wkv_b[:, -v_head_dim:]; "Rotate first features" page: MLA
// RoPE pairs features 2j and 2j+1. The q_absorb and out_absorb GEMMs stream their activations once
// and are bound by memory (at decode by the 16.8 MB of weights each reads): TMA tiles with 128-byte
// swizzle, tcgen05 MMAs from shared memory into a double-buffered TMEM accumulator, and one bulk
// copy (TMA engine) per output row.
#include <cuda_bf16.h>

#include <algorithm>

#include "common.cuh"
#include "kernels.h"

namespace dsa {
namespace {

constexpr int kHeadsA = 128;       // MLA heads
constexpr int kNope = 128;         // qk_nope_head_dim
constexpr int kLat = 512;          // kv_lora_rank
constexpr int kRopeD = 64;         // qk_rope_head_dim
constexpr int kVd = 128;           // v_head_dim
constexpr int kQk = kLat + kRopeD;  // 576
constexpr int kRows = 128;         // rows (tokens) per tile = MMA M = TMEM lanes
constexpr int kThreads = 192;      // warp 0 TMA, warp 1 MMA + TMEM owner, warps 2-5 epilogue
constexpr int kRegion = 16384;     // one 128-row x 128-byte swizzled tile region

struct AbsorbParams {
  const uint16_t* q_pe;      // q_absorb: [rows][128][64]
  const int32_t* pos;        // q_absorb: [rows]
  const float* rope_cs;      // [max_pos][32][2]
  int max_pos;
  int64_t rows;
  int tiles_per_cta;         // out_absorb: row tiles each CTA runs (for one head)
  uint16_t* out;             // q_absorb [rows][128][576]; out_absorb [rows][128][128]
  int* status;
};

// 8 packed bf16 pairs (2i, 2i+1) rotated by the (cos, sin) of pairs p0..p0+3 of a table row.
__device__ __forceinline__ uint4 rope_pairs4(uint4 x, const float4* cs2) {
  const float4 c01 = __ldg(cs2), c23 = __ldg(cs2 + 1);       // (cos, sin) of 4 pairs
  const float cs[8] = {c01.x, c01.y, c01.z, c01.w, c23.x, c23.y, c23.z, c23.w};
  const uint32_t in[4] = {x.x, x.y, x.z, x.w};
  uint32_t o[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float a = __uint_as_float(in[i] << 16), b = __uint_as_float(in[i] & 0xFFFF0000u);
    const float c = cs[2 * i], s = cs[2 * i + 1];
    o[i] = pack_bf16(__fsub_rn(__fmul_rn(a, c), __fmul_rn(b, s)), __fadd_rn(__fmul_rn(a, s), __fmul_rn(b, c)));
  }
  return make_uint4(o[0], o[1], o[2], o[3]);
}

// Interleaved RoPE of one 64-feature row (128 B at src) into dst (16-byte aligned). Returns false
// (and writes zeros) for a position outside the table.
__device__ __forceinline__ bool rope_row(const uint16_t* src, int pos, const AbsorbParams& p, uint4* dst) {
  const uint4* s4 = reinterpret_cast<const uint4*>(src);
  if (pos < 0 || pos >= p.max_pos) {
#pragma unroll
    for (int i = 0; i < 8; ++i) dst[i] = make_uint4(0u, 0u, 0u, 0u);
    return false;
  }
  const float4* cs = reinterpret_cast<const float4*>(p.rope_cs + (int64_t)pos * kRopeD);
#pragma unroll
  for (int i = 0; i < 8; ++i) dst[i] = rope_pairs4(__ldg(s4 + i), cs + 2 * i);
  return true;
}

// fp32 TMEM columns -> bf16 in shared memory: 32 columns become 64 bytes
__device__ __forceinline__ void store_bf16_32(uint8_t* dst, const uint32_t (&v)[32]) {
  uint4* d = reinterpret_cast<uint4*>(dst);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint32_t* w = &v[8 * i];
    d[i] = make_uint4(pack_bf16(__uint_as_float(w[0]), __uint_as_float(w[1])),
                      pack_bf16(__uint_as_float(w[2]), __uint_as_float(w[3])),
                      pack_bf16(__uint_as_float(w[4]), __uint_as_float(w[5])),
                      pack_bf16(__uint_as_float(w[6]), __uint_as_float(w[7])));
  }
}

// ------------------------------------------------------------------------------------ q_absorb
// Work item = (head h, 128-row tile): the whole 576-feature q row of head h for the tile's tokens,
// so each q_nope tile is read once. Items are ordered head-major and each CTA (one per SM) runs an
// equal range of them, which crosses into at most a few heads; the head's W_UK[h] (128 KB) stays
// resident in shared memory until its last item, then the next head's is loaded in its place.
// Per item the two 256-feature halves accumulate in their own TMEM accumulator (512 columns), so
// the epilogue drains one half while the MMAs of the other (or of the next tile) run. Each
// epilogue warp writes its 32 rows in 64-feature chunks through four swizzled 4 KB staging buffers
// with TMA tensor stores (full 128-byte lines; rows past the end are clipped by the tensor map).
// Four more warps rotate q_pe (features 512..575, one 128-byte segment per row) for the same
// items, off the epilogue's path: their position -> table loads are the longest latency here.
namespace qa {
constexpr int kThreads = 320;                         // warp 0 TMA, 1 MMA + TMEM owner, 2-5 epilogue, 6-9 RoPE
constexpr int kOffB = 0;                              // W_UK[h]: 8 MN-major regions (64 c x 128 d rows)
constexpr int kOffA = 8 * kRegion;                    // the q_nope tile: 2 K-major regions (128 rows x 64 d)
constexpr int kAStage = 2 * kRegion;
constexpr int kAStages = 1;                           // an item's drain outlasts the next tile's load
constexpr int kStageBytes = 32 * 128;                 // one warp's 32 rows x 64 features, 128B swizzle
constexpr int kStageBufs = 4;                         // staging buffers per epilogue warp (stores in flight)
constexpr int kOffStage = kOffA + kAStages * kAStage;
constexpr int kOffBar = kOffStage + 4 * kStageBufs * kStageBytes;
constexpr int kSmemBytes = kOffBar + 128 + 1024;       // + alignment slack
constexpr int kTmemCols = 512;                        // the two 128 x 256 fp32 halves of one tile
static_assert(kSmemBytes <= 227 * 1024, "shared memory");
static_assert(kOffStage % 1024 == 0 && kStageBytes % 1024 == 0, "128B-swizzled staging alignment");
}  // namespace qa

// TMA tensor store of a shared-memory box to (x, y, z) of the map's tensor, in the bulk group.
__device__ __forceinline__ void tma_store_3d(const CUtensorMap* map, const void* src, int32_t x, int32_t y, int32_t z) {
  asm volatile("cp.async.bulk.tensor.3d.global.shared::cta.bulk_group [%0, {%2, %3, %4}], [%1];"
               ::"l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(src)), "r"(x), "r"(y), "r"(z) : "memory");
}

// Wait until at most N of this thread's bulk groups still have to read their shared-memory source.
template <int N>
__device__ __forceinline__ void bulk_wait_read_n() { asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory"); }

__global__ void __launch_bounds__(qa::kThreads, 1)
    q_absorb_kernel(const __grid_constant__ CUtensorMap a_map, const __grid_constant__ CUtensorMap w_map,
                    const __grid_constant__ CUtensorMap o_map, const AbsorbParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + qa::kOffBar);
  uint64_t* w_full = bars;               // a head's weights landed
  uint64_t* w_empty = bars + 1;          // the MMAs of a head's last item are done with its weights
  uint64_t* a_full = bars + 2;           // [2] q_nope tile landed
  uint64_t* a_empty = bars + 4;          // [2] MMAs done reading the tile
  uint64_t* acc_full = bars + 6;         // [2] half n of the item's product ready
  uint64_t* acc_empty = bars + 8;        // [2] half n drained (128 arrivals)
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_flag;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int64_t ntiles = (p.rows + kRows - 1) / kRows;
  const int64_t items = (int64_t)kHeadsA * ntiles;
  const int64_t i0 = (int64_t)blockIdx.x * items / gridDim.x;
  const int my_items = (int)((int64_t)(blockIdx.x + 1) * items / gridDim.x - i0);
  const int h0 = (int)(i0 / ntiles);
  // item j of this CTA: its head, its tile, and whether it is the first of its head here
  auto head_of = [&](int j) { return (int)((i0 + j) / ntiles); };
  auto tile_of = [&](int j) { return (i0 + j) % ntiles; };
  auto new_head = [&](int j) { return j == 0 || tile_of(j) == 0; };

  if (tid == 0) {
    abort_flag = 0;
    mbar_init(w_full, 1);
    mbar_init(w_empty, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&a_full[i], 1);
      mbar_init(&a_empty[i], 1);
      mbar_init(&acc_full[i], 1);
      mbar_init(&acc_empty[i], 4 * 32);
    }
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(&tmem_base_sh, qa::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_sh;
  grid_dep_wait();                       // activations and outputs are shared with earlier kernels
  grid_dep_launch();

  if (warp == 0) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0 && my_items > 0) {
      prefetch_tensormap(&a_map);
      prefetch_tensormap(&w_map);
      for (int j = 0; j < my_items; ++j) {
        const int h = head_of(j);
        if (new_head(j)) {
          const int seg = h - h0;
          if (seg > 0 && !mbar_wait(w_empty, (seg - 1) & 1, &abort_flag, p.status, DSA_SITE_ABSORB_W)) break;
          mbar_arrive_expect_tx(w_full, 8 * kRegion);
          for (int r = 0; r < 8; ++r) tma_load_3d(smem + qa::kOffB + r * kRegion, &w_map, w_full, 64 * r, 0, h);
        }
        const int s = j % qa::kAStages;
        if (j >= qa::kAStages &&
            !mbar_wait(&a_empty[s], (j / qa::kAStages - 1) & 1, &abort_flag, p.status, DSA_SITE_ABSORB_A_EMPTY))
          break;
        mbar_arrive_expect_tx(&a_full[s], qa::kAStage);
        const int32_t t = (int32_t)(tile_of(j) * kRows);
        uint8_t* dst = smem + qa::kOffA + s * qa::kAStage;
        tma_load_3d(dst, &a_map, &a_full[s], 0, h, t);
        tma_load_3d(dst + kRegion, &a_map, &a_full[s], 64, h, t);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0 && my_items > 0) {
      constexpr uint32_t idesc = idesc_f32acc(1, 1, kRows, 256, 0, 1 /*B MN-major*/);
      const uint32_t b_addr = smem_u32(smem + qa::kOffB);
      bool ok = true;
      for (int j = 0; ok && j < my_items; ++j) {
        if (new_head(j) && !mbar_wait(w_full, (head_of(j) - h0) & 1, &abort_flag, p.status, DSA_SITE_ABSORB_W)) break;
        const int s = j % qa::kAStages;
        if (!mbar_wait(&a_full[s], (j / qa::kAStages) & 1, &abort_flag, p.status, DSA_SITE_ABSORB_A_FULL)) break;
        const uint32_t a_addr = smem_u32(smem + qa::kOffA + s * qa::kAStage);
        for (int n = 0; n < 2; ++n) {
          if (j >= 1 && !mbar_wait(&acc_empty[n], (j - 1) & 1, &abort_flag, p.status, DSA_SITE_ABSORB_ACC_EMPTY)) {
            ok = false;
            break;
          }
          tc_fence_after();
#pragma unroll
          for (int ks = 0; ks < kNope / 16; ++ks) {
            const uint64_t ad = sdesc_kmajor_sw128(a_addr + (ks >> 2) * kRegion + (ks & 3) * 32);
            const uint64_t bd = sdesc_mnmajor_sw128(b_addr + n * 4 * kRegion + ks * 2048, kRegion, 1024);
            mma_f16_ss(tmem + n * 256, ad, bd, idesc, ks > 0 ? 1u : 0u);
          }
          mma_commit(&acc_full[n]);
        }
        if (!ok) break;
        mma_commit(&a_empty[s]);
        if (j + 1 < my_items && new_head(j + 1)) mma_commit(w_empty);   // the next head may replace the weights
      }
    }
  } else if (warp >= 6) {
    // ------------------------------------------------------------------ RoPE (warps 6-9)
    // thread = tile row; the next item's position is loaded one item ahead
    const int r = tid - 6 * 32;
    auto row_of = [&](int j) { return tile_of(j) * kRows + r; };
    int pos_next = my_items > 0 && row_of(0) < p.rows ? __ldg(p.pos + row_of(0)) : 0;
    for (int j = 0; j < my_items; ++j) {
      const int64_t t = row_of(j);
      const int pos = pos_next;
      if (j + 1 < my_items && row_of(j + 1) < p.rows) pos_next = __ldg(p.pos + row_of(j + 1));
      if (t >= p.rows) continue;
      const int h = head_of(j);
      uint4 rv[8];
      if (!rope_row(p.q_pe + (t * kHeadsA + h) * kRopeD, pos, p, rv)) set_status(p.status, DSA_ERR_DEVICE_BOUNDS);
      uint4* dst = reinterpret_cast<uint4*>(p.out + (t * kHeadsA + h) * kQk + kLat);
#pragma unroll
      for (int c = 0; c < 8; ++c) dst[c] = rv[c];
    }
  } else {
    // ------------------------------------------------------------------ epilogue (warps 2-5)
    // warp w reads TMEM lane quadrant w % 4: one tile row per thread, 32 rows per warp
    const int quad = warp & 3;
    uint8_t* stage = smem + qa::kOffStage + quad * qa::kStageBufs * qa::kStageBytes;
    uint32_t chunks = 0;                                     // 64-feature chunks this warp has staged
    // stage one 64-feature chunk (32 packed bf16 pairs) of this lane's row, then store the warp's box
    auto put = [&](const uint32_t (&v)[32], int feat, int h, int32_t z, bool live) {
      uint8_t* buf = stage + (chunks % qa::kStageBufs) * qa::kStageBytes;
      if (lane == 0 && chunks >= qa::kStageBufs)            // the store that last read this buffer is done
        bulk_wait_read_n<qa::kStageBufs - 1>();
      __syncwarp();
#pragma unroll
      for (int c = 0; c < 8; ++c)                            // 128B swizzle: 16-byte chunk c of row r at c ^ (r % 8)
        *reinterpret_cast<uint4*>(buf + lane * 128 + ((c ^ (lane & 7)) << 4)) =
            make_uint4(v[4 * c], v[4 * c + 1], v[4 * c + 2], v[4 * c + 3]);
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0 && live) {
        tma_store_3d(&o_map, buf, feat, h, z);
        bulk_commit();
      }
      ++chunks;
    };
    for (int j = 0; j < my_items; ++j) {
      const int h = head_of(j);
      const int32_t z = (int32_t)(tile_of(j) * kRows + quad * 32);   // this warp's first row
      const bool live = z < p.rows;
      bool ok = true;
      for (int n = 0; n < 2; ++n) {
        if (!__all_sync(0xffffffffu, mbar_wait(&acc_full[n], j & 1, &abort_flag, p.status, DSA_SITE_ABSORB_ACC_FULL))) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t taddr = tmem + ((uint32_t)(quad * 32) << 16) + n * 256;
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
          uint32_t x0[32], x1[32], v[32];
          tmem_ld32(taddr + c * 64, x0);
          tmem_ld32(taddr + c * 64 + 32, x1);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            v[i] = pack_bf16(__uint_as_float(x0[2 * i]), __uint_as_float(x0[2 * i + 1]));
            v[16 + i] = pack_bf16(__uint_as_float(x1[2 * i]), __uint_as_float(x1[2 * i + 1]));
          }
          put(v, 256 * n + 64 * c, h, z, live);
        }
        tc_fence_before();
        mbar_arrive(&acc_empty[n]);
      }
      if (!ok) break;
    }
    if (lane == 0) bulk_wait_all();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, qa::kTmemCols);
  }
}

// ------------------------------------------------------------------------------------ out_absorb
// CTA = (group of row tiles, head h): x[t][h][0:128] for its tiles. K (512 latent features) streams
// in 8 chunks of 64 through a 4-stage ring; each stage holds the o chunk (128 rows x 64 c, K-major)
// and the w_uv chunk (128 d rows x 64 c, K-major). Accumulator: 128 x 128 fp32, double-buffered.
namespace oa {
constexpr int kStages = 4;
constexpr int kStageBytes = 2 * kRegion;
constexpr int kRowBytes = 272;                        // 256 B (128 bf16) + 16 B pad
constexpr int kOffStage = kStages * kStageBytes;
constexpr int kOffBar = kOffStage + kRows * kRowBytes;
constexpr int kSmemBytes = kOffBar + 128 + 1024;
constexpr int kTmemCols = 256;
constexpr int kChunks = kLat / 64;
static_assert(kSmemBytes <= 227 * 1024, "shared memory");
}  // namespace oa

__global__ void __launch_bounds__(kThreads, 1)
    out_absorb_kernel(const __grid_constant__ CUtensorMap a_map, const __grid_constant__ CUtensorMap w_map,
                      const AbsorbParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + oa::kOffBar);
  uint64_t* full = bars;                          // [kStages]
  uint64_t* empty = bars + oa::kStages;           // [kStages]
  uint64_t* acc_full = bars + 2 * oa::kStages;    // [2]
  uint64_t* acc_empty = acc_full + 2;             // [2]
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_flag;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int h = blockIdx.x % kHeadsA;
  const int64_t g = blockIdx.x / kHeadsA;
  const int64_t ntiles = (p.rows + kRows - 1) / kRows;
  const int64_t tile0 = g * p.tiles_per_cta;
  const int my_tiles = (int)max((int64_t)0, min((int64_t)p.tiles_per_cta, ntiles - tile0));

  if (tid == 0) {
    abort_flag = 0;
    for (int s = 0; s < oa::kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&acc_full[i], 1);
      mbar_init(&acc_empty[i], 4 * 32);
    }
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(&tmem_base_sh, oa::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_sh;
  grid_dep_wait();                       // activations and outputs are shared with earlier kernels
  grid_dep_launch();
  const int nsteps = my_tiles * oa::kChunks;

  if (warp == 0) {
    if (lane == 0 && my_tiles > 0) {
      prefetch_tensormap(&a_map);
      prefetch_tensormap(&w_map);
      for (int q = 0; q < nsteps; ++q) {
        const int s = q % oa::kStages, kc = q % oa::kChunks;
        if (q >= oa::kStages &&
            !mbar_wait(&empty[s], ((q / oa::kStages) + 1) & 1, &abort_flag, p.status, DSA_SITE_ABSORB_A_EMPTY))
          break;
        mbar_arrive_expect_tx(&full[s], oa::kStageBytes);
        const int32_t t = (int32_t)((tile0 + q / oa::kChunks) * kRows);
        uint8_t* dst = smem + s * oa::kStageBytes;
        tma_load_3d(dst, &a_map, &full[s], 64 * kc, h, t);
        tma_load_3d(dst + kRegion, &w_map, &full[s], 64 * kc, 0, h);
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && my_tiles > 0) {
      constexpr uint32_t idesc = idesc_f32acc(1, 1, kRows, kVd, 0, 0);
      bool ok = true;
      for (int i = 0; ok && i < my_tiles; ++i) {
        const int a = i & 1;
        if (i >= 2 && !mbar_wait(&acc_empty[a], ((i >> 1) + 1) & 1, &abort_flag, p.status, DSA_SITE_ABSORB_ACC_EMPTY))
          break;
        for (int kc = 0; kc < oa::kChunks; ++kc) {
          const int q = i * oa::kChunks + kc, s = q % oa::kStages;
          if (!mbar_wait(&full[s], (q / oa::kStages) & 1, &abort_flag, p.status, DSA_SITE_ABSORB_A_FULL)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t base = smem_u32(smem + s * oa::kStageBytes);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_f16_ss(tmem + a * kVd, sdesc_kmajor_sw128(base + kk * 32), sdesc_kmajor_sw128(base + kRegion + kk * 32),
                       idesc, (kc | kk) ? 1u : 0u);
          mma_commit(&empty[s]);
        }
        if (ok) mma_commit(&acc_full[a]);
      }
    }
  } else {
    const int quad = warp & 3;
    const int r = quad * 32 + lane;
    uint8_t* srow = smem + oa::kOffStage + r * oa::kRowBytes;
    for (int i = 0; i < my_tiles; ++i) {
      const int a = i & 1;
      if (!__all_sync(0xffffffffu, mbar_wait(&acc_full[a], (i >> 1) & 1, &abort_flag, p.status,
                                             DSA_SITE_ABSORB_ACC_FULL)))
        break;
      tc_fence_after();
      const int64_t t = (tile0 + i) * kRows + r;
      if (i > 0) bulk_wait_read();
      const uint32_t taddr = tmem + ((uint32_t)(quad * 32) << 16) + a * kVd;
#pragma unroll 1
      for (int c = 0; c < 4; c += 2) {
        uint32_t v0[32], v1[32];
        tmem_ld32(taddr + c * 32, v0);
        tmem_ld32(taddr + (c + 1) * 32, v1);
        tmem_ld_wait();
        store_bf16_32(srow + c * 64, v0);
        store_bf16_32(srow + (c + 1) * 64, v1);
      }
      tc_fence_before();
      mbar_arrive(&acc_empty[a]);
      if (t < p.rows) {
        fence_proxy_async_smem();
        bulk_store_s2g(p.out + (t * kHeadsA + h) * kVd, smem_u32(srow), kVd * 2);
        bulk_commit();
      }
    }
    bulk_wait_all();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, oa::kTmemCols);
  }
}

// ------------------------------------------------------------------------------------ few rows
// Decode shapes (rows <= 64): one CTA per head in the swapped orientation, weights on M and the
// tokens on N (rows rounded up to 16), so each head's 128 KB of weights is read once, by one CTA,
// in under one wave. The weight chunks land behind per-chunk barriers and the MMAs start as they
// arrive; after the last MMA the weight buffer stages the output rows (one bulk copy per token).
namespace fr {
constexpr int kMaxRows = 64;
constexpr int kOffW = 0;                          // 8 regions of 16 KB (weights)
constexpr int kOffX = 8 * kRegion;                // activation regions, kMaxRows x 128 B each
constexpr int kXRegion = kMaxRows * 128;
constexpr int kOffBar = kOffX + 8 * kXRegion;
constexpr int kSmemBytes = kOffBar + 128 + 1024;
constexpr int kTmemCols = 256;
static_assert(kSmemBytes <= 227 * 1024, "shared memory");
}  // namespace fr

__device__ __forceinline__ void st_shared_u16(uint8_t* p, uint16_t v) {
  asm volatile("st.shared.u16 [%0], %1;" ::"r"(smem_u32(p)), "h"(v) : "memory");
}
__device__ __forceinline__ uint16_t bf16_bits(float x) {
  return (uint16_t)(pack_bf16(x, 0.f) & 0xFFFFu);
}

// q_absorb, rows <= 64: D^T[c][t] = sum_d w_uk[h][d][c] q_nope[t][h][d]; A = the weights as four
// 128-c M blocks (MN-major: c contiguous), B = the q_nope rows (K-major), N = n_pad.
__global__ void __launch_bounds__(kThreads, 1)
    q_absorb_few_kernel(const __grid_constant__ CUtensorMap a_map, const __grid_constant__ CUtensorMap w_map,
                        const AbsorbParams p, int n_pad) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + fr::kOffBar);
  uint64_t* w_full = bars;          // [4] weights of M block m landed
  uint64_t* x_full = bars + 4;      // q_nope rows landed
  uint64_t* acc_full = bars + 5;    // all MMAs done
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_flag;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int h = blockIdx.x;
  const int rows = (int)p.rows;
  if (tid == 0) {
    abort_flag = 0;
    for (int i = 0; i < 6; ++i) mbar_init(&bars[i], 1);
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(&tmem_base_sh, fr::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_sh;
  grid_dep_wait();                       // activations and outputs are shared with earlier kernels
  grid_dep_launch();

  if (warp == 0) {
    if (lane == 0) {
      mbar_arrive_expect_tx(x_full, 2 * n_pad * 128);
      for (int r = 0; r < 2; ++r) tma_load_3d(smem + fr::kOffX + r * fr::kXRegion, &a_map, x_full, 64 * r, h, 0);
      for (int m = 0; m < 4; ++m) {
        mbar_arrive_expect_tx(&w_full[m], 2 * kRegion);
        for (int j = 2 * m; j < 2 * m + 2; ++j)
          tma_load_3d(smem + fr::kOffW + j * kRegion, &w_map, &w_full[m], 64 * j, 0, h);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = idesc_f32acc(1, 1, kRows, (uint32_t)n_pad, 1 /*A MN-major*/, 0);
      const uint32_t w_addr = smem_u32(smem + fr::kOffW), x_addr = smem_u32(smem + fr::kOffX);
      bool ok = mbar_wait(x_full, 0, &abort_flag, p.status, DSA_SITE_ABSORB_A_FULL);
      for (int m = 0; ok && m < 4; ++m) {
        if (!mbar_wait(&w_full[m], 0, &abort_flag, p.status, DSA_SITE_ABSORB_W)) {
          ok = false;
          break;
        }
        tc_fence_after();
#pragma unroll
        for (int ks = 0; ks < kNope / 16; ++ks) {
          const uint64_t ad = sdesc_mnmajor_sw128(w_addr + 2 * m * kRegion + ks * 2048, kRegion, 1024);
          const uint64_t bd = sdesc_kmajor_sw128(x_addr + (ks >> 2) * fr::kXRegion + (ks & 3) * 32);
          mma_f16_ss(tmem + m * n_pad, ad, bd, idesc, ks > 0 ? 1u : 0u);
        }
      }
      if (ok) mma_commit(acc_full);
    }
  } else {
    const int quad = warp & 3, et = tid - 64;           // epilogue thread 0..127
    uint8_t* stage = smem + fr::kOffW;                   // rows of 1152 B over the consumed weights
    // rotary inputs of this thread's (token, pair) entries, loaded while the MMAs run
    constexpr int kPairsPerThread = fr::kMaxRows * 32 / 128;
    uint32_t pe[kPairsPerThread];
    float2 pcs[kPairsPerThread];
    int pps[kPairsPerThread];
#pragma unroll
    for (int r = 0; r < kPairsPerThread; ++r) {
      const int i = et + r * 128, t = i >> 5, pr = i & 31;
      pps[r] = -1;
      if (i < rows * 32) {
        pps[r] = __ldg(p.pos + t);
        pe[r] = __ldg(reinterpret_cast<const uint32_t*>(p.q_pe + ((int64_t)t * kHeadsA + h) * kRopeD) + pr);
      }
    }
#pragma unroll
    for (int r = 0; r < kPairsPerThread; ++r) {
      const int pr = (et + r * 128) & 31;
      pcs[r] = make_float2(1.f, 0.f);
      if (pps[r] >= 0 && pps[r] < p.max_pos)
        pcs[r] = __ldg(reinterpret_cast<const float2*>(p.rope_cs + (int64_t)pps[r] * kRopeD) + pr);
    }
    const bool ok = __all_sync(0xffffffffu, mbar_wait(acc_full, 0, &abort_flag, p.status, DSA_SITE_ABSORB_ACC_FULL));
    if (ok) {
      tc_fence_after();
      for (int m = 0; m < 4; ++m) {
        const int c = 128 * m + 32 * quad + lane;
        for (int cc = 0; cc < n_pad; cc += 32) {
          uint32_t v[32];
          tmem_ld32(tmem + ((uint32_t)(quad * 32) << 16) + m * n_pad + cc, v);
          tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < 32; ++j)
            if (cc + j < rows) st_shared_u16(stage + (cc + j) * (kQk * 2) + c * 2, bf16_bits(__uint_as_float(v[j])));
        }
      }
      // rotary part: thread = (token, pair)
#pragma unroll
      for (int r = 0; r < kPairsPerThread; ++r) {
        const int i = et + r * 128, t = i >> 5, pr = i & 31;
        if (i >= rows * 32) continue;
        uint32_t o = 0u;
        if (pps[r] >= 0 && pps[r] < p.max_pos) {
          const float a = __uint_as_float(pe[r] << 16), b = __uint_as_float(pe[r] & 0xFFFF0000u);
          const float2 cs = pcs[r];
          o = pack_bf16(__fsub_rn(__fmul_rn(a, cs.x), __fmul_rn(b, cs.y)), __fadd_rn(__fmul_rn(a, cs.y), __fmul_rn(b, cs.x)));
        } else if (pr == 0) {
          set_status(p.status, DSA_ERR_DEVICE_BOUNDS);
        }
        *reinterpret_cast<uint32_t*>(stage + t * (kQk * 2) + kLat * 2 + pr * 4) = o;
      }
      fence_proxy_async_smem();
    }
    // every epilogue warp reaches the barrier, whether or not its wait succeeded
    asm volatile("bar.sync 1, 128;" ::: "memory");        // the epilogue warps' rows are complete
    if (ok) {
      for (int t = et; t < rows; t += 128) {
        bulk_store_s2g(p.out + ((int64_t)t * kHeadsA + h) * kQk, smem_u32(stage + t * (kQk * 2)), kQk * 2);
        bulk_commit();
      }
      bulk_wait_all();
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, fr::kTmemCols);
  }
}

// out_absorb, rows <= 64: D^T[d][t] = sum_c w_uv[h][d][c] o[t][h][c]; A = the weights (K-major),
// B = the o rows (K-major), K streamed in 8 chunks of 64 behind per-chunk barriers.
__global__ void __launch_bounds__(kThreads, 1)
    out_absorb_few_kernel(const __grid_constant__ CUtensorMap a_map, const __grid_constant__ CUtensorMap w_map,
                          const AbsorbParams p, int n_pad) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + fr::kOffBar);
  uint64_t* full = bars;            // [8] chunk kc (weights + rows) landed
  uint64_t* acc_full = bars + 8;
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_flag;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int h = blockIdx.x;
  const int rows = (int)p.rows;
  if (tid == 0) {
    abort_flag = 0;
    for (int i = 0; i < 9; ++i) mbar_init(&bars[i], 1);
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(&tmem_base_sh, fr::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_sh;
  grid_dep_wait();                       // activations and outputs are shared with earlier kernels
  grid_dep_launch();

  if (warp == 0) {
    if (lane == 0) {
      for (int kc = 0; kc < 8; ++kc) {
        mbar_arrive_expect_tx(&full[kc], kRegion + n_pad * 128);
        tma_load_3d(smem + fr::kOffW + kc * kRegion, &w_map, &full[kc], 64 * kc, 0, h);
        tma_load_3d(smem + fr::kOffX + kc * fr::kXRegion, &a_map, &full[kc], 64 * kc, h, 0);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = idesc_f32acc(1, 1, kRows, (uint32_t)n_pad, 0, 0);
      const uint32_t w_addr = smem_u32(smem + fr::kOffW), x_addr = smem_u32(smem + fr::kOffX);
      bool ok = true;
      for (int kc = 0; ok && kc < 8; ++kc) {
        if (!mbar_wait(&full[kc], 0, &abort_flag, p.status, DSA_SITE_ABSORB_A_FULL)) {
          ok = false;
          break;
        }
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_f16_ss(tmem, sdesc_kmajor_sw128(w_addr + kc * kRegion + kk * 32),
                     sdesc_kmajor_sw128(x_addr + kc * fr::kXRegion + kk * 32), idesc, (kc | kk) ? 1u : 0u);
      }
      if (ok) mma_commit(acc_full);
    }
  } else {
    const int quad = warp & 3, et = tid - 64;
    uint8_t* stage = smem + fr::kOffW;                   // rows of 256 B over the consumed weights
    const bool ok = __all_sync(0xffffffffu, mbar_wait(acc_full, 0, &abort_flag, p.status, DSA_SITE_ABSORB_ACC_FULL));
    if (ok) {
      tc_fence_after();
      const int d = 32 * quad + lane;
      for (int cc = 0; cc < n_pad; cc += 32) {
        uint32_t v[32];
        tmem_ld32(tmem + ((uint32_t)(quad * 32) << 16) + cc, v);
        tmem_ld_wait();
#pragma unroll
        for (int j = 0; j < 32; ++j)
          if (cc + j < rows) st_shared_u16(stage + (cc + j) * (kVd * 2) + d * 2, bf16_bits(__uint_as_float(v[j])));
      }
      fence_proxy_async_smem();
    }
    asm volatile("bar.sync 1, 128;" ::: "memory");        // reached by every epilogue warp
    if (ok) {
      for (int t = et; t < rows; t += 128) {
        bulk_store_s2g(p.out + ((int64_t)t * kHeadsA + h) * kVd, smem_u32(stage + t * (kVd * 2)), kVd * 2);
        bulk_commit();
      }
      bulk_wait_all();
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, fr::kTmemCols);
  }
}

// ------------------------------------------------------------------------------------ kv_entry
// One warp per token: lanes copy the 1 KB latent row (two 16-byte chunks each) and rotate one
// rotary pair each into the cache row dst_row[t].
__global__ void __launch_bounds__(256) kv_entry_kernel(const uint16_t* kv, const uint16_t* k_pe, const int32_t* pos,
                                                       const float* rope_cs, int max_pos, int64_t rows,
                                                       const int64_t* dst_row, uint16_t* cache, int64_t cache_rows,
                                                       int* status) {
  const int64_t t = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  grid_dep_wait();
  grid_dep_launch();
  if (t >= rows) return;
  const int64_t dst = __ldg(dst_row + t);
  const int ps = __ldg(pos + t);
  if (dst < 0 || dst >= cache_rows || ps < 0 || ps >= max_pos) {
    if (lane == 0) set_status(status, DSA_ERR_DEVICE_BOUNDS);
    return;
  }
  const uint4* src = reinterpret_cast<const uint4*>(kv + t * kLat);
  uint4* out = reinterpret_cast<uint4*>(cache + dst * kQk);
  const uint4 v0 = __ldg(src + lane), v1 = __ldg(src + 32 + lane);
  const uint32_t x = __ldg(reinterpret_cast<const uint32_t*>(k_pe + t * kRopeD) + lane);
  const float2 cs = __ldg(reinterpret_cast<const float2*>(rope_cs + (int64_t)ps * kRopeD) + lane);
  const float a = __uint_as_float(x << 16), b = __uint_as_float(x & 0xFFFF0000u);
  out[lane] = v0;
  out[32 + lane] = v1;
  reinterpret_cast<uint32_t*>(cache + dst * kQk + kLat)[lane] =
      pack_bf16(__fsub_rn(__fmul_rn(a, cs.x), __fmul_rn(b, cs.y)), __fadd_rn(__fmul_rn(a, cs.y), __fmul_rn(b, cs.x)));
}

// Row tiles per CTA: enough CTAs for about eight per SM over the whole grid, at least one tile each.
int tiles_per_cta(int64_t ntiles, int64_t ctas_per_group) {
  const int64_t target = (int64_t)dsa_host::device_sm_count() * 8;
  int64_t tpc = (ntiles * ctas_per_group + target - 1) / target;
  return (int)std::max<int64_t>(1, std::min<int64_t>(tpc, ntiles));
}

bool configure(const void* func, int smem_bytes) {
  return cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_bytes) == cudaSuccess;
}

}  // namespace

int launch_mla_q_absorb(const uint16_t* q_nope, const uint16_t* q_pe, const int32_t* pos, const float* rope_cs,
                        int max_pos, const uint16_t* w_uk, int64_t w_head_stride, int64_t rows, uint16_t* q_out,
                        cudaStream_t stream, int* status) {
  if (rows == 0) return DSA_OK;
  CUtensorMap a_map, w_map;
  const uint64_t a_dims[3] = {kNope, kHeadsA, (uint64_t)rows};
  const uint64_t a_str[2] = {kNope * 2, (uint64_t)kHeadsA * kNope * 2};
  const uint32_t a_box[3] = {64, 1, kRows};
  const uint64_t w_dims[3] = {kLat, kNope, kHeadsA};
  const uint64_t w_str[2] = {kLat * 2, (uint64_t)w_head_stride * 2};
  const uint32_t w_box[3] = {64, kNope, 1};
  if (!dsa_host::encode_tensor_map_3d(&a_map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, (void*)q_nope, a_dims, a_str, a_box,
                                      CU_TENSOR_MAP_SWIZZLE_128B) ||
      !dsa_host::encode_tensor_map_3d(&w_map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, (void*)w_uk, w_dims, w_str, w_box,
                                      CU_TENSOR_MAP_SWIZZLE_128B))
    return DSA_ERR_CUDA;
  static uint64_t configured[dsa_host::kMaxSetupDevices] = {};
  if (dsa_host::needs_setup(configured, nullptr)) {
    if (!configure((const void*)q_absorb_kernel, qa::kSmemBytes) ||
        !configure((const void*)q_absorb_few_kernel, fr::kSmemBytes))
      return DSA_ERR_CUDA;
    dsa_host::mark_setup(configured);
  }
  const int64_t ntiles = (rows + kRows - 1) / kRows;
  AbsorbParams p{};
  p.q_pe = q_pe; p.pos = pos; p.rope_cs = rope_cs; p.max_pos = max_pos; p.rows = rows;
  if (rows <= fr::kMaxRows) {
    const int n_pad = (int)((rows + 15) / 16 * 16);
    const uint32_t x_box[3] = {64, 1, (uint32_t)n_pad};
    CUtensorMap x_map;
    if (!dsa_host::encode_tensor_map_3d(&x_map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, (void*)q_nope, a_dims, a_str,
                                        x_box, CU_TENSOR_MAP_SWIZZLE_128B))
      return DSA_ERR_CUDA;
    p.tiles_per_cta = 1;
    p.out = q_out; p.status = status;
    return dsa_host::launch(q_absorb_few_kernel, dim3(kHeadsA), dim3(kThreads), fr::kSmemBytes, stream, x_map, w_map,
                            p, n_pad);
  }
  // the output q [rows][128][576], written in boxes of 32 rows x 64 features of one head
  CUtensorMap o_map;
  const uint64_t o_dims[3] = {kQk, kHeadsA, (uint64_t)rows};
  const uint64_t o_str[2] = {kQk * 2, (uint64_t)kHeadsA * kQk * 2};
  const uint32_t o_box[3] = {64, 1, 32};
  if (!dsa_host::encode_tensor_map_3d(&o_map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, (void*)q_out, o_dims, o_str, o_box,
                                      CU_TENSOR_MAP_SWIZZLE_128B))
    return DSA_ERR_CUDA;
  p.tiles_per_cta = 0;                       // items are split evenly over one CTA per SM
  p.out = q_out; p.status = status;
  const int64_t grid = std::min<int64_t>(dsa_host::device_sm_count(), ntiles * kHeadsA);
  return dsa_host::launch(q_absorb_kernel, dim3((unsigned)grid), dim3(qa::kThreads), qa::kSmemBytes, stream, a_map,
                          w_map, o_map, p);
}

int launch_mla_out_absorb(const uint16_t* o, const uint16_t* w_uv, int64_t w_head_stride, int64_t rows,
                          uint16_t* out, cudaStream_t stream, int* status) {
  if (rows == 0) return DSA_OK;
  CUtensorMap a_map, w_map;
  const uint64_t a_dims[3] = {kLat, kHeadsA, (uint64_t)rows};
  const uint64_t a_str[2] = {kLat * 2, (uint64_t)kHeadsA * kLat * 2};
  const uint32_t a_box[3] = {64, 1, kRows};
  const uint64_t w_dims[3] = {kLat, kVd, kHeadsA};
  const uint64_t w_str[2] = {kLat * 2, (uint64_t)w_head_stride * 2};
  const uint32_t w_box[3] = {64, kVd, 1};
  if (!dsa_host::encode_tensor_map_3d(&a_map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, (void*)o, a_dims, a_str, a_box,
                                      CU_TENSOR_MAP_SWIZZLE_128B) ||
      !dsa_host::encode_tensor_map_3d(&w_map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, (void*)w_uv, w_dims, w_str, w_box,
                                      CU_TENSOR_MAP_SWIZZLE_128B))
    return DSA_ERR_CUDA;
  static uint64_t configured[dsa_host::kMaxSetupDevices] = {};
  if (dsa_host::needs_setup(configured, nullptr)) {
    if (!configure((const void*)out_absorb_kernel, oa::kSmemBytes) ||
        !configure((const void*)out_absorb_few_kernel, fr::kSmemBytes))
      return DSA_ERR_CUDA;
    dsa_host::mark_setup(configured);
  }
  const int64_t ntiles = (rows + kRows - 1) / kRows;
  AbsorbParams p{};
  p.rows = rows;
  if (rows <= fr::kMaxRows) {
    const int n_pad = (int)((rows + 15) / 16 * 16);
    const uint32_t x_box[3] = {64, 1, (uint32_t)n_pad};
    CUtensorMap x_map;
    if (!dsa_host::encode_tensor_map_3d(&x_map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, (void*)o, a_dims, a_str, x_box,
                                        CU_TENSOR_MAP_SWIZZLE_128B))
      return DSA_ERR_CUDA;
    p.tiles_per_cta = 1;
    p.out = out; p.status = status;
    return dsa_host::launch(out_absorb_few_kernel, dim3(kHeadsA), dim3(kThreads), fr::kSmemBytes, stream, x_map,
                            w_map, p, n_pad);
  }
  p.tiles_per_cta = tiles_per_cta(ntiles, kHeadsA);
  p.out = out; p.status = status;
  const int64_t grid = (ntiles + p.tiles_per_cta - 1) / p.tiles_per_cta * kHeadsA;
  if (grid > 0x7fffffff) return DSA_ERR_INVALID_ARG;
  return dsa_host::launch(out_absorb_kernel, dim3((unsigned)grid), dim3(kThreads), oa::kSmemBytes, stream, a_map,
                          w_map, p);
}

int launch_mla_kv_entry(const uint16_t* kv, const uint16_t* k_pe, const int32_t* pos, const float* rope_cs,
                        int max_pos, int64_t rows, const int64_t* dst_row, uint16_t* kv_cache, int64_t cache_rows,
                        cudaStream_t stream, int* status) {
  if (rows == 0) return DSA_OK;
  const int64_t grid = (rows + 7) / 8;
  if (grid > 0x7fffffff) return DSA_ERR_INVALID_ARG;
  return dsa_host::launch(kv_entry_kernel, dim3((unsigned)grid), dim3(256), 0, stream, kv, k_pe, pos, rope_cs, max_pos,
                          rows, dst_row, kv_cache, cache_rows, status);
}

}  // namespace dsa
