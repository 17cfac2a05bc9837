// dsa_sparse_mla: sparse MQA-style latent attention over the selected positions.
//
// For each (b, t, head h): z_u = scale * q[h] . kv[idx_u] over the 576 features (512 latent +
// 64 rotary), p = softmax over the selected u, out[h] = sum_u p_u kv[idx_u][0:512]. This is the
// absorbed MQA decode of "DeepSeek-V3.2-Exp - Similarities" (model.py 590-606 excerpt: latent and
// rotary score terms, index mask, softmax, latent-weighted sum) with the index mask replaced by a
// gather of the selected rows, and the sparse-attention steps of the dense-block page
// (S' = S m^2/sqrt 192, A = softmax, O = AV).
//
// Tensor cores (tcgen05, kind::f16, bf16 in / fp32 accumulate in TMEM). A 128-head x 512 fp32
// output accumulator alone would fill all 512 TMEM columns, so each (query, key split) runs on two
// CTAs that split the OUTPUT features: CTA c accumulates out[:, 256c:256c+256) (256 TMEM columns).
// Each CTA computes the full 576-feature score itself (Q for all 128 heads resident on chip: features
// 0..255 in TMEM as bf16 pairs, 256..575 in shared memory via TMA), so the pair never exchanges data: this costs 1.5x the Q K^T work
// of a single pass, but exchanging 128 x 64 fp32 partial scores per tile between CTAs runs into
// the limited bandwidth of distributed shared memory.
//
// Selected 1152-byte latent rows are gathered by four warps with 16-byte cp.async, one warp-wide
// coalesced 512-byte request per instruction, written straight into the 128B-swizzled operand
// layout (unselected slots are zero-filled) into a double-buffered ring of 64-key tiles. (Measured
// on B200 with one CTA per SM: this moves ~2.5x more bytes per SM than TMA tile::gather4 with
// 128-byte boxes.) One shared-memory tile is both the
// K-major B operand of Q K^T (N = keys) and the MN-major B operand of P V (N = features).
// TMEM: O [0,256), two score buffers S0 [256,320) and S1 [320,384), Q features 0..255 as bf16
// pairs [384,512) (the A operand of the first 16 K-steps of Q K^T; the last 20 read Q from shared
// memory). The probabilities of tile j overwrite the first 32 columns of the score buffer they came
// from (bf16 pairs, the A operand of P V), so the MMA thread can run a fixed order
// S0, S1, PV0, S2, PV1, S3, ...: Q K^T of tile j+2 is issued after P V of tile j, which the tensor
// pipe executes in order, and it never waits for the softmax to free a buffer.
// Per CTA: 4 softmax warps (thread = head = TMEM lane), 1 MMA-issuing thread that issues Q K^T and
// P V in whichever order their inputs become ready, 4 gather warps (the first also loads Q by TMA). The running max is only moved
// (and O rescaled in TMEM) when it grows by more than 2^8. With several key splits per query, fp32
// partials (O, max, sum) go to the caller's workspace and a second kernel merges them.
#include <cuda_bf16.h>
#include <math.h>

#include <algorithm>

#include "common.cuh"
#include "kernels.h"

namespace dsa {

namespace {

constexpr int kHeads = 128;
constexpr int kDqk = 576;
constexpr int kDv = 512;
constexpr int kKeys = 64;                          // selected keys per tile (N of Q K^T)
constexpr int kRegions = 9;                        // 576 features = 9 blocks of 64 (128 B), 128B swizzle
constexpr int kQTmemRegions = 4;                   // features 0..255 live in TMEM
constexpr int kQRegion = kHeads * 128;             // 16 KB
constexpr int kQBytes = (kRegions - kQTmemRegions) * kQRegion;   // 80 KB: features 256..575
constexpr int kKvRegion = kKeys * 128;             // 8 KB
constexpr int kStageBytes = kRegions * kKvRegion;  // 72 KB
constexpr int kStages = 2;
constexpr int kOffQ = 0;
constexpr int kOffKV = kOffQ + kQBytes;
constexpr int kOffBar = kOffKV + kStages * kStageBytes;
constexpr int kSmemBytes = 1024 + kOffBar + 256;
constexpr int kSoftmaxWarps = 4, kMmaWarp = 4, kGatherWarp = 5, kGatherWarps = 4;
constexpr int kMlaThreads = (kSoftmaxWarps + 1 + kGatherWarps) * 32;
constexpr int kMaxSlots = 2048;                    // selected slots per CTA (split chunk cap)
constexpr int kTmemCols = 512;
constexpr uint32_t kTmemO = 0, kTmemS = 256, kTmemQ = 384;   // S: two 64-column buffers
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRescaleThreshold = 8.0f;          // log2 units

struct MlaSplit {
  int nsplit;
  int chunk;     // selected slots per split (multiple of kKeys, at most kMaxSlots)
};

MlaSplit choose_split(int64_t BT, int k, int sms) {
  MlaSplit s;
  const int64_t ctas_per_split = BT * 2;
  int n = (int)std::max<int64_t>(1, (sms + ctas_per_split - 1) / ctas_per_split);
  const int max_split = std::max(1, (k + 63) / 64);
  n = std::min(n, max_split);
  int chunk = (k + n - 1) / n;
  chunk = (chunk + 63) / 64 * 64;
  chunk = std::min(chunk, kMaxSlots);
  s.chunk = chunk;
  s.nsplit = (k + chunk - 1) / chunk;
  return s;
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
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
  int nsplit, chunk;
  float scale_log2;          // softmax_scale * log2(e)
  uint16_t* out;
  float* lse;
  float* part_o;             // [BT][nsplit][128][512]   (nsplit > 1)
  float* part_ml;            // [BT][nsplit][128][2]     running max (log2 domain), sum
  int* status;
};

__global__ void __launch_bounds__(kMlaThreads, 1)
    sparse_mla_kernel(const __grid_constant__ CUtensorMap q_map, const __grid_constant__ CUtensorMap kv_map,
                      const MlaParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* q_sm = smem + kOffQ;
  uint8_t* kv_sm = smem + kOffKV;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kOffBar);
  uint64_t* kv_full = bars;                    // [kStages] gather (cp.async) -> MMA
  uint64_t* kv_empty = bars + kStages;         // [kStages] MMA (after P V) -> gather
  uint64_t* s_full = bars + 2 * kStages;       // [2] MMA -> softmax (per score buffer)
  uint64_t* q_full = s_full + 2;               // TMA (Q in smem) + softmax (Q in TMEM) -> MMA
  uint64_t* p_full = s_full + 3;               // softmax (P in TMEM) -> MMA
  uint64_t* p_empty = s_full + 4;              // MMA (P V done) -> softmax (O rescale only)
  uint64_t* o_full = s_full + 5;               // MMA -> softmax (all P V done)
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_flag;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int half = blockIdx.x & 1;             // output features [256*half, 256*half + 256)
  const int unit = blockIdx.x >> 1;
  const int split = unit % p.nsplit;
  const int64_t bt = unit / p.nsplit;
  const int b = (int)(bt / p.T);
  const int slot0 = split * p.chunk;
  const int nslots = max(0, min(p.k, slot0 + p.chunk) - slot0);
  const int ntiles = (nslots + kKeys - 1) / kKeys;
  const int32_t* idx_row = p.idx + bt * p.k + slot0;

  if (tid == 0) {
    abort_flag = 0;
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&kv_full[s], kGatherWarps * 32);
      mbar_init(&kv_empty[s], 1);
    }
    mbar_init(&s_full[0], 1);
    mbar_init(&s_full[1], 1);
    mbar_init(q_full, 1 + kSoftmaxWarps * 32);
    mbar_init(p_full, kSoftmaxWarps * 32);
    mbar_init(p_empty, 1);
    mbar_init(o_full, 1);
    fence_barrier_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(&tmem_base_sh, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_sh;

  if (warp >= kGatherWarp) {
    // ------------------------------------------------------------------ gather warps
    // gather warp w copies keys 16w..16w+15 of each tile; per key, lanes take 16-byte chunks
    // lane, lane+32, lane+64 of the 72 in the row (contiguous 512-byte warp requests)
    const int w = warp - kGatherWarp;
    if (w == 0 && lane == 0 && ntiles > 0) {
      prefetch_tensormap(&q_map);
      mbar_arrive_expect_tx(q_full, kQBytes);
      for (int r = kQTmemRegions; r < kRegions; ++r)
        tma_load_2d(q_sm + (r - kQTmemRegions) * kQRegion, &q_map, q_full, 64 * r, (int32_t)(bt * kHeads));
    }
    const uint16_t* kv_b = p.kv + (int64_t)b * p.S_max * kDqk;
    auto load_idx = [&](int j) -> int {
      const int slot = j * kKeys + 16 * w + (lane & 15);
      return (j < ntiles && slot < nslots) ? __ldg(idx_row + slot) : -1;
    };
    int idx_next = load_idx(0);
    for (int j = 0; j < ntiles; ++j) {
      const int s = j % kStages;
      const int idx_cur = idx_next;
      idx_next = load_idx(j + 1);                     // one tile ahead
      if (lane < 16 && idx_cur >= p.S_max) set_status(p.status, DSA_ERR_DEVICE_BOUNDS);
      if (j >= kStages &&
          !__all_sync(0xffffffffu, mbar_wait(&kv_empty[s], ((j / kStages) + 1) & 1, &abort_flag, p.status, DSA_SITE_MLA_KV_EMPTY)))
        break;
      const uint32_t base = smem_u32(kv_sm + s * kStageBytes);
#pragma unroll 4
      for (int kk = 0; kk < 16; ++kk) {
        const int v = __shfl_sync(0xffffffffu, idx_cur, kk);
        const bool ok = v >= 0 && v < p.S_max;
        const int key = 16 * w + kk;
        const uint16_t* src = kv_b + (int64_t)(ok ? v : 0) * kDqk;
#pragma unroll
        for (int i = 0; i < 3; ++i) {
          const int c = lane + 32 * i;
          if (c < 72)
            cp_async_16_zfill(base + (c >> 3) * kKvRegion + sw128(key, c & 7), src + c * 8, ok);
        }
      }
      cp_async_mbar_arrive(&kv_full[s]);
    }
    cp_async_wait_all();
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0 && ntiles > 0) {
      constexpr uint32_t idesc_s = idesc_f32acc(1 /*BF16*/, 1, 128, kKeys, 0, 0);
      constexpr uint32_t idesc_pv = idesc_f32acc(1, 1, 128, 256, 0, 1 /*B MN-major*/);
      const uint32_t q_base = smem_u32(q_sm);
      bool ok = mbar_wait(q_full, 0, &abort_flag, p.status, DSA_SITE_MLA_Q);
      auto issue_s = [&](int j) -> bool {     // Q K^T of tile j into score buffer j & 1
        if (!mbar_wait(&kv_full[j % kStages], (j / kStages) & 1, &abort_flag, p.status, DSA_SITE_MLA_KV_FULL)) return false;
        fence_proxy_async_smem();        // cp.async (generic proxy) writes -> MMA (async proxy) reads
        tc_fence_after();
        const uint32_t kv_base = smem_u32(kv_sm + (j % kStages) * kStageBytes);
        const uint32_t d = tmem + kTmemS + (j & 1) * kKeys;
#pragma unroll
        for (int ks = 0; ks < 4 * kQTmemRegions; ++ks)          // Q from TMEM
          mma_f16_ts(d, tmem + kTmemQ + ks * 8,
                     sdesc_kmajor_sw128(kv_base + (ks >> 2) * kKvRegion + (ks & 3) * 32), idesc_s, ks > 0 ? 1u : 0u);
#pragma unroll
        for (int ks = 4 * kQTmemRegions; ks < kDqk / 16; ++ks)  // Q from shared memory
          mma_f16_ss(d, sdesc_kmajor_sw128(q_base + ((ks >> 2) - kQTmemRegions) * kQRegion + (ks & 3) * 32),
                     sdesc_kmajor_sw128(kv_base + (ks >> 2) * kKvRegion + (ks & 3) * 32), idesc_s, 1u);
        mma_commit(&s_full[j & 1]);
        return true;
      };
      auto issue_pv = [&](int j) -> bool {    // P V of tile j (P in score buffer j & 1)
        if (!mbar_wait(p_full, j & 1, &abort_flag, p.status, DSA_SITE_MLA_P_FULL)) return false;
        tc_fence_after();
        const uint32_t v_base = smem_u32(kv_sm + (j % kStages) * kStageBytes) + 4 * half * kKvRegion;
#pragma unroll
        for (int kk = 0; kk < kKeys / 16; ++kk)
          mma_f16_ts(tmem + kTmemO, tmem + kTmemS + (j & 1) * kKeys + kk * 8,
                     sdesc_mnmajor_sw128(v_base + kk * 2048, kKvRegion, 1024), idesc_pv,
                     (j > 0 || kk > 0) ? 1u : 0u);
        mma_commit(p_empty);
        mma_commit(&kv_empty[j % kStages]);
        return true;
      };
      if (ok) ok = issue_s(0);
      if (ok && ntiles > 1) ok = issue_s(1);
      for (int j = 0; ok && j < ntiles; ++j) {
        ok = issue_pv(j);
        if (ok && j + 2 < ntiles) ok = issue_s(j + 2);
      }
      mma_commit(o_full);
    }
  } else {
    // ------------------------------------------------------------------ softmax warps (thread = head)
    const int h = tid;
    const uint32_t t_row = tmem + ((uint32_t)(warp * 32) << 16);
    // Q features 0..255 of head h -> TMEM as bf16 pairs (feature f in column f/2)
    if (ntiles > 0) {
      const uint4* qrow = reinterpret_cast<const uint4*>(p.q + (bt * kHeads + h) * kDqk);
      uint32_t buf[128];
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        const uint4 v = __ldg(qrow + i);
        buf[4 * i] = v.x; buf[4 * i + 1] = v.y; buf[4 * i + 2] = v.z; buf[4 * i + 3] = v.w;
      }
#pragma unroll
      for (int c = 0; c < 4; ++c) tmem_st32(t_row + kTmemQ + c * 32, *reinterpret_cast<uint32_t(*)[32]>(buf + 32 * c));
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(q_full);
    }
    float m = -INFINITY, l = 0.f;
    bool ok = true;
#pragma unroll 1
    for (int j = 0; ok && j < ntiles; ++j) {
      const uint32_t s_col = kTmemS + (j & 1) * kKeys;
      if (!__all_sync(0xffffffffu, mbar_wait(&s_full[j & 1], (j >> 1) & 1, &abort_flag, p.status, DSA_SITE_MLA_S_FULL))) { ok = false; break; }
      tc_fence_after();
      uint32_t r0[32], r1[32];
      tmem_ld32(t_row + s_col, r0);
      tmem_ld32(t_row + s_col + 32, r1);
      const int sa = j * kKeys + lane, sb = sa + 32;
      const int va = sa < nslots ? __ldg(idx_row + sa) : -1;
      const int vb = sb < nslots ? __ldg(idx_row + sb) : -1;
      const uint32_t vlo = __ballot_sync(0xffffffffu, va >= 0 && va < p.S_max);
      const uint32_t vhi = __ballot_sync(0xffffffffu, vb >= 0 && vb < p.S_max);
      tmem_ld_wait();
      float z[kKeys];
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        z[i] = ((vlo >> i) & 1u) ? __uint_as_float(r0[i]) * p.scale_log2 : -INFINITY;
        z[32 + i] = ((vhi >> i) & 1u) ? __uint_as_float(r1[i]) * p.scale_log2 : -INFINITY;
      }
      float t8[8];
#pragma unroll
      for (int g = 0; g < 8; ++g)
        t8[g] = fmaxf(fmaxf(fmaxf(z[8 * g], z[8 * g + 1]), fmaxf(z[8 * g + 2], z[8 * g + 3])),
                      fmaxf(fmaxf(z[8 * g + 4], z[8 * g + 5]), fmaxf(z[8 * g + 6], z[8 * g + 7])));
      const float mx = fmaxf(fmaxf(fmaxf(t8[0], t8[1]), fmaxf(t8[2], t8[3])), fmaxf(fmaxf(t8[4], t8[5]), fmaxf(t8[6], t8[7])));
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
      // O rescale: every P V issued so far (tiles < j) must be done first
      const bool rescale = (m != -INFINITY) && (m_new != m);
      if (__any_sync(0xffffffffu, rescale)) {
        if (j >= 1 && !__all_sync(0xffffffffu, mbar_wait(p_empty, (j - 1) & 1, &abort_flag, p.status, DSA_SITE_MLA_P_EMPTY))) {
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
      tmem_st32(t_row + s_col, pk);              // P over the scores it came from
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(p_full);
    }
    // ---- epilogue: O row (this CTA's 256 output features) / l
    const bool have_o = ntiles > 0 && ok &&
                        __all_sync(0xffffffffu, mbar_wait(o_full, 0, &abort_flag, p.status, DSA_SITE_MLA_O_FULL));
    if (have_o) tc_fence_after();
    const float inv = l > 0.f ? 1.f / l : 0.f;
    if (p.nsplit == 1) {
      uint16_t* dst = p.out + (bt * kHeads + h) * kDv + 256 * half;
#pragma unroll 1
      for (int c = 0; c < 8; ++c) {
        uint32_t o[32];
        if (have_o) {
          tmem_ld32(t_row + kTmemO + c * 32, o);
          tmem_ld_wait();
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] = 0u;
        }
        uint4* d4 = reinterpret_cast<uint4*>(dst + c * 32);
#pragma unroll
        for (int i = 0; i < 4; ++i)
          d4[i] = make_uint4(pack_bf16(__uint_as_float(o[8 * i]) * inv, __uint_as_float(o[8 * i + 1]) * inv),
                             pack_bf16(__uint_as_float(o[8 * i + 2]) * inv, __uint_as_float(o[8 * i + 3]) * inv),
                             pack_bf16(__uint_as_float(o[8 * i + 4]) * inv, __uint_as_float(o[8 * i + 5]) * inv),
                             pack_bf16(__uint_as_float(o[8 * i + 6]) * inv, __uint_as_float(o[8 * i + 7]) * inv));
      }
      if (p.lse && half == 0)
        p.lse[bt * kHeads + h] = l > 0.f ? (m + log2f(l)) * 0.6931471805599453f : -INFINITY;
    } else {
      const int64_t prow = (bt * p.nsplit + split) * kHeads + h;
      float* dst = p.part_o + prow * kDv + 256 * half;
#pragma unroll 1
      for (int c = 0; c < 8; ++c) {
        uint32_t o[32];
        if (have_o) {
          tmem_ld32(t_row + kTmemO + c * 32, o);
          tmem_ld_wait();
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] = 0u;
        }
        float4* d4 = reinterpret_cast<float4*>(dst + c * 32);
#pragma unroll
        for (int i = 0; i < 8; ++i)
          d4[i] = make_float4(__uint_as_float(o[4 * i]), __uint_as_float(o[4 * i + 1]),
                              __uint_as_float(o[4 * i + 2]), __uint_as_float(o[4 * i + 3]));
      }
      if (half == 0) *reinterpret_cast<float2*>(p.part_ml + prow * 2) = make_float2(m, l);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// Merge the key-split partials: one warp per (query, head), 16 output features per lane.
__global__ void __launch_bounds__(256) sparse_mla_combine_kernel(const MlaParams p, int64_t rows) {
  const int64_t wid = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (wid >= rows) return;
  const int64_t bt = wid / kHeads;
  const int head = (int)(wid - bt * kHeads);
  float m_all = -INFINITY;
  for (int s = 0; s < p.nsplit; ++s) {
    const float m = p.part_ml[((bt * p.nsplit + s) * kHeads + head) * 2];
    m_all = fmaxf(m_all, m);
  }
  float acc[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) acc[i] = 0.f;
  float l_all = 0.f;
  for (int s = 0; s < p.nsplit; ++s) {
    const int64_t prow = (bt * p.nsplit + s) * kHeads + head;
    const float2 ml = *reinterpret_cast<const float2*>(p.part_ml + prow * 2);
    if (ml.x == -INFINITY) continue;
    const float wgt = exp2f(ml.x - m_all);
    l_all += ml.y * wgt;
    const float4* src = reinterpret_cast<const float4*>(p.part_o + prow * kDv + lane * 16);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float4 v = src[i];
      acc[4 * i] += v.x * wgt; acc[4 * i + 1] += v.y * wgt;
      acc[4 * i + 2] += v.z * wgt; acc[4 * i + 3] += v.w * wgt;
    }
  }
  const float inv = l_all > 0.f ? 1.f / l_all : 0.f;
  uint32_t packed[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) packed[i] = pack_bf16(acc[2 * i] * inv, acc[2 * i + 1] * inv);
  uint4* dst = reinterpret_cast<uint4*>(p.out + (bt * kHeads + head) * kDv + lane * 16);
  dst[0] = make_uint4(packed[0], packed[1], packed[2], packed[3]);
  dst[1] = make_uint4(packed[4], packed[5], packed[6], packed[7]);
  if (p.lse && lane == 0)
    p.lse[bt * kHeads + head] = l_all > 0.f ? (m_all + log2f(l_all)) * 0.6931471805599453f : -INFINITY;
}

size_t sparse_mla_workspace_size(int B, int T, int k) {
  const int64_t BT = (int64_t)B * T;
  const MlaSplit s = choose_split(BT, k, dsa_host::device_sm_count());
  if (s.nsplit <= 1) return 0;
  return (size_t)BT * s.nsplit * kHeads * (kDv + 2) * sizeof(float);
}

int launch_sparse_mla(const uint16_t* q, const uint16_t* kv, const int32_t* idx, int B, int T,
                      int S_max, int k, float softmax_scale, uint16_t* out, float* lse,
                      void* workspace, size_t ws_bytes, cudaStream_t stream, int* status) {
  const int64_t BT = (int64_t)B * T;
  if (BT == 0) return DSA_OK;
  const MlaSplit s = choose_split(BT, k, dsa_host::device_sm_count());
  MlaParams p{};
  p.q = q; p.kv = kv; p.idx = idx; p.B = B; p.T = T; p.S_max = S_max; p.k = k;
  p.nsplit = s.nsplit; p.chunk = s.chunk;
  p.scale_log2 = softmax_scale * kLog2e;
  p.out = out; p.lse = lse; p.status = status;
  if (s.nsplit > 1) {
    const size_t need = (size_t)BT * s.nsplit * kHeads * (kDv + 2) * sizeof(float);
    if (workspace == nullptr || ws_bytes < need) return DSA_ERR_WORKSPACE;
    p.part_o = static_cast<float*>(workspace);
    p.part_ml = p.part_o + (size_t)BT * s.nsplit * kHeads * kDv;
  }
  static bool configured[64] = {false};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 64 && !configured[dev]) {
    if (cudaFuncSetAttribute(sparse_mla_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes) !=
        cudaSuccess)
      return DSA_ERR_CUDA;
    configured[dev] = true;
  }
  const int64_t grid = BT * s.nsplit * 2;          // two CTAs (output-feature halves) per (query, split)
  if (grid > 0x7fffffff) return DSA_ERR_INVALID_ARG;
  CUtensorMap q_map, kv_map;
  if (!dsa_host::encode_tensor_map_2d(&q_map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, (void*)q, kDqk,
                                      (uint64_t)BT * kHeads, kDqk * 2, 64, kHeads, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !dsa_host::encode_tensor_map_2d(&kv_map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, (void*)kv, kDqk,
                                      (uint64_t)B * S_max, kDqk * 2, 64, 1, CU_TENSOR_MAP_SWIZZLE_128B))
    return DSA_ERR_CUDA;
  sparse_mla_kernel<<<(unsigned)grid, kMlaThreads, kSmemBytes, stream>>>(q_map, kv_map, p);
  int rc = dsa_host::check_launch();
  if (rc != DSA_OK || s.nsplit == 1) return rc;
  const int64_t rows = BT * kHeads;
  sparse_mla_combine_kernel<<<(unsigned)((rows + 7) / 8), 256, 0, stream>>>(p, rows);
  return dsa_host::check_launch();
}

}  // namespace dsa
