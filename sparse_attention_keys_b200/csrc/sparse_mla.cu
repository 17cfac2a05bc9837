// dsa_sparse_mla: sparse MQA-style latent attention over the selected positions.
//
// For each (b, t, head h): z_u = scale * q[h] . kv[idx_u] over the 576 features (512 latent +
// 64 rotary), p = softmax over the selected u, out[h] = sum_u p_u kv[idx_u][0:512]. This is the
// absorbed MQA decode of "DeepSeek-V3.2-Exp - Similarities" (model.py 590-606 excerpt: latent and
// rotary score terms, index mask, softmax, latent-weighted sum) with the index mask replaced by a
// gather of the selected rows, and the sparse-attention steps of the dense-block page
// (S' = S m^2/sqrt 192, A = softmax, O = AV).
//
// CTA = (query, key split, half of the 128 heads): eight warps; warps 0-3 own 16 heads each and
// output features 0..255, warps 4-7 the same heads and features 256..511. Selected latent rows
// are gathered with 16-byte cp.async into a 3-stage shared-memory ring (32 rows per stage), the
// scores and P.V run on bf16 tensor-core tiles (m16n8k16) with an fp32 online softmax in
// registers. With several key splits per query, fp32 partials (O, running max, running sum) go to
// the caller's workspace and a second kernel merges them.
#include <cuda_bf16.h>

#include <algorithm>

#include "common.cuh"
#include "kernels.h"

namespace dsa {

namespace {

constexpr int kHeads = 128;
constexpr int kDqk = 576;
constexpr int kDv = 512;
constexpr int kHeadsPerCta = 64;
constexpr int kKeysPerStage = 32;
constexpr int kStages = 3;
constexpr int kRowBytes = kDqk * 2 + 16;                  // padded: conflict-free ldmatrix
constexpr int kQBytes = kHeadsPerCta * kRowBytes;
constexpr int kStageBytes = kKeysPerStage * kRowBytes;
constexpr int kMlaThreads = 256;
constexpr int kSmemBytes = kQBytes + kStages * kStageBytes + kStages * kKeysPerStage * 4;
constexpr float kLog2e = 1.4426950408889634f;

struct MlaSplit {
  int nsplit;
  int chunk;     // selected slots per split (multiple of kKeysPerStage)
};

MlaSplit choose_split(int64_t BT, int k, int sms) {
  MlaSplit s;
  const int64_t ctas_per_split = BT * (kHeads / kHeadsPerCta);
  int n = (int)std::max<int64_t>(1, (sms + ctas_per_split - 1) / ctas_per_split);
  const int max_split = std::max(1, (k + 63) / 64);
  n = std::min(n, max_split);
  int chunk = (k + n - 1) / n;
  chunk = (chunk + kKeysPerStage - 1) / kKeysPerStage * kKeysPerStage;
  s.chunk = chunk;
  s.nsplit = (k + chunk - 1) / chunk;
  return s;
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                               uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

}  // namespace

struct MlaParams {
  const uint16_t* q;
  const uint16_t* kv;
  const int32_t* idx;
  int T, S_max, k;
  int nsplit, chunk;
  float scale_log2;          // softmax_scale * log2(e)
  uint16_t* out;
  float* lse;
  float* part_o;             // [BT][nsplit][128][512]   (nsplit > 1)
  float* part_ml;            // [BT][nsplit][128][2]     running max (log2 domain), sum
  int* status;
};

__global__ void __launch_bounds__(kMlaThreads, 1) sparse_mla_kernel(const MlaParams p) {
  extern __shared__ __align__(16) uint8_t smem[];
  uint8_t* q_sm = smem;
  uint8_t* kv_sm = smem + kQBytes;
  int32_t* slot_idx = reinterpret_cast<int32_t*>(smem + kQBytes + kStages * kStageBytes);  // [stage][32]

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int hh = blockIdx.x & 1;                      // head half
  const int split = (blockIdx.x >> 1) % p.nsplit;
  const int64_t bt = (blockIdx.x >> 1) / p.nsplit;
  const int b = (int)(bt / p.T);
  const int slot0 = split * p.chunk;
  const int nslots = max(0, min(p.k, slot0 + p.chunk) - slot0);
  const int nstages_total = (nslots + kKeysPerStage - 1) / kKeysPerStage;
  const int32_t* idx_row = p.idx + bt * p.k + slot0;
  const uint16_t* kv_b = p.kv + (int64_t)b * p.S_max * kDqk;

  // Q: 64 heads x 576 bf16 into padded rows (72 chunks of 16 B per row)
  {
    const uint16_t* qsrc = p.q + (bt * kHeads + hh * kHeadsPerCta) * kDqk;
    for (int c = tid; c < kHeadsPerCta * 72; c += kMlaThreads) {
      const int r = c / 72, ch = c - r * 72;
      cp_async_16(smem_u32(q_sm + r * kRowBytes + ch * 16), qsrc + r * kDqk + ch * 8);
    }
  }
  auto load_stage = [&](int st, int buf) {
    const int base = st * kKeysPerStage;
    if (tid < kKeysPerStage) {
      int v = -1;
      if (base + tid < nslots) {
        v = idx_row[base + tid];
        if (v >= p.S_max) { set_status(p.status, DSA_ERR_DEVICE_BOUNDS); v = -1; }
        if (v < -1) v = -1;
      }
      slot_idx[buf * kKeysPerStage + tid] = v;
    }
    // each of the 32 rows is 72 chunks; rows with idx -1 are zero-filled
    uint8_t* dst = kv_sm + buf * kStageBytes;
    for (int c = tid; c < kKeysPerStage * 72; c += kMlaThreads) {
      const int r = c / 72, ch = c - r * 72;
      const int slot = base + r;
      int v = slot < nslots ? idx_row[slot] : -1;
      const bool ok = v >= 0 && v < p.S_max;
      cp_async_16_zfill(smem_u32(dst + r * kRowBytes + ch * 16), kv_b + (int64_t)(ok ? v : 0) * kDqk + ch * 8, ok);
    }
  };

  for (int s = 0; s < kStages - 1; ++s) {
    if (s < nstages_total) load_stage(s, s);
    cp_async_commit();
  }

  const int wq = warp & 3;            // head group of 16 within the CTA's 64
  const int vhalf = warp >> 2;        // output features [vhalf*256, +256)
  float o[32][4];
#pragma unroll
  for (int j = 0; j < 32; ++j) o[j][0] = o[j][1] = o[j][2] = o[j][3] = 0.f;
  float m_r[2] = {-INFINITY, -INFINITY};   // rows lane/4 and lane/4+8, log2 domain
  float l_r[2] = {0.f, 0.f};

  const uint32_t q_base = smem_u32(q_sm) + (wq * 16) * kRowBytes;
  // ldmatrix lane addressing
  const int a_row = (lane & 7) + ((lane >> 3) & 1) * 8, a_col = (lane >> 4) * 8;
  const int b_key = (lane & 7) + (lane >> 4) * 8, b_col = ((lane >> 3) & 1) * 8;
  const int v_key = (lane & 7) + ((lane >> 3) & 1) * 8, v_col = (lane >> 4) * 8;

  for (int st = 0; st < nstages_total; ++st) {
    const int buf = st % kStages;
    if (st + kStages - 1 < nstages_total) load_stage(st + kStages - 1, (st + kStages - 1) % kStages);
    cp_async_commit();
    cp_async_wait<kStages - 1>();
    __syncthreads();

    const uint32_t kv_base = smem_u32(kv_sm + buf * kStageBytes);
    // S = Q K^T: 16 heads x 32 keys
    float s[4][4];
#pragma unroll
    for (int j = 0; j < 4; ++j) s[j][0] = s[j][1] = s[j][2] = s[j][3] = 0.f;
#pragma unroll 4
    for (int kk = 0; kk < kDqk / 16; ++kk) {
      uint32_t a0, a1, a2, a3;
      ldsm_x4(q_base + a_row * kRowBytes + (kk * 16 + a_col) * 2, a0, a1, a2, a3);
#pragma unroll
      for (int jp = 0; jp < 2; ++jp) {
        uint32_t b0, b1, b2, b3;
        ldsm_x4(kv_base + (jp * 16 + b_key) * kRowBytes + (kk * 16 + b_col) * 2, b0, b1, b2, b3);
        mma_bf16_16816(s[2 * jp], a0, a1, a2, a3, b0, b1);
        mma_bf16_16816(s[2 * jp + 1], a0, a1, a2, a3, b2, b3);
      }
    }
    // mask, online softmax (base 2)
    const int32_t* sidx = slot_idx + buf * kKeysPerStage;
    float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int key = j * 8 + (lane & 3) * 2 + (e & 1);
        const float z = sidx[key] >= 0 ? s[j][e] * p.scale_log2 : -INFINITY;
        s[j][e] = z;
        mx[e >> 1] = fmaxf(mx[e >> 1], z);
      }
    }
    float alpha[2];
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      mx[r] = fmaxf(mx[r], __shfl_xor_sync(0xffffffffu, mx[r], 1));
      mx[r] = fmaxf(mx[r], __shfl_xor_sync(0xffffffffu, mx[r], 2));
      const float m_new = fmaxf(m_r[r], mx[r]);
      alpha[r] = (m_new == -INFINITY) ? 1.f : exp2f(m_r[r] - m_new);
      m_r[r] = m_new;
    }
    float rs[2] = {0.f, 0.f};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float m = m_r[e >> 1];
        const float pv = (m == -INFINITY) ? 0.f : exp2f(s[j][e] - m);
        s[j][e] = pv;
        rs[e >> 1] += pv;
      }
    }
#pragma unroll
    for (int r = 0; r < 2; ++r) l_r[r] = l_r[r] * alpha[r] + rs[r];
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      o[j][0] *= alpha[0]; o[j][1] *= alpha[0];
      o[j][2] *= alpha[1]; o[j][3] *= alpha[1];
    }
    // O += P V over this stage's 32 keys (two k16 steps)
#pragma unroll
    for (int ks = 0; ks < 2; ++ks) {
      const uint32_t a0 = pack_bf16(s[2 * ks][0], s[2 * ks][1]);
      const uint32_t a1 = pack_bf16(s[2 * ks][2], s[2 * ks][3]);
      const uint32_t a2 = pack_bf16(s[2 * ks + 1][0], s[2 * ks + 1][1]);
      const uint32_t a3 = pack_bf16(s[2 * ks + 1][2], s[2 * ks + 1][3]);
#pragma unroll
      for (int jp = 0; jp < 16; ++jp) {
        uint32_t b0, b1, b2, b3;
        const int col = vhalf * 256 + jp * 16 + v_col;
        ldsm_x4_t(kv_base + (ks * 16 + v_key) * kRowBytes + col * 2, b0, b1, b2, b3);
        mma_bf16_16816(o[2 * jp], a0, a1, a2, a3, b0, b1);
        mma_bf16_16816(o[2 * jp + 1], a0, a1, a2, a3, b2, b3);
      }
    }
    __syncthreads();     // this buffer is refilled by the next iteration's prefetch
  }
  cp_async_wait<0>();

  // finish: full row sums across the quad
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    l_r[r] += __shfl_xor_sync(0xffffffffu, l_r[r], 1);
    l_r[r] += __shfl_xor_sync(0xffffffffu, l_r[r], 2);
  }
  const int head0 = hh * kHeadsPerCta + wq * 16 + (lane >> 2);
  if (p.nsplit == 1) {
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      const int head = head0 + r * 8;
      const float inv = l_r[r] > 0.f ? 1.f / l_r[r] : 0.f;
      uint16_t* dst = p.out + (bt * kHeads + head) * kDv + vhalf * 256;
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        const int col = j * 8 + (lane & 3) * 2;
        *reinterpret_cast<uint32_t*>(dst + col) = pack_bf16(o[j][2 * r] * inv, o[j][2 * r + 1] * inv);
      }
      if (p.lse && vhalf == 0 && (lane & 3) == 0)
        p.lse[bt * kHeads + head] = l_r[r] > 0.f ? (m_r[r] + log2f(l_r[r])) * 0.6931471805599453f : -INFINITY;
    }
  } else {
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      const int head = head0 + r * 8;
      const int64_t prow = (bt * p.nsplit + split) * kHeads + head;
      float* dst = p.part_o + prow * kDv + vhalf * 256;
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        const int col = j * 8 + (lane & 3) * 2;
        *reinterpret_cast<float2*>(dst + col) = make_float2(o[j][2 * r], o[j][2 * r + 1]);
      }
      if (vhalf == 0 && (lane & 3) == 0)
        *reinterpret_cast<float2*>(p.part_ml + prow * 2) = make_float2(m_r[r], l_r[r]);
    }
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
  p.q = q; p.kv = kv; p.idx = idx; p.T = T; p.S_max = S_max; p.k = k;
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
  const int64_t grid = BT * s.nsplit * (kHeads / kHeadsPerCta);
  if (grid > 0x7fffffff) return DSA_ERR_INVALID_ARG;
  sparse_mla_kernel<<<(unsigned)grid, kMlaThreads, kSmemBytes, stream>>>(p);
  int rc = dsa_host::check_launch();
  if (rc != DSA_OK || s.nsplit == 1) return rc;
  const int64_t rows = BT * kHeads;
  sparse_mla_combine_kernel<<<(unsigned)((rows + 7) / 8), 256, 0, stream>>>(p, rows);
  return dsa_host::check_launch();
}

}  // namespace dsa
