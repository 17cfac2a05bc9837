// dsa_topk: per-query top-k of the index scores over the visible (causal) positions.
//
// Restates index_score.topk(min(index_topk, end_pos)) after the mask add in Indexer.forward
// ("DeepSeek-V3.2-Exp - Rotate first features", Indexer.forward excerpt) and top_2048 of the
// lightning-indexer steps (dense-block page). Ties go to the smaller position; the selection
// is written in ascending position order, then -1 padding.
//
// One CTA per score row. The row's visible scores are staged once into shared memory as
// order-preserving 32-bit keys (coalesced 16-byte loads), then a 3-pass radix select (12, 10,
// 10 bits) finds the k-th largest key with shared-memory histograms, and a warp-ballot
// compaction writes the selected positions in order. HBM-bound: 4 B read per visible score,
// 4 B written per selected index.
#include "common.cuh"
#include "kernels.h"

namespace dsa {

namespace {

constexpr int kTopkThreads = 512;
constexpr int kTopkWarps = kTopkThreads / 32;
constexpr int kHistBins = 4096;

// Larger float -> larger key; -0.0 is folded onto +0.0 so the two compare equal.
__device__ __forceinline__ uint32_t order_key(float f) {
  uint32_t u = __float_as_uint(f);
  if ((u << 1) == 0) u = 0;
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Inclusive scan of one value per thread across the CTA (kTopkThreads threads).
__device__ __forceinline__ uint32_t block_inclusive_scan(uint32_t v, uint32_t* warp_tot) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int d = 1; d < 32; d <<= 1) {
    const uint32_t o = __shfl_up_sync(0xffffffffu, v, d);
    if (lane >= d) v += o;
  }
  if (lane == 31) warp_tot[warp] = v;
  __syncthreads();
  if (warp == 0) {
    uint32_t t = lane < kTopkWarps ? warp_tot[lane] : 0;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
      const uint32_t o = __shfl_up_sync(0xffffffffu, t, d);
      if (lane >= d) t += o;
    }
    if (lane < kTopkWarps) warp_tot[lane] = t;   // inclusive totals per warp
  }
  __syncthreads();
  const uint32_t before = warp > 0 ? warp_tot[warp - 1] : 0;
  __syncthreads();
  return v + before;
}

}  // namespace

__global__ void __launch_bounds__(kTopkThreads) topk_kernel(const float* __restrict__ scores,
                                                            int64_t ld,
                                                            const int32_t* __restrict__ q_pos,
                                                            const int32_t* __restrict__ kv_len,
                                                            int T, int k, int max_row,
                                                            int32_t* __restrict__ idx,
                                                            int* status) {
  extern __shared__ __align__(16) uint32_t smem[];
  uint32_t* hist = smem;                       // kHistBins
  uint32_t* keys = smem + kHistBins;           // max_row
  __shared__ uint32_t warp_tot[kTopkWarps];
  __shared__ uint32_t sel_digit, sel_remaining;

  const int64_t row = blockIdx.x;
  const int b = (int)(row / T);
  const int tid = threadIdx.x;
  int32_t* out = idx + row * (int64_t)k;
  int n = min(q_pos[row] + 1, kv_len[b]);
  if (n < 0) n = 0;

  if (n <= k) {   // everything visible is selected
    for (int i = tid; i < k; i += kTopkThreads) out[i] = i < n ? i : -1;
    return;
  }
  if (n > max_row) {
    if (tid == 0) set_status(status, DSA_ERR_DEVICE_BOUNDS);
    for (int i = tid; i < k; i += kTopkThreads) out[i] = -1;
    return;
  }

  // Stage the visible scores as keys.
  const float* src = scores + row * ld;
  const int n4 = n >> 2;
  for (int i = tid; i < n4; i += kTopkThreads) {
    const float4 f = reinterpret_cast<const float4*>(src)[i];
    reinterpret_cast<uint4*>(keys)[i] = make_uint4(order_key(f.x), order_key(f.y), order_key(f.z), order_key(f.w));
  }
  for (int i = (n4 << 2) + tid; i < n; i += kTopkThreads) keys[i] = order_key(src[i]);

  // Radix select of the k-th largest key: digits of 12, 10 and 10 bits from the top.
  uint32_t prefix = 0, prefix_mask = 0, remaining = (uint32_t)k;
#pragma unroll 1
  for (int pass = 0; pass < 3; ++pass) {
    const int shift = pass == 0 ? 20 : (pass == 1 ? 10 : 0);
    const int nb = pass == 0 ? 4096 : 1024;
    for (int i = tid; i < nb; i += kTopkThreads) hist[i] = 0;
    __syncthreads();
    for (int i = tid; i < n; i += kTopkThreads) {
      const uint32_t key = keys[i];
      if ((key & prefix_mask) == prefix) atomicAdd(&hist[(key >> shift) & (nb - 1)], 1u);
    }
    __syncthreads();
    // thread t owns bins nb-1-t*c .. nb-(t+1)*c (descending); c = nb / threads
    const int c = nb / kTopkThreads;
    uint32_t local = 0;
    for (int j = 0; j < c; ++j) local += hist[nb - 1 - tid * c - j];
    const uint32_t incl = block_inclusive_scan(local, warp_tot);
    uint32_t before = incl - local;
    if (before < remaining && remaining <= incl) {
      for (int j = 0; j < c; ++j) {
        const int bin = nb - 1 - tid * c - j;
        const uint32_t h = hist[bin];
        if (before + h >= remaining) {
          sel_digit = (uint32_t)bin;
          sel_remaining = remaining - before;
          break;
        }
        before += h;
      }
    }
    __syncthreads();
    prefix |= sel_digit << shift;
    prefix_mask |= (uint32_t)(nb - 1) << shift;
    remaining = sel_remaining;
    __syncthreads();
  }
  const uint32_t thr = prefix;           // the k-th largest key
  const uint32_t need_eq = remaining;    // how many keys equal to thr are selected

  // Compaction in ascending position order. Warp w owns a contiguous chunk.
  const int warp = tid >> 5, lane = tid & 31;
  const int chunk = ((n + kTopkWarps - 1) / kTopkWarps + 31) & ~31;
  const int beg = min(n, warp * chunk), end = min(n, beg + chunk);
  uint32_t n_gt = 0, n_eq = 0;
  for (int base = beg; base < end; base += 32) {
    const int i = base + lane;
    const uint32_t key = i < end ? keys[i] : 0;
    n_gt += __popc(__ballot_sync(0xffffffffu, i < end && key > thr));
    n_eq += __popc(__ballot_sync(0xffffffffu, i < end && key == thr));
  }
  // exclusive offsets across warps (lane 0 of each warp contributes its counts)
  __shared__ uint32_t gt_off[kTopkWarps], eq_off[kTopkWarps];
  if (lane == 0) { gt_off[warp] = n_gt; eq_off[warp] = n_eq; }
  __syncthreads();
  if (tid == 0) {
    uint32_t g = 0, e = 0;
    for (int w = 0; w < kTopkWarps; ++w) {
      const uint32_t tg = gt_off[w], te = eq_off[w];
      gt_off[w] = g; eq_off[w] = e;
      g += tg; e += te;
    }
  }
  __syncthreads();
  uint32_t gt_seen = gt_off[warp], eq_seen = eq_off[warp];
  const uint32_t lt_mask = (1u << lane) - 1u;
  for (int base = beg; base < end; base += 32) {
    const int i = base + lane;
    const uint32_t key = i < end ? keys[i] : 0;
    const bool gt = i < end && key > thr;
    const bool eq = i < end && key == thr;
    const uint32_t mg = __ballot_sync(0xffffffffu, gt);
    const uint32_t me = __ballot_sync(0xffffffffu, eq);
    const uint32_t g_before = gt_seen + __popc(mg & lt_mask);
    const uint32_t e_before = eq_seen + __popc(me & lt_mask);
    if (gt) out[g_before + min(e_before, need_eq)] = i;
    else if (eq && e_before < need_eq) out[g_before + e_before] = i;
    gt_seen += __popc(mg);
    eq_seen += __popc(me);
  }
}

int launch_topk(const float* scores, int64_t ld, const int32_t* q_pos, const int32_t* kv_len, int B,
                int T, int k, int32_t* idx, cudaStream_t stream, int* status) {
  const int64_t rows = (int64_t)B * T;
  if (rows == 0) return DSA_OK;
  const int max_row = (int)(ld < DSA_TOPK_MAX_ROW ? ld : DSA_TOPK_MAX_ROW);
  const size_t smem = (size_t)(kHistBins + ((max_row + 3) & ~3)) * sizeof(uint32_t);
  static int configured_smem = 0;
  if ((int)smem > configured_smem) {
    if (cudaFuncSetAttribute(topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
        cudaSuccess)
      return DSA_ERR_CUDA;
    configured_smem = (int)smem;
  }
  topk_kernel<<<(unsigned)rows, kTopkThreads, smem, stream>>>(scores, ld, q_pos, kv_len, T, k, max_row,
                                                              idx, status);
  return dsa_host::check_launch();
}

}  // namespace dsa
