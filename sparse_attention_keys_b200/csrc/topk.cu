// dsa_topk: per-query top-k of the index scores over the visible (causal) positions.
//
// Restates index_score.topk(min(index_topk, end_pos)) after the mask add in Indexer.forward
// ("DeepSeek-V3.2-Exp - Rotate first features", Indexer.forward excerpt) and top_2048 of the
// lightning-indexer steps (dense-block page). Ties go to the smaller position; the selection
// is written in ascending position order (with DSA_SORTED: by descending score, equal scores by
// ascending position, via a bitonic sort in shared memory), then -1 padding.
//
// One CTA per score row. The row's visible scores are staged once into shared memory as
// order-preserving 32-bit keys (coalesced 16-byte loads, four in flight per thread), histogramming
// their top 12 bits on the way. A radix select finds the k-th largest key: the first digit (12 bits)
// from that histogram, then one sweep counts the keys above it per warp chunk and collects the
// positions of the keys on it, and the last two digits (10 bits each) run over those candidates only
// (over every key if they exceed a quarter of the row). A compaction (four keys per lane, warp
// shuffle scans of the per-lane counts) writes the selected positions in order. HBM-bound: 4 B read
// per visible score, 4 B written per selected index.
#include <algorithm>

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

__device__ __forceinline__ void hist_add(uint32_t* hist, uint32_t bin, bool active) {
  if (active) atomicAdd(&hist[bin], 1u);
}

// The radix digit holding the `remaining`-th largest key: bins are scanned from the top; thread t
// owns bins nb-1-t*c .. nb-(t+1)*c (c = nb / threads). Writes the digit and how many keys of that
// digit are still needed to *digit / *rem (shared); all threads call it; ends with a barrier.
__device__ void select_digit(const uint32_t* hist, int nb, uint32_t remaining, uint32_t* warp_tot,
                             uint32_t* digit, uint32_t* rem) {
  const int tid = threadIdx.x;
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
        *digit = (uint32_t)bin;
        *rem = remaining - before;
        break;
      }
      before += h;
    }
  }
  __syncthreads();
}

// Ascending bitonic sort of buf[0, n) (n a power of two) by the CTA, then out[i] = the position in
// the low word of buf[i] for i < count, and -1 for count <= i < k.
__device__ void sort_and_write(uint64_t* buf, int n, int count, int k, int32_t* out) {
  __syncthreads();
  for (int size = 2; size <= n; size <<= 1) {
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      for (int i = threadIdx.x; i < (n >> 1); i += kTopkThreads) {
        const int lo = 2 * stride * (i / stride) + (i % stride), hi = lo + stride;
        const bool up = (lo & size) == 0;
        const uint64_t a = buf[lo], b = buf[hi];
        if ((a > b) == up) { buf[lo] = b; buf[hi] = a; }
      }
      __syncthreads();
    }
  }
  for (int i = threadIdx.x; i < k; i += kTopkThreads) out[i] = i < count ? (int32_t)(uint32_t)buf[i] : -1;
}

}  // namespace

__global__ void __launch_bounds__(kTopkThreads, 4) topk_kernel(const float* __restrict__ scores,
                                                            int64_t ld,
                                                            const int32_t* __restrict__ q_pos,
                                                            const int32_t* __restrict__ kv_len,
                                                            int T, int k, int max_row, int cand_cap,
                                                            uint32_t flags, int sort_n,
                                                            int32_t* __restrict__ idx,
                                                            int* status) {
  extern __shared__ __align__(16) uint32_t smem[];
  uint32_t* hist = smem;                       // kHistBins
  uint32_t* keys = smem + kHistBins;           // max_row (rounded up to 4)
  uint32_t* cand = keys + ((max_row + 3) & ~3);  // cand_cap positions (a multiple of 4)
  // DSA_SORTED: sort_n (a power of two >= k) 64-bit keys, (~score key) << 32 | position
  uint64_t* sbuf = reinterpret_cast<uint64_t*>(cand + cand_cap);
  const bool sorted = (flags & DSA_SORTED) != 0;
  __shared__ uint32_t warp_tot[kTopkWarps];
  __shared__ uint32_t sel_digit, sel_remaining, n_cand_sh;
  __shared__ uint32_t gt_off[kTopkWarps], eq_off[kTopkWarps];

  const int64_t row = blockIdx.x;
  const int b = (int)(row / T);
  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  grid_dep_wait();                             // the scores come from the preceding kernel
  grid_dep_launch();
  int32_t* out = idx + row * (int64_t)k;
  int n = min(q_pos[row] + 1, kv_len[b]);
  if (n < 0) n = 0;

  if (n <= k && !sorted) {   // everything visible is selected
    for (int i = tid; i < k; i += kTopkThreads) out[i] = i < n ? i : -1;
    return;
  }
  if (n > max_row) {
    if (tid == 0) set_status(status, DSA_ERR_DEVICE_BOUNDS);
    for (int i = tid; i < k; i += kTopkThreads) out[i] = -1;
    return;
  }

  // Stage the visible scores as keys (zero-padded to a multiple of four) and histogram their top
  // 12 bits (the first radix digit) on the way.
  for (int i = tid; i < kHistBins; i += kTopkThreads) hist[i] = 0;
  if (tid == 0) n_cand_sh = 0;
  __syncthreads();
  const float* src = scores + row * ld;
  const int n4 = n >> 2;
  constexpr int kInFlight = 4;                 // float4 loads issued before any is used
  for (int i0 = 0; i0 < n4; i0 += kInFlight * kTopkThreads) {
    float4 f[kInFlight];
#pragma unroll
    for (int u = 0; u < kInFlight; ++u) {
      const int i = i0 + u * kTopkThreads + tid;
      if (i < n4) f[u] = reinterpret_cast<const float4*>(src)[i];
    }
#pragma unroll
    for (int u = 0; u < kInFlight; ++u) {
      const int i = i0 + u * kTopkThreads + tid;
      if (i < n4) {
        const uint4 kk = make_uint4(order_key(f[u].x), order_key(f[u].y), order_key(f[u].z), order_key(f[u].w));
        reinterpret_cast<uint4*>(keys)[i] = kk;
        atomicAdd(&hist[kk.x >> 20], 1u);
        atomicAdd(&hist[kk.y >> 20], 1u);
        atomicAdd(&hist[kk.z >> 20], 1u);
        atomicAdd(&hist[kk.w >> 20], 1u);
      }
    }
  }
  if (tid < 4 && (n4 << 2) + tid < ((n + 3) & ~3)) {   // the n % 4 tail
    const int i = (n4 << 2) + tid;
    const uint32_t kv = i < n ? order_key(src[i]) : 0u;
    keys[i] = kv;
    if (i < n) atomicAdd(&hist[kv >> 20], 1u);
  }
  __syncthreads();

  if (n <= k) {                               // DSA_SORTED with everything selected
    for (int i = tid; i < sort_n; i += kTopkThreads)
      sbuf[i] = i < n ? ((uint64_t)(~keys[i]) << 32) | (uint32_t)i : ~0ull;
    sort_and_write(sbuf, sort_n, n, k, out);
    return;
  }

  // First digit (12 bits) of the k-th largest key, from the staged histogram.
  select_digit(hist, 4096, (uint32_t)k, warp_tot, &sel_digit, &sel_remaining);
  const uint32_t d1 = sel_digit;
  const uint32_t rem1 = sel_remaining;

  // Warp w owns a contiguous chunk of whole 128-key steps; in each step lane l holds keys
  // 4l..4l+3 (one 16-byte shared-memory load).
  const int steps = (n + 127) / 128;
  const int per_warp = (steps + kTopkWarps - 1) / kTopkWarps;
  const int s_beg = min(steps, warp * per_warp), s_end = min(steps, s_beg + per_warp);

  // Candidate sweep: keys above the first digit are selected for sure (counted per warp); the
  // positions of keys on it are collected (in no particular order) for the last two digits.
  uint32_t n_def = 0;
  for (int st = s_beg; st < s_end; ++st) {
    const int i = st * 128 + 4 * lane;
    uint32_t def4 = 0, cand4 = 0;
    if (i < n) {
      const uint4 kk = reinterpret_cast<const uint4*>(keys)[i >> 2];
      const uint32_t v[4] = {kk.x, kk.y, kk.z, kk.w};
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const bool in = i + u < n;
        def4 |= (uint32_t)(in && (v[u] >> 20) > d1) << u;
        cand4 |= (uint32_t)(in && (v[u] >> 20) == d1) << u;
      }
    }
    n_def += __popc(def4);
    const uint32_t c = __popc(cand4);
    uint32_t incl = c;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
      const uint32_t o = __shfl_up_sync(0xffffffffu, incl, d);
      if (lane >= d) incl += o;
    }
    const uint32_t total = __shfl_sync(0xffffffffu, incl, 31);
    uint32_t base = 0;
    if (lane == 0 && total) base = atomicAdd(&n_cand_sh, total);
    uint32_t slot = __shfl_sync(0xffffffffu, base, 0) + incl - c;
#pragma unroll
    for (int u = 0; u < 4; ++u)
      if ((cand4 >> u) & 1u) {
        if (slot < (uint32_t)cand_cap) cand[slot] = (uint32_t)(i + u);
        ++slot;
      }
  }
#pragma unroll
  for (int d = 16; d > 0; d >>= 1) n_def += __shfl_xor_sync(0xffffffffu, n_def, d);
  if (lane == 0) { gt_off[warp] = n_def; eq_off[warp] = 0; }
  __syncthreads();
  const uint32_t n_cand = n_cand_sh;

  auto classify = [&](int st, uint32_t thr, uint32_t& gt4, uint32_t& eq4) {   // 4-bit masks of keys > thr, == thr
    const int i = st * 128 + 4 * lane;
    gt4 = 0; eq4 = 0;
    if (i < n) {
      const uint4 kk = reinterpret_cast<const uint4*>(keys)[i >> 2];
      const uint32_t v[4] = {kk.x, kk.y, kk.z, kk.w};
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const bool in = i + u < n;
        gt4 |= (uint32_t)(in && v[u] > thr) << u;
        eq4 |= (uint32_t)(in && v[u] == thr) << u;
      }
    }
  };

  uint32_t thr, need_eq;
  if (n_cand <= (uint32_t)cand_cap) {
    // digits 2 and 3 (10 bits each) over the candidates only
    uint32_t prefix = d1 << 20, mask = 0xFFF00000u, remaining = rem1;
#pragma unroll 1
    for (int pass = 0; pass < 2; ++pass) {
      const int shift = pass == 0 ? 10 : 0;
      for (int i = tid; i < 1024; i += kTopkThreads) hist[i] = 0;
      __syncthreads();
      for (uint32_t j = tid; j < n_cand; j += kTopkThreads) {
        const uint32_t kv = keys[cand[j]];
        if ((kv & mask) == prefix) atomicAdd(&hist[(kv >> shift) & 1023u], 1u);
      }
      __syncthreads();
      select_digit(hist, 1024, remaining, warp_tot, &sel_digit, &sel_remaining);
      prefix |= sel_digit << shift;
      mask |= 1023u << shift;
      remaining = sel_remaining;
      __syncthreads();
    }
    thr = prefix;
    need_eq = remaining;
    // the candidates above / at the threshold, added to their warp chunk's counts
    for (uint32_t j = tid; j < n_cand; j += kTopkThreads) {
      const uint32_t pos = cand[j];
      const uint32_t kv = keys[pos];
      const int w = (int)(pos >> 7) / per_warp;
      if (kv > thr) atomicAdd(&gt_off[w], 1u);
      else if (kv == thr) atomicAdd(&eq_off[w], 1u);
    }
  } else {
    // too many keys on the first digit: digits 2 and 3 over all keys, then per-warp counts
    uint32_t prefix = d1 << 20, mask = 0xFFF00000u, remaining = rem1;
#pragma unroll 1
    for (int pass = 0; pass < 2; ++pass) {
      const int shift = pass == 0 ? 10 : 0;
      for (int i = tid; i < 1024; i += kTopkThreads) hist[i] = 0;
      __syncthreads();
      for (int i4 = tid; 4 * i4 < n; i4 += kTopkThreads) {
        const uint4 kk = reinterpret_cast<const uint4*>(keys)[i4];
        const int i = 4 * i4;
        hist_add(hist, (kk.x >> shift) & 1023u, (kk.x & mask) == prefix);
        hist_add(hist, (kk.y >> shift) & 1023u, i + 1 < n && (kk.y & mask) == prefix);
        hist_add(hist, (kk.z >> shift) & 1023u, i + 2 < n && (kk.z & mask) == prefix);
        hist_add(hist, (kk.w >> shift) & 1023u, i + 3 < n && (kk.w & mask) == prefix);
      }
      __syncthreads();
      select_digit(hist, 1024, remaining, warp_tot, &sel_digit, &sel_remaining);
      prefix |= sel_digit << shift;
      mask |= 1023u << shift;
      remaining = sel_remaining;
      __syncthreads();
    }
    thr = prefix;
    need_eq = remaining;
    uint32_t n_gt = 0, n_eq = 0;
    for (int st = s_beg; st < s_end; ++st) {
      uint32_t g4, e4;
      classify(st, thr, g4, e4);
      n_gt += __popc(g4);
      n_eq += __popc(e4);
    }
#pragma unroll
    for (int d = 16; d > 0; d >>= 1) {
      n_gt += __shfl_xor_sync(0xffffffffu, n_gt, d);
      n_eq += __shfl_xor_sync(0xffffffffu, n_eq, d);
    }
    if (lane == 0) { gt_off[warp] = n_gt; eq_off[warp] = n_eq; }
  }
  __syncthreads();
  // exclusive offsets across warps
  if (tid == 0) {
    uint32_t g = 0, e = 0;
    for (int w = 0; w < kTopkWarps; ++w) {
      const uint32_t tg = gt_off[w], te = eq_off[w];
      gt_off[w] = g; eq_off[w] = e;
      g += tg; e += te;
    }
  }
  __syncthreads();

  // Write sweep in ascending position order: keys above the threshold, and the first need_eq keys
  // equal to it (ties go to the smaller position).
  uint32_t gt_seen = gt_off[warp], eq_seen = eq_off[warp];
  for (int st = s_beg; st < s_end; ++st) {
    uint32_t g4, e4;
    classify(st, thr, g4, e4);
    // exclusive prefix of the per-lane counts (lane order = position order)
    uint32_t gi = __popc(g4), ei = __popc(e4);
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
      const uint32_t og = __shfl_up_sync(0xffffffffu, gi, d), oe = __shfl_up_sync(0xffffffffu, ei, d);
      if (lane >= d) { gi += og; ei += oe; }
    }
    const uint32_t g_tot = __shfl_sync(0xffffffffu, gi, 31), e_tot = __shfl_sync(0xffffffffu, ei, 31);
    uint32_t g_before = gt_seen + gi - __popc(g4), e_before = eq_seen + ei - __popc(e4);
    const int i = st * 128 + 4 * lane;
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      int slot = -1;
      if ((g4 >> u) & 1u) {
        slot = (int)(g_before + min(e_before, need_eq));
        ++g_before;
      } else if ((e4 >> u) & 1u) {
        if (e_before < need_eq) slot = (int)(g_before + e_before);
        ++e_before;
      }
      if (slot >= 0) {
        if (sorted) sbuf[slot] = ((uint64_t)(~keys[i + u]) << 32) | (uint32_t)(i + u);
        else out[slot] = i + u;
      }
    }
    gt_seen += g_tot;
    eq_seen += e_tot;
  }
  if (sorted) {                                 // the k selected entries, by descending score
    for (int i = k + tid; i < sort_n; i += kTopkThreads) sbuf[i] = ~0ull;
    sort_and_write(sbuf, sort_n, k, k, out);
  }
}

int launch_topk(const float* scores, int64_t ld, const int32_t* q_pos, const int32_t* kv_len, int B,
                int T, int k, uint32_t flags, int32_t* idx, cudaStream_t stream, int* status) {
  const int64_t rows = (int64_t)B * T;
  if (rows == 0) return DSA_OK;
  const int max_row = (int)(ld < DSA_TOPK_MAX_ROW ? ld : DSA_TOPK_MAX_ROW);
  int sort_n = 0;
  if (flags & DSA_SORTED)
    for (sort_n = 1; sort_n < k; sort_n <<= 1) {
    }
  // candidate positions on the first radix digit: a quarter of the longest row (at least 256)
  const int cand_cap = std::max(256, ((max_row + 3) & ~3) / 4 / 4 * 4);
  const size_t smem = (size_t)(kHistBins + ((max_row + 3) & ~3) + cand_cap) * sizeof(uint32_t) + (size_t)sort_n * 8;
  // the largest dynamic shared memory set so far, per device, in the context it was set in
  static uint64_t configured[dsa_host::kMaxSetupDevices] = {};
  static int configured_smem[dsa_host::kMaxSetupDevices] = {};
  int dev = 0;
  const bool fresh = dsa_host::needs_setup(configured, &dev);
  const bool tracked = dev >= 0 && dev < dsa_host::kMaxSetupDevices;
  if (fresh || !tracked || (int)smem > configured_smem[dev]) {
    if (cudaFuncSetAttribute(topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
        cudaSuccess)
      return DSA_ERR_CUDA;
    if (tracked) {
      if (fresh) configured_smem[dev] = 0;
      configured_smem[dev] = std::max(configured_smem[dev], (int)smem);
      dsa_host::mark_setup(configured);
    }
  }
  return dsa_host::launch(topk_kernel, dim3((unsigned)rows), dim3(kTopkThreads), smem, stream, scores, ld, q_pos,
                          kv_len, T, k, max_row, cand_cap, flags, sort_n, idx, status);
}

}  // namespace dsa
