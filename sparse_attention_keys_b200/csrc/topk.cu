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

// Ascending bitonic sort of buf[0, n) (n a power of two) by the CTA of NT threads, then out[i] = the
// position in the low word of buf[i] for i < count, and -1 for count <= i < k.
template <int NT = kTopkThreads>
__device__ void sort_and_write(uint64_t* buf, int n, int count, int k, int32_t* out) {
  __syncthreads();
  for (int size = 2; size <= n; size <<= 1) {
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      for (int i = threadIdx.x; i < (n >> 1); i += NT) {
        const int lo = 2 * stride * (i / stride) + (i % stride), hi = lo + stride;
        const bool up = (lo & size) == 0;
        const uint64_t a = buf[lo], b = buf[hi];
        if ((a > b) == up) { buf[lo] = b; buf[hi] = a; }
      }
      __syncthreads();
    }
  }
  for (int i = threadIdx.x; i < k; i += NT) out[i] = i < count ? (int32_t)(uint32_t)buf[i] : -1;
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

// ------------------------------------------------------------------------------------------------
// Register-resident variant, for rows of at most kRegRowMax keys (every workload of the pages'
// model: max_seq_len is 16384). The row is read with coalesced 16-byte loads and transposed through
// shared memory so that thread t holds the KPT order keys of positions [t*KPT, t*KPT+KPT) in
// registers. Every later step works on per-thread bit masks over those keys (bit i: position
// t*KPT + i), with branch-free per-key loops:
//   - digit 1 (key bits 31..21) is histogrammed over every key, digit 2 (bits 20..10) over the
//     keys on digit 1 only;
//   - the few keys left on the first 22 bits go to a short shared-memory list, where one step finds
//     the k-th largest key exactly (ties by position) and marks each listed key above or equal to
//     it in per-thread mask words (a radix pass over bits 9..0 does this instead if the list would
//     overflow);
//   - one block scan of packed (above, equal) counts orders the selection by position (each thread's
//     run is contiguous), and the positions are staged in shared memory and leave in coalesced
//     16-byte stores.
// NT threads per CTA: 512 (two CTAs per SM, for launches with many rows) or 1024 (one per SM, for
// launches with fewer rows than SMs, where each row's latency is the launch's).
constexpr int kRegRowMax = 16384;
constexpr int kListCap = 256;                               // keys on the first 22 bits picked directly
// shared words: h1 (2048) | h2 (2048) | h3 (1024) | above / equal masks (NT + NT) | list keys,
// positions (kListCap each) | a region for the transposed row, later the staged output
__host__ __device__ constexpr int reg_fixed_words(int nt) { return 2048 + 2048 + 1024 + 2 * nt + 2 * kListCap; }
__host__ __device__ constexpr int reg_row_words(int kpt, int nt) { return kpt * nt / 32 * 36; }

// hist[bin] += 1 when `pred`, as one predicated shared-memory reduction (no branch, no return value).
__device__ __forceinline__ void hist_inc_if(uint32_t* hist, uint32_t bin, bool pred) {
  asm volatile("{\n\t.reg .pred p;\n\tsetp.ne.u32 p, %1, 0;\n\t@p red.shared.add.u32 [%0], 1;\n\t}" ::"r"(
                   smem_u32(hist + bin)),
               "r"((uint32_t)pred)
               : "memory");
}

// dst[0] = v when `pred` (a predicated shared-memory store).
__device__ __forceinline__ void st_shared_if(int32_t* dst, int32_t v, bool pred) {
  asm volatile("{\n\t.reg .pred p;\n\tsetp.ne.u32 p, %2, 0;\n\t@p st.shared.s32 [%0], %1;\n\t}" ::"r"(smem_u32(dst)),
               "r"(v), "r"((uint32_t)pred)
               : "memory");
}

// Bulk prefetch of [p, p + bytes) into the L2 (p 16-byte aligned, bytes a multiple of 16).
__device__ __forceinline__ void prefetch_l2(const void* p, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}

// Exclusive prefix, in thread order, of one value per thread of the CTA (NT threads); *total gets
// the sum. One barrier; `tot` (NT / 32 words) is written before it and read after it, so a call
// must not reuse the `tot` of the previous call before another barrier.
template <int NT>
__device__ __forceinline__ uint32_t block_excl_scan(uint32_t v, uint32_t* tot, uint32_t* total) {
  constexpr int kRegWarps = NT / 32;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t incl = v;
#pragma unroll
  for (int d = 1; d < 32; d <<= 1) {
    const uint32_t o = __shfl_up_sync(0xffffffffu, incl, d);
    if (lane >= d) incl += o;
  }
  if (lane == 31) tot[warp] = incl;
  __syncthreads();
  const uint32_t wt = lane < kRegWarps ? tot[lane] : 0u;
  uint32_t ws = wt;
#pragma unroll
  for (int d = 1; d < kRegWarps; d <<= 1) {
    const uint32_t o = __shfl_up_sync(0xffffffffu, ws, d);
    if (lane >= d) ws += o;
  }
  const uint32_t warp_before = __shfl_sync(0xffffffffu, ws - wt, warp);
  *total = __shfl_sync(0xffffffffu, ws, kRegWarps - 1);
  return warp_before + incl - v;
}

// The bin holding the target-th largest histogrammed key (bins scanned from the top; thread t
// owns bins NB-1-t*C .. NB-C-t*C). Writes the bin to sel[0], the target's rank inside it (1-based)
// to sel[1] and the bin's count to sel[2]; ends with a barrier.
template <int NB, int NT>
__device__ __forceinline__ void select_bin(const uint32_t* hist, uint32_t target, uint32_t* tot, uint32_t* sel) {
  constexpr int C = NB / NT;
  static_assert(C >= 1, "bins per thread");
  const int top = NB - 1 - (int)threadIdx.x * C;
  uint32_t h[C];
  uint32_t local = 0;
#pragma unroll
  for (int j = 0; j < C; ++j) {
    h[j] = hist[top - j];
    local += h[j];
  }
  uint32_t total;
  uint32_t before = block_excl_scan<NT>(local, tot, &total);
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

template <int KPT, int NT>
__global__ void __launch_bounds__(NT, 1024 / NT) topk_regs_kernel(const float* __restrict__ scores, int64_t ld,
                                                                   const int32_t* __restrict__ q_pos,
                                                                   const int32_t* __restrict__ kv_len, int T, int k,
                                                                   uint32_t flags, int sort_n, int ahead,
                                                                   int32_t* __restrict__ idx, int* status) {
  static_assert(KPT % 4 == 0 && KPT <= 32 && KPT * NT <= kRegRowMax, "keys per thread");
  constexpr int kRegThreads = NT, kRegWarps = NT / 32, kRegFixedWords = reg_fixed_words(NT);
  extern __shared__ __align__(16) uint32_t smem[];
  uint32_t* h1 = smem;                                      // 2048 bins: key bits 31..21
  uint32_t* h2 = smem + 2048;                               // 2048 bins: key bits 20..10
  uint32_t* h3 = smem + 4096;                               // 1024 bins: key bits 9..0 (list overflow)
  uint32_t* gt_words = smem + 5120;                         // per thread: its keys above the k-th (list keys)
  uint32_t* eq_words = gt_words + kRegThreads;              //             and equal to it
  uint32_t* list_key = eq_words + kRegThreads;              // keys on the first 22 bits of the k-th
  int32_t* list_pos = reinterpret_cast<int32_t*>(list_key + kListCap);
  uint32_t* region = smem + kRegFixedWords;                 // the transposed row, then the output
  int32_t* stage = reinterpret_cast<int32_t*>(region);      // k positions, or
  uint64_t* sbuf = reinterpret_cast<uint64_t*>(region);     // sort_n (score, position) keys
  __shared__ uint32_t tots[4][kRegWarps];
  __shared__ uint32_t sel[3];
  __shared__ uint32_t n_list, thr_sh, need_sh;

  const int64_t row = blockIdx.x;
  const int b = (int)(row / T);
  const int tid = threadIdx.x;
  const bool sorted = (flags & DSA_SORTED) != 0;
  grid_dep_wait();                                          // the scores come from the preceding kernel
  grid_dep_launch();
  int32_t* out = idx + row * (int64_t)k;
  // The row that the CTA taking a slot `ahead` launches later will read goes into the L2 now
  // (rows are dispatched in order, and a slot frees about one row's time later), so that its load
  // phase reads the L2 instead of waiting on DRAM.
  if (ahead > 0 && tid < 32 && row + ahead < (int64_t)gridDim.x) {
    const int64_t nrow = row + ahead;
    const int nn = min(q_pos[nrow] + 1, kv_len[nrow / T]);
    if ((nn > k || sorted) && nn > 0 && (int64_t)nn <= ld) {
      const uint32_t bytes = (uint32_t)((nn + 3) >> 2) * 16u;
      const char* base = reinterpret_cast<const char*>(scores + nrow * ld);
      for (uint32_t off = (uint32_t)tid * 4096u; off < bytes; off += 32u * 4096u)
        prefetch_l2(base + off, min(4096u, bytes - off));
    }
  }
  int n = min(q_pos[row] + 1, kv_len[b]);
  if (n < 0) n = 0;
  if (n <= k && !sorted) {                                  // everything visible is selected
    for (int i = tid; i < k; i += kRegThreads) out[i] = i < n ? i : -1;
    return;
  }
  if ((int64_t)n > ld) {                                    // the row buffer is shorter than the visible keys
    if (tid == 0) set_status(status, DSA_ERR_DEVICE_BOUNDS);
    for (int i = tid; i < k; i += kRegThreads) out[i] = -1;
    return;
  }
  // coalesced 16-byte loads (ld is a multiple of 4, so a float4 that starts below n lies in the
  // row), converted to order keys and written to the transposed layout: position p at word
  // p + 4 (p / 32). The row stays there, readable by position, until the output is staged.
  // All of a thread's loads are issued before the first store, so that their latencies overlap.
  const float* src = scores + row * ld;
  const int n4 = (n + 3) >> 2;
  float4 ld4[KPT / 4];
#pragma unroll
  for (int c = 0; c < KPT / 4; ++c) {
    const int f = c * kRegThreads + tid;
    ld4[c] = f < n4 ? __ldcs(reinterpret_cast<const float4*>(src) + f) : make_float4(0.f, 0.f, 0.f, 0.f);
  }
  for (int i = tid; i < kRegFixedWords - 2 * kListCap; i += kRegThreads) smem[i] = 0u;   // while they fly
  if (tid == 0) n_list = 0;
#pragma unroll
  for (int c = 0; c < KPT / 4; ++c) {
    const int f = c * kRegThreads + tid;
    if (f < n4)
      *reinterpret_cast<uint4*>(region + 4 * f + 4 * (f >> 3)) =
          make_uint4(order_key(ld4[c].x), order_key(ld4[c].y), order_key(ld4[c].z), order_key(ld4[c].w));
  }
  __syncthreads();
  auto key_at = [&](int pos) -> uint32_t { return region[pos + 4 * (pos >> 5)]; };
  const int p0 = tid * KPT;
  const int nv = max(0, min(KPT, n - p0));
  uint32_t key[KPT];
#pragma unroll
  for (int c = 0; c < KPT / 4; ++c) {
    uint4 kk = make_uint4(0u, 0u, 0u, 0u);
    const int pc = p0 + 4 * c;                              // at word pc + 4 (pc / 32)
    if (4 * c < nv) kk = *reinterpret_cast<const uint4*>(region + pc + 4 * (pc >> 5));
    key[4 * c] = kk.x;
    key[4 * c + 1] = kk.y;
    key[4 * c + 2] = kk.z;
    key[4 * c + 3] = kk.w;
  }

  if (n <= k) {                                             // DSA_SORTED with everything selected
    __syncthreads();                                        // the region becomes the sort buffer
#pragma unroll
    for (int i = 0; i < KPT; ++i)
      if (i < nv) sbuf[p0 + i] = ((uint64_t)(~key[i]) << 32) | (uint32_t)(p0 + i);
    for (int i = n + tid; i < sort_n; i += kRegThreads) sbuf[i] = ~0ull;
    sort_and_write<NT>(sbuf, sort_n, n, k, out);
    return;
  }

  const uint32_t valid = nv >= 32 ? 0xffffffffu : ((1u << nv) - 1u);
  // digit 1 over every key (threads past the end of a short row skip the per-key work)
  if (nv == KPT) {
#pragma unroll
    for (int i = 0; i < KPT; ++i) hist_inc_if(h1, key[i] >> 21, true);
  } else if (nv > 0) {
#pragma unroll
    for (int i = 0; i < KPT; ++i) hist_inc_if(h1, key[i] >> 21, i < nv);
  }
  __syncthreads();
  select_bin<2048, NT>(h1, (uint32_t)k, tots[0], sel);
  const uint32_t d1 = sel[0];
  uint32_t rem = sel[1];
  uint32_t m_gt = 0, m_on = 0;                              // above the k-th key / still undecided
  if (nv > 0) {
#pragma unroll
    for (int i = 0; i < KPT; ++i) {
      const uint32_t dg = key[i] >> 21;
      m_gt |= (uint32_t)(dg > d1) << i;
      m_on |= (uint32_t)(dg == d1) << i;
    }
    m_gt &= valid;
    m_on &= valid;
  }
  // digit 2 over the keys on digit 1 (a few per thread: read back by position)
  for (uint32_t m = m_on; m; m &= m - 1u) atomicAdd(&h2[(key_at(p0 + __ffs(m) - 1) >> 10) & 2047u], 1u);
  __syncthreads();
  select_bin<2048, NT>(h2, rem, tots[1], sel);
  const uint32_t pre22 = (d1 << 11) | sel[0];
  rem = sel[1];
  const uint32_t n_on = sel[2];                             // keys on the first 22 bits of the k-th
  {
    uint32_t m2 = 0;
    for (uint32_t m = m_on; m; m &= m - 1u) {
      const int i = __ffs(m) - 1;
      const uint32_t pfx = key_at(p0 + i) >> 10;
      m_gt |= (uint32_t)(pfx > pre22) << i;
      m2 |= (uint32_t)(pfx == pre22) << i;
    }
    m_on = m2;
  }

  uint32_t m_eq = 0, need_eq = 0;
  if (rem == n_on) {
    // the k-th key is the smallest on its first 22 bits (always so when it is alone there): every
    // key on them is selected, with no tie to break
    m_gt |= m_on;
  } else if (n_on <= (uint32_t)kListCap) {
    // the keys on the first 22 bits, into the list (positions in any order)
    for (uint32_t m = m_on; m; m &= m - 1u) {
      const int i = __ffs(m) - 1;
      const uint32_t slot = atomicAdd(&n_list, 1u);
      list_key[slot] = key_at(p0 + i);
      list_pos[slot] = p0 + i;
    }
    __syncthreads();
    // the rem-th largest listed key (equal keys ranked by position): entry j's rank is the number
    // of entries above it in (key descending, position ascending) order
    const uint32_t nl = n_list;
    if ((uint32_t)tid < nl) {
      const uint32_t kj = list_key[tid];
      const int pj = list_pos[tid];
      uint32_t rank = 0;
      for (uint32_t e = 0; e < nl; ++e) {
        const uint32_t ke = list_key[e];
        rank += (ke > kj || (ke == kj && list_pos[e] < pj)) ? 1u : 0u;
      }
      if (rank == rem - 1u) thr_sh = kj;
    }
    __syncthreads();
    const uint32_t thr = thr_sh;
    if ((uint32_t)tid < nl) {                               // mark the listed keys for their owners
      const uint32_t kj = list_key[tid];
      const int pj = list_pos[tid];
      if (kj > thr) atomicOr(&gt_words[pj / KPT], 1u << (pj % KPT));
      else if (kj == thr) atomicOr(&eq_words[pj / KPT], 1u << (pj % KPT));
    }
    if (tid == 0) {
      uint32_t above = 0;
      for (uint32_t e = 0; e < nl; ++e) above += list_key[e] > thr ? 1u : 0u;
      need_sh = rem - above;                                // keys equal to the k-th that are selected
    }
    __syncthreads();
    m_gt |= gt_words[tid];
    m_eq = eq_words[tid];
    need_eq = need_sh;
  } else {
    // many keys share the first 22 bits: the last 10 bits by one more radix pass
#pragma unroll
    for (int i = 0; i < KPT; ++i) hist_inc_if(h3, key[i] & 1023u, (m_on >> i) & 1u);
    __syncthreads();
    select_bin<1024, NT>(h3, rem, tots[2], sel);
    const uint32_t thr = (pre22 << 10) | sel[0];
    if (tid == 0) need_sh = sel[1];
    uint32_t g3 = 0, e3 = 0;
#pragma unroll
    for (int i = 0; i < KPT; ++i) {
      g3 |= (uint32_t)(key[i] > thr) << i;
      e3 |= (uint32_t)(key[i] == thr) << i;
    }
    m_gt |= g3 & m_on;
    m_eq = e3 & m_on;
    __syncthreads();
    need_eq = need_sh;
  }

  // compaction in position order: keys above the k-th, and the first need_eq equal to it
  uint32_t total;
  const uint32_t before =
      block_excl_scan<NT>(((uint32_t)__popc(m_gt) << 16) | (uint32_t)__popc(m_eq), tots[3], &total);
  const uint32_t gb = before >> 16, eb = before & 0xFFFFu;
  uint32_t m_sel = m_gt;
  if (m_eq) {                                               // this thread's equal keys ranked eb, eb+1, ...
    uint32_t m = m_eq;
    for (uint32_t r = eb; m && r < need_eq; ++r) {
      m_sel |= m & (0u - m);                                // lowest remaining equal key
      m &= m - 1u;
    }
  }
  const uint32_t base = gb + min(eb, need_eq);
  if (sorted) {
#pragma unroll
    for (int i = 0; i < KPT; ++i)
      if ((m_sel >> i) & 1u)
        sbuf[base + (uint32_t)__popc(m_sel & ((1u << i) - 1u))] = ((uint64_t)(~key[i]) << 32) | (uint32_t)(p0 + i);
    for (int i = k + tid; i < sort_n; i += kRegThreads) sbuf[i] = ~0ull;
    sort_and_write<NT>(sbuf, sort_n, k, k, out);
    return;
  }
  if (4 * k <= n) {            // a sparse selection (row-uniform): visit only the selected keys
    uint32_t r = base;
    for (uint32_t m = m_sel; m; m &= m - 1u) stage[r++] = p0 + __ffs(m) - 1;
  } else if (m_sel) {
#pragma unroll
    for (int i = 0; i < KPT; ++i)
      st_shared_if(stage + base + (uint32_t)__popc(m_sel & ((1u << i) - 1u)), p0 + i, (m_sel >> i) & 1u);
  }
  __syncthreads();
  if ((k & 3) == 0) {
    const int4* s4 = reinterpret_cast<const int4*>(stage);
    int4* o4 = reinterpret_cast<int4*>(out);
    for (int i = tid; i < (k >> 2); i += kRegThreads) o4[i] = s4[i];
  } else {
    for (int i = tid; i < k; i += kRegThreads) out[i] = stage[i];
  }
}

template <int KPT, int NT>
static int launch_topk_regs(const float* scores, int64_t ld, const int32_t* q_pos, const int32_t* kv_len,
                            int64_t rows, int T, int k, uint32_t flags, int sort_n, int32_t* idx,
                            cudaStream_t stream, int* status) {
  const size_t smem = (size_t)reg_fixed_words(NT) * 4 +
                      std::max({(size_t)reg_row_words(KPT, NT) * 4, (size_t)k * 4, (size_t)sort_n * 8});
  static uint64_t configured[dsa_host::kMaxSetupDevices] = {};
  static int configured_smem[dsa_host::kMaxSetupDevices] = {};
  int dev = 0;
  const bool fresh = dsa_host::needs_setup(configured, &dev);
  const bool tracked = dev >= 0 && dev < dsa_host::kMaxSetupDevices;
  if (smem > 48 * 1024 && (fresh || !tracked || (int)smem > configured_smem[dev])) {
    if (cudaFuncSetAttribute(topk_regs_kernel<KPT, NT>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
        cudaSuccess)
      return DSA_ERR_CUDA;
    if (tracked) {
      if (fresh) configured_smem[dev] = 0;
      configured_smem[dev] = std::max(configured_smem[dev], (int)smem);
      dsa_host::mark_setup(configured);
    }
  }
  // the CTAs resident at once: the distance to the row whose scores a CTA prefetches into the L2
  int ahead = 0;
  if (rows > dsa_host::device_sm_count()) {
    int per_sm = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, topk_regs_kernel<KPT, NT>, NT, smem) != cudaSuccess)
      return DSA_ERR_CUDA;
    ahead = std::max(1, per_sm) * dsa_host::device_sm_count();
  }
  return dsa_host::launch(topk_regs_kernel<KPT, NT>, dim3((unsigned)rows), dim3(NT), smem, stream, scores, ld,
                          q_pos, kv_len, T, k, flags, sort_n, ahead, idx, status);
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
  // rows of at most 16384 keys: the register-resident kernel, sized to the longest row; 1024 threads
  // per row when the launch has fewer rows than SMs (each row's latency is then the launch's)
  if (rows < dsa_host::device_sm_count() && max_row <= 1024 * 16) {
    if (max_row <= 1024 * 8)
      return launch_topk_regs<8, 1024>(scores, ld, q_pos, kv_len, rows, T, k, flags, sort_n, idx, stream, status);
    return launch_topk_regs<16, 1024>(scores, ld, q_pos, kv_len, rows, T, k, flags, sort_n, idx, stream, status);
  }
  if (max_row <= 512 * 8)
    return launch_topk_regs<8, 512>(scores, ld, q_pos, kv_len, rows, T, k, flags, sort_n, idx, stream, status);
  if (max_row <= 512 * 16)
    return launch_topk_regs<16, 512>(scores, ld, q_pos, kv_len, rows, T, k, flags, sort_n, idx, stream, status);
  if (max_row <= 512 * 32)
    return launch_topk_regs<32, 512>(scores, ld, q_pos, kv_len, rows, T, k, flags, sort_n, idx, stream, status);
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
