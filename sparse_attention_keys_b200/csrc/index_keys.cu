// dsa_index_keys: indexer query/key transform and block FP8 quantisation.
//
// Restates, per 128-feature head row, the steps of Indexer.forward ("DeepSeek-V3.2-Exp - Rotate
// first features", Indexer.forward excerpt): non-interleaved RoPE on the first 64 features
// (feature j pairs with j+32, apply_rotary_emb with interleaved=False), rotate_activation
// ((1/sqrt 128) H_128, dense-block page indexer steps), act_quant with 128-element blocks
// (news page), and the k_cache / k_scale_cache write.
//
// One warp per 128-element block; lane l holds features 4l..4l+3 (one 16-byte load), so the
// row is read and written with fully coalesced 512-byte / 128-byte warp transactions. The
// Hadamard is a 7-stage butterfly: stages over feature bits 0-1 stay in registers, bits 2-6 are
// warp shuffles (lane bits 0-4). HBM-bound: 512 B read + 132 B written per block.
#include <cuda_fp8.h>

#include "common.cuh"
#include "kernels.h"

namespace dsa {

// Four consecutive features of block `blk` for lane `lane`, widened to fp32 (bf16 widening is exact).
template <typename In>
__device__ __forceinline__ float4 load4(const In* __restrict__ x, int64_t blk, int lane);
template <>
__device__ __forceinline__ float4 load4<float>(const float* __restrict__ x, int64_t blk, int lane) {
  return reinterpret_cast<const float4*>(x + blk * 128)[lane];
}
template <>
__device__ __forceinline__ float4 load4<uint16_t>(const uint16_t* __restrict__ x, int64_t blk, int lane) {
  const uint2 u = reinterpret_cast<const uint2*>(x + blk * 128)[lane];
  return make_float4(__uint_as_float(u.x << 16), __uint_as_float(u.x & 0xffff0000u), __uint_as_float(u.y << 16),
                     __uint_as_float(u.y & 0xffff0000u));
}

// One transform problem: `blocks` 128-element blocks of x ([rows][heads][128]), their positions
// and outputs (dense, or scattered to the rows dst_row names).
struct KeysJob {
  const void* x;
  int64_t blocks;
  int heads;
  const int32_t* pos;
  uint8_t* out_fp8;
  float* out_scale;
  const int64_t* dst_row;
};

// One warp transforms block `blk` of job `j`.
template <typename In>
__device__ __forceinline__ void transform_block(const KeysJob& j, int64_t blk, int lane,
                                                const float* __restrict__ rope_cs, int max_pos, uint32_t flags,
                                                int* status) {
  const In* __restrict__ x = static_cast<const In*>(j.x);
  const int64_t row = blk / j.heads;
  const int head = (int)(blk - row * j.heads);
  // the three loads that do not depend on the position go out together, before the RoPE table
  // load that does (a warp's only work is this one block, so its latency is the chain of loads)
  const float4 v4 = load4<In>(x, blk, lane);
  const int64_t dst = j.dst_row ? __ldg(j.dst_row + row) : -1;
  const int p = j.pos[row];
  if (p < 0 || p >= max_pos) {
    if (lane == 0) set_status(status, DSA_ERR_DEVICE_BOUNDS);
    return;
  }
  float v[4] = {v4.x, v4.y, v4.z, v4.w};

  // RoPE on features 0..63: lanes 0-7 hold the first halves a_j (j = 4*lane + i), lanes 8-15
  // the second halves b_j; a_j' = a c - b s, b_j' = a s + b c.
  {
    float partner[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) partner[i] = __shfl_xor_sync(0xffffffffu, v[i], 8);
    if (lane < 16) {
      const int j0 = 4 * (lane & 7);
      const float4* cs = reinterpret_cast<const float4*>(rope_cs + ((int64_t)p * 32 + j0) * 2);
      const float4 c01 = cs[0], c23 = cs[1];   // (cos, sin) of pairs j0..j0+3
      const float c[4] = {c01.x, c01.z, c23.x, c23.z};
      const float s[4] = {c01.y, c01.w, c23.y, c23.w};
      if (lane < 8) {
#pragma unroll
        for (int i = 0; i < 4; ++i) v[i] = __fsub_rn(__fmul_rn(v[i], c[i]), __fmul_rn(partner[i], s[i]));
      } else {
#pragma unroll
        for (int i = 0; i < 4; ++i) v[i] = __fadd_rn(__fmul_rn(partner[i], s[i]), __fmul_rn(v[i], c[i]));
      }
    }
  }

  if (flags & DSA_HADAMARD) {
    // feature bit 0 and 1: in registers
    float t0 = v[0] + v[1], t1 = v[0] - v[1], t2 = v[2] + v[3], t3 = v[2] - v[3];
    v[0] = t0 + t2; v[2] = t0 - t2; v[1] = t1 + t3; v[3] = t1 - t3;
    // feature bits 2..6 = lane bits 0..4
#pragma unroll
    for (int m = 1; m < 32; m <<= 1) {
      const bool upper = (lane & m) != 0;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float o = __shfl_xor_sync(0xffffffffu, v[i], m);
        v[i] = upper ? (o - v[i]) : (v[i] + o);
      }
    }
    const float inv_sqrt128 = 0.08838834764831845f;
#pragma unroll
    for (int i = 0; i < 4; ++i) v[i] = __fmul_rn(v[i], inv_sqrt128);
  }

  float amax = fmaxf(fmaxf(fabsf(v[0]), fabsf(v[1])), fmaxf(fabsf(v[2]), fabsf(v[3])));
#pragma unroll
  for (int m = 16; m > 0; m >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, m));
  amax = fmaxf(amax, 1e-4f);
  const float scale = __fdiv_rn(amax, 448.0f);

  const __nv_fp8x2_storage_t lo =
      __nv_cvt_float2_to_fp8x2(make_float2(__fdiv_rn(v[0], scale), __fdiv_rn(v[1], scale)),
                               __NV_SATFINITE, __NV_E4M3);
  const __nv_fp8x2_storage_t hi =
      __nv_cvt_float2_to_fp8x2(make_float2(__fdiv_rn(v[2], scale), __fdiv_rn(v[3], scale)),
                               __NV_SATFINITE, __NV_E4M3);
  const uint32_t packed = (uint32_t)lo | ((uint32_t)hi << 16);

  const int64_t out_blk = j.dst_row ? dst * j.heads + head : blk;
  reinterpret_cast<uint32_t*>(j.out_fp8 + out_blk * 128)[lane] = packed;
  if (lane == 0) j.out_scale[out_blk] = scale;
}

constexpr int kKeysWarps = 8;   // blocks (warps) per CTA

// Two jobs in one launch: CTAs [0, a_ctas) transform job a, the rest job b (one block per warp).
template <typename In>
__global__ void __launch_bounds__(kKeysWarps * 32) index_keys_kernel(const KeysJob a, const KeysJob b, int64_t a_ctas,
                                                                     const float* __restrict__ rope_cs, int max_pos,
                                                                     uint32_t flags, int* status) {
  const int lane = threadIdx.x & 31;
  const bool in_a = (int64_t)blockIdx.x < a_ctas;
  const int64_t cta = in_a ? (int64_t)blockIdx.x : (int64_t)blockIdx.x - a_ctas;
  const int64_t blk = cta * kKeysWarps + (threadIdx.x >> 5);
  grid_dep_wait();
  grid_dep_launch();
  const KeysJob j = in_a ? a : b;
  if (blk >= j.blocks) return;
  transform_block<In>(j, blk, lane, rope_cs, max_pos, flags, status);
}

int launch_index_qk(const void* kx, int64_t k_rows, const int32_t* k_pos, const int64_t* k_dst_row,
                    uint8_t* k_out_fp8, float* k_out_scale, const void* qx, int64_t q_rows, int q_heads,
                    const int32_t* q_pos, uint8_t* q_out_fp8, float* q_out_scale, int x_dtype,
                    const float* rope_cs, int max_pos, uint32_t flags, cudaStream_t stream, int* status) {
  const KeysJob a{kx, k_rows, 1, k_pos, k_out_fp8, k_out_scale, k_dst_row};
  const KeysJob b{qx, q_rows * q_heads, q_heads, q_pos, q_out_fp8, q_out_scale, nullptr};
  const int64_t a_ctas = (a.blocks + kKeysWarps - 1) / kKeysWarps;
  const int64_t grid = a_ctas + (b.blocks + kKeysWarps - 1) / kKeysWarps;
  if (grid == 0) return DSA_OK;
  if (grid > 0x7fffffff) return DSA_ERR_INVALID_ARG;
  if (x_dtype == DSA_BF16)
    return dsa_host::launch(index_keys_kernel<uint16_t>, dim3((unsigned)grid), dim3(kKeysWarps * 32), 0, stream, a, b,
                            a_ctas, rope_cs, max_pos, flags, status);
  return dsa_host::launch(index_keys_kernel<float>, dim3((unsigned)grid), dim3(kKeysWarps * 32), 0, stream, a, b,
                          a_ctas, rope_cs, max_pos, flags, status);
}

int launch_index_keys(const void* x, int x_dtype, int64_t rows, int heads, const int32_t* pos,
                      const float* rope_cs, int max_pos, uint32_t flags, uint8_t* out_fp8,
                      float* out_scale, const int64_t* dst_row, cudaStream_t stream, int* status) {
  const KeysJob a{x, rows * heads, heads, pos, out_fp8, out_scale, dst_row};
  const KeysJob none{x, 0, 1, pos, out_fp8, out_scale, nullptr};
  const int64_t grid = (a.blocks + kKeysWarps - 1) / kKeysWarps;
  if (grid == 0) return DSA_OK;
  if (grid > 0x7fffffff) return DSA_ERR_INVALID_ARG;
  if (x_dtype == DSA_BF16)
    return dsa_host::launch(index_keys_kernel<uint16_t>, dim3((unsigned)grid), dim3(kKeysWarps * 32), 0, stream, a,
                            none, grid, rope_cs, max_pos, flags, status);
  return dsa_host::launch(index_keys_kernel<float>, dim3((unsigned)grid), dim3(kKeysWarps * 32), 0, stream, a, none,
                          grid, rope_cs, max_pos, flags, status);
}

}  // namespace dsa
