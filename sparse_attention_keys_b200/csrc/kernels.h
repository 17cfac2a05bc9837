// Internal launchers behind the C ABI (dsa_abi.cu validates arguments, then calls these).
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace dsa {

int launch_index_keys(const void* x, int x_dtype, int64_t rows, int heads, const int32_t* pos,
                      const float* rope_cs, int max_pos, uint32_t flags, uint8_t* out_fp8,
                      float* out_scale, const int64_t* dst_row, cudaStream_t stream, int* status);
// dsa_index_keys on the new keys (heads 1, optionally scattered by k_dst_row) and on the queries
// (q_heads per row, dense) in one launch
int launch_index_qk(const void* kx, int64_t k_rows, const int32_t* k_pos, const int64_t* k_dst_row,
                    uint8_t* k_out_fp8, float* k_out_scale, const void* qx, int64_t q_rows, int q_heads,
                    const int32_t* q_pos, uint8_t* q_out_fp8, float* q_out_scale, int x_dtype,
                    const float* rope_cs, int max_pos, uint32_t flags, cudaStream_t stream, int* status);

int launch_index_topk(const uint8_t* q8, const float* q_scale, const float* w, const uint8_t* k8,
                      const float* k_scale, const int32_t* q_pos, const int32_t* kv_len, int B, int T,
                      int S_max, float softmax_scale, int k, int32_t* idx, cudaStream_t stream, int* status);
int launch_index_scores(const uint8_t* q8, const float* q_scale, const float* w, const uint8_t* k8,
                        const float* k_scale, const int32_t* q_pos, const int32_t* kv_len, int B,
                        int T, int S_max, float softmax_scale, float* scores, int64_t ld,
                        uint32_t flags, cudaStream_t stream, int* status);

int launch_index_scores_paged(const uint8_t* q8, const float* q_scale, const float* w, const uint8_t* k8_pool,
                              const float* k_scale_pool, int64_t num_pages, const int32_t* block_table,
                              int max_pages, int page_size, const int32_t* q_pos, const int32_t* kv_len, int B,
                              int T, float softmax_scale, float* scores, int64_t ld, uint32_t flags,
                              cudaStream_t stream, int* status);

int launch_topk(const float* scores, int64_t ld, const int32_t* q_pos, const int32_t* kv_len, int B,
                int T, int k, uint32_t flags, int32_t* idx, cudaStream_t stream, int* status);

size_t sparse_mla_workspace_size(int B, int T, int k, int heads);
int launch_sparse_mla_paged(const uint16_t* q, const uint16_t* kv_pool, int64_t num_pages,
                            const int32_t* block_table, int max_pages, int page_size, const int32_t* idx, int B,
                            int T, int k, float softmax_scale, uint16_t* out, float* lse, void* workspace,
                            size_t ws_bytes, cudaStream_t stream, int* status);
int launch_mla_q_absorb(const uint16_t* q_nope, const uint16_t* q_pe, const int32_t* pos, const float* rope_cs,
                        int max_pos, const uint16_t* w_uk, int64_t w_head_stride, int64_t rows, uint16_t* q_out,
                        cudaStream_t stream, int* status);
int launch_mla_kv_entry(const uint16_t* kv, const uint16_t* k_pe, const int32_t* pos, const float* rope_cs,
                        int max_pos, int64_t rows, const int64_t* dst_row, uint16_t* kv_cache, int64_t cache_rows,
                        cudaStream_t stream, int* status);
int launch_mla_out_absorb(const uint16_t* o, const uint16_t* w_uv, int64_t w_head_stride, int64_t rows,
                          uint16_t* out, cudaStream_t stream, int* status);
int launch_sparse_mla(const uint16_t* q, const uint16_t* kv, const int32_t* idx, int B, int T,
                      int S_max, int k, int heads, float softmax_scale, uint16_t* out, float* lse,
                      void* workspace, size_t ws_bytes, bool q_ready, cudaStream_t stream, int* status);

}  // namespace dsa
