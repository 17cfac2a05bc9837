/*
 * dsa.h - C ABI of libdsa, the B200 (sm_100a) hot path of DeepSeek Sparse Attention.
 *
 * The path: lightning-indexer transform of queries and keys (non-interleaved YaRN RoPE on the
 * first 64 features, (1/sqrt 128) H_128, FP8-e4m3 quantisation with one fp32 scale per
 * 128-element block, K-cache write) -> index scores I[t,s] = sum_j w[t,j] ReLU(q[t,j].k[s]) ->
 * causal per-query top-k -> sparse MQA-style latent attention over the selected positions.
 *
 * Sources (web pages on DeepSeek-V3.2-Exp):
 *   [news]    "DeepSeek fixes RoPE mismatch in the V3.2-Exp inference demo": index-score
 *             formula, ReLU, 128-element FP8 blocks, non-interleaved indexer RoPE.
 *   [rope]    "DeepSeek-V3.2-Exp - RoPE coefficients": YaRN precompute excerpt, ModelArgs.
 *   [dense]   "DeepSeek-V3.2-Exp - Dense transformer block, Sparse latent attention": the
 *             43-step equation list (indexer steps, sparse attention steps, m = 1 + 0.1 ln 40).
 *   [rotate]  "DeepSeek-V3.2-Exp - Rotate first features": Indexer.forward excerpt,
 *             apply_rotary_emb excerpt.
 *   [sim]     "DeepSeek-V3.2-Exp - Similarities": absorbed MQA decode excerpt.
 *
 * Conventions for every entry point:
 *   - All tensor pointers are DEVICE pointers unless a comment says "host". The caller owns
 *     every buffer; the library allocates nothing in these calls and keeps no per-call state.
 *   - Calls are asynchronous and ordered on `stream` (NULL = the legacy default stream).
 *     Kernels are launched with programmatic stream serialisation: each may start while the
 *     previous kernel on the stream finishes, and waits for it (griddepcontrol.wait) before
 *     reading or writing anything an earlier kernel touches. Each also lets the next kernel start
 *     early. A caller's kernel launched with the same attribute right after a dsa call must
 *     therefore wait the same way (cudaGridDependencySynchronize) before reading its outputs.
 *     Kernels launched without it see plain stream order.
 *   - Return value: DSA_OK, or an error code for arguments rejected on the host before any
 *     launch (nothing is launched then) or a failed launch. Errors found on the device
 *     (index or position out of range, a bounded wait that ran out) are recorded in a device
 *     status word and reported by dsa_get_device_status().
 *   - Pointers must be 16-byte aligned; sizes are in elements unless stated.
 *   - bf16 tensors are passed as uint16_t bit patterns.
 *   - No C++ exception crosses this boundary and nothing aborts or traps.
 */
#ifndef DSA_H_
#define DSA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define DSA_API __attribute__((visibility("default")))
#else
#define DSA_API
#endif

typedef struct CUstream_st* dsa_stream_t; /* a cudaStream_t */

/* Status codes */
#define DSA_OK 0
#define DSA_ERR_INVALID_ARG 1   /* null/misaligned pointer or bad size; nothing launched       */
#define DSA_ERR_UNSUPPORTED 2   /* device is not sm_100 (B200 class)                           */
#define DSA_ERR_CUDA 3          /* a CUDA runtime call or kernel launch failed                 */
#define DSA_ERR_TIMEOUT 4       /* device: a bounded wait gave up (status word)                */
#define DSA_ERR_DEVICE_BOUNDS 5 /* device: a position or index outside its buffer (status word) */
#define DSA_ERR_WORKSPACE 6     /* workspace pointer null or smaller than the size query says   */

/* Fixed model dimensions (ModelArgs of DeepSeek-V3.2-Exp, [rope] model-args excerpt; [dense]) */
#define DSA_INDEX_HEADS 64      /* H_I */
#define DSA_INDEX_DIM 128       /* indexer head dim = one FP8 block */
#define DSA_ROPE_PAIRS 32       /* qk_rope_head_dim / 2 */
#define DSA_MLA_HEADS 128
#define DSA_MLA_LATENT 512      /* kv_lora_rank: the value / output width */
#define DSA_MLA_ROPE 64
#define DSA_MLA_QK 576          /* latent + rotary key width */
#define DSA_MAX_POS 1048576     /* positions accepted by dsa_rope_table / dsa_index_keys */
#define DSA_TOPK_MAX_ROW 32768  /* longest score row dsa_topk accepts (kept in shared memory) */
#define DSA_TOPK_SORT_MAX 4096  /* largest k with DSA_SORTED                                    */

/* Flags */
#define DSA_HADAMARD 0x1u      /* dsa_index_keys: apply (1/sqrt 128) H_128 after RoPE ([dense]
                                  indexer steps; rotate_activation in Indexer.forward)         */
#define DSA_SORTED 0x4u        /* dsa_topk: order the selection by descending score, ties by
                                  ascending position (default: ascending position)           */
#define DSA_Q_READY 0x8u       /* dsa_sparse_mla_ex: q is complete before the call (a host copy,
                                  or written two or more kernels earlier): the kernel may stage
                                  it while the preceding kernel on the stream finishes        */
#define DSA_F32 0              /* dsa_index_keys input element types                           */
#define DSA_BF16 1
#define DSA_FILL_MASKED 0x2u   /* dsa_index_scores: write -inf at masked (s > pos) entries of
                                  each row up to S_max (the mask add of Indexer.forward)       */

/*
 * dsa_rope_table - HOST function. Writes the (cos, sin) table of the 32 rotary frequencies,
 * fp32 [max_pos][32][2], into the HOST buffer `table`.
 * Frequencies: theta^(-2i/64), theta = 1e4, blended by YaRN (factor 40, beta_fast 32, beta_slow 1,
 * original length 4096; always on because max_seq_len 16384 > 4096) as in the precompute excerpt
 * of [rope]; the correction-range and ramp helpers (omitted on the page) follow the YaRN paper.
 * angle = fp32(pos * fp32(freq)); cos/sin evaluated in double and rounded to fp32.
 * Returns DSA_ERR_INVALID_ARG if table is NULL or max_pos is outside [1, DSA_MAX_POS].
 */
DSA_API int dsa_rope_table(float* table, int max_pos);

/*
 * dsa_index_keys - indexer query/key transform and block FP8 quantisation
 * ([rotate] Indexer.forward: RoPE on q_pe/k_pe with interleaved=False, rotate_activation,
 * act_quant, k_cache / k_scale_cache write; [news] 128-element blocks).
 *
 *   x        [rows][heads][128] of x_dtype: DSA_F32 (fp32) or DSA_BF16 (bf16 bit patterns,
 *            widened exactly to fp32); rows = tokens; heads = 64 for queries, 1 for keys
 *   pos      int32 [rows]              absolute position of each row (0 <= pos < max_pos)
 *   rope_cs  fp32 [max_pos][32][2]     table from dsa_rope_table (copied to the device)
 *   flags    DSA_HADAMARD or 0
 *   out_fp8  uint8 e4m3 codes; out_scale fp32 scales (one per 128-block)
 *   dst_row  int64 [rows] or NULL. NULL: outputs are dense, [rows][heads][128] and
 *            [rows][heads]. Otherwise row r is written to out_fp8 + dst_row[r]*heads*128 and
 *            out_scale + dst_row[r]*heads (e.g. dst_row = b*S_max + pos for a K-cache
 *            [B][S_max][128]); dst_row values must be >= 0 and distinct and lie inside
 *            the caller's buffers (not checked).
 * Per 128-block: features j<32 pair with j+32 and rotate by pos*freq_j (fp32 arithmetic);
 * features 64..127 pass through; optional Hadamard; amax = max(|y|, 1e-4);
 * scale = amax / 448 (IEEE fp32 division); code = e4m3 round-to-nearest-even, saturating, of
 * the IEEE fp32 quotient y / scale.
 * A pos outside [0, max_pos) sets DSA_ERR_DEVICE_BOUNDS and leaves that row unwritten.
 */
DSA_API int dsa_index_keys(const void* x, int x_dtype, int64_t rows, int heads, const int32_t* pos,
                   const float* rope_cs, int max_pos, uint32_t flags,
                   uint8_t* out_fp8, float* out_scale, const int64_t* dst_row,
                   dsa_stream_t stream);

/*
 * dsa_index_qk - the indexer's key and query transforms of one step in a single launch
 * ([rotate] Indexer.forward applies the same RoPE, rotate_activation and act_quant to the new
 * key and to the queries before fp8_index). Equivalent to
 *   dsa_index_keys(kx, x_dtype, k_rows, 1, k_pos, ..., k_out_fp8, k_out_scale, k_dst_row) and
 *   dsa_index_keys(qx, x_dtype, q_rows, q_heads, q_pos, ..., q_out_fp8, q_out_scale, NULL)
 * with the same rope_cs, max_pos and flags, bit for bit, and the same argument checks and errors
 * (either side may have 0 rows; its pointers are then not read). The key outputs and the query
 * outputs must not overlap (not checked).
 */
DSA_API int dsa_index_qk(const void* kx, int64_t k_rows, const int32_t* k_pos, const int64_t* k_dst_row,
                         uint8_t* k_out_fp8, float* k_out_scale,
                         const void* qx, int64_t q_rows, int q_heads, const int32_t* q_pos,
                         uint8_t* q_out_fp8, float* q_out_scale,
                         int x_dtype, const float* rope_cs, int max_pos, uint32_t flags, dsa_stream_t stream);

/*
 * dsa_index_scores - lightning-indexer scores (fp8_index in Indexer.forward; [dense]
 * S^I_{t,s} = 1/(sqrt 64 sqrt 128) sum_h w_{t,h} ReLU(Q^I_{h,t} . k^I_s)).
 *
 *   q8       uint8 e4m3 [B][T][64][128]     q_scale fp32 [B][T][64]
 *   w        fp32 [B][T][64]                raw head weights (weights_proj output)
 *   k8       uint8 e4m3 [B][S_max][128]     K-cache;  k_scale fp32 [B][S_max]
 *   q_pos    int32 [B][T]   position of each query; kv_len int32 [B] keys present
 *   scores   fp32 [B][T][ld], ld >= S_max, ld a multiple of 4
 * scores[b][t][s] = k_scale[b][s] * sum_j w'[b][t][j] * max(0, sum_i q8[b][t][j][i]*k8[b][s][i])
 * with w' = w * 64^-0.5 * q_scale * softmax_scale (softmax_scale = 128^-0.5 in the model), for
 * every visible s: s <= q_pos[b][t] and s < kv_len[b] (the causal mask; decode passes the last
 * position). Other entries are left untouched, or set to -inf with DSA_FILL_MASKED.
 * Products accumulate in fp32 on the tensor cores (kind::f8f6f4).
 * Constraints: B, T >= 1; 1 <= S_max; q_pos and kv_len within [0, S_max] (kv_len) and
 * [-1, S_max) (q_pos; -1 = no visible key). Not checked on the device beyond masking.
 */
DSA_API int dsa_index_scores(const uint8_t* q8, const float* q_scale, const float* w,
                     const uint8_t* k8, const float* k_scale,
                     const int32_t* q_pos, const int32_t* kv_len,
                     int B, int T, int S_max, float softmax_scale,
                     float* scores, int64_t ld, uint32_t flags, dsa_stream_t stream);

/*
 * dsa_topk - per query, the min(k, n_valid) visible positions with the largest scores
 * (index_score.topk(min(index_topk, end_pos)) after the mask in Indexer.forward; [dense]
 * top_2048). n_valid = min(q_pos+1, kv_len). Only visible entries of `scores` are read.
 *
 *   scores fp32 [B][T][ld];  idx int32 [B][T][k] (output)
 * Ties go to the smaller position. The selected positions are written in ascending order, or
 * with flags = DSA_SORTED by descending score (equal scores by ascending position), then -1 up
 * to k. NaN scores are not allowed. -0.0 and +0.0 compare equal.
 * DSA_SORTED needs k <= DSA_TOPK_SORT_MAX (it sorts the selection in shared memory).
 * Constraints: 1 <= k; every row's n_valid <= DSA_TOPK_MAX_ROW (ld may be larger).
 */
DSA_API int dsa_topk(const float* scores, int64_t ld, const int32_t* q_pos, const int32_t* kv_len,
             int B, int T, int k, uint32_t flags, int32_t* idx, dsa_stream_t stream);

/*
 * dsa_index_topk - the decode indexer fused with its top-k: the selection dsa_index_scores
 * followed by dsa_topk would make (fp8_index, the causal mask and topk(min(index_topk, end_pos)) of
 * Indexer.forward; [dense] S^I and top_2048), in one launch, without writing the scores anywhere.
 *
 *   q8, q_scale, w, k8, k_scale, q_pos, kv_len: as for dsa_index_scores (dense K-cache)
 *   idx int32 [B][T][k] (output): the min(k, n_valid) visible positions with the largest scores,
 *   in ascending order, then -1 up to k; ties go to the smaller position.
 * The scores are the fp32 values dsa_index_scores computes, bit for bit, so idx equals
 * dsa_topk(dsa_index_scores(...)) exactly. Each query's key tiles are scored by a thread-block
 * cluster of up to 8 CTAs that merge their radix histograms in distributed shared memory.
 * Constraints: as dsa_index_scores, plus 1 <= k and S_max <= 32768 (at most 32 key tiles of 128
 * per CTA of the cluster). No workspace; flags are reserved (0).
 */
DSA_API int dsa_index_topk(const uint8_t* q8, const float* q_scale, const float* w,
                   const uint8_t* k8, const float* k_scale,
                   const int32_t* q_pos, const int32_t* kv_len,
                   int B, int T, int S_max, float softmax_scale, int k, uint32_t flags,
                   int32_t* idx, dsa_stream_t stream);

/*
 * dsa_sparse_mla - sparse MQA-style latent attention over the selected positions
 * ([sim] MQA decode: scores over the latent and rotary parts, index mask, softmax, latent-
 * weighted sum; [dense] sparse attention steps S' = S m^2 / sqrt 192; the MLA prefill excerpt
 * in [rope] computed in the same absorbed form).
 *
 *   q      bf16 [B][T][128][576]   absorbed query: 512 latent features then 64 rotary
 *   kv     bf16 [B][S_max][576]    latent cache row = 512 latent features then 64 rotary key
 *   idx    int32 [B][T][k]         selected positions (distinct; -1 = unused slot)
 *   out    bf16 [B][T][128][512];  lse fp32 [B][T][128] or NULL (natural log)
 *   workspace / ws_bytes: device scratch of at least dsa_sparse_mla_workspace_size(B, T, k)
 *          bytes (may be NULL when that size is 0)
 * For each (b, t, head h): z_u = softmax_scale * q[h] . kv[idx_u] over all 576 features,
 * p = softmax(z) over the slots with idx_u >= 0, out[h] = sum_u p_u * kv[idx_u][0:512].
 * In the model softmax_scale = 192^-0.5 * (1 + 0.1 ln 40)^2. A row with no selected position
 * writes zeros and lse = -inf. An idx >= S_max sets DSA_ERR_DEVICE_BOUNDS (that slot is skipped).
 */
DSA_API int dsa_sparse_mla(const uint16_t* q, const uint16_t* kv, const int32_t* idx,
                   int B, int T, int S_max, int k, float softmax_scale,
                   uint16_t* out, float* lse, void* workspace, size_t ws_bytes,
                   dsa_stream_t stream);

/*
 * dsa_sparse_mla_ex - dsa_sparse_mla with flags: 0, or DSA_Q_READY when q is complete before the
 * call (not written by the kernel launched right before on the stream). The kernel then loads q
 * while that kernel finishes, and waits for it only before reading idx. Same arguments, results
 * and errors as dsa_sparse_mla; other flag bits return DSA_ERR_INVALID_ARG.
 */
DSA_API int dsa_sparse_mla_ex(const uint16_t* q, const uint16_t* kv, const int32_t* idx,
                      int B, int T, int S_max, int k, float softmax_scale,
                      uint16_t* out, float* lse, void* workspace, size_t ws_bytes,
                      uint32_t flags, dsa_stream_t stream);

/*
 * dsa_sparse_mla_noalloc - the same computation and arguments as dsa_sparse_mla, minus the
 * workspace, for callers that cannot allocate device memory themselves (for example code inside
 * a host framework whose memory manager owns every device allocation, or a serving loop that
 * must not call cudaMalloc/cudaFree because they can synchronise the device). The pages have no
 * counterpart to this call; it exists only for such callers.
 *   - Allocates nothing. The split-KV scratch comes from one fixed device array inside the
 *     library, dsa_sparse_mla_noalloc_scratch_bytes() = 32 MiB, which every GPU that loads the
 *     library keeps until the process exits.
 *   - A shape whose scratch need (dsa_sparse_mla_workspace_size) exceeds that array is rejected
 *     with DSA_ERR_WORKSPACE before any launch.
 *   - The first call on each device looks up the array's device address with that device current
 *     (again after the device's context is re-created, e.g. by cudaDeviceReset); make that first
 *     call before any stream capture.
 *   - Argument checks and errors are those of dsa_sparse_mla, which this call forwards to with
 *     the fixed array as its workspace.
 *   - Every call shares the one array and it keeps the last call's contents (nothing in it needs
 *     to start at zero: each call overwrites all the scratch it reads). Calls whose work overlaps
 *     on the GPU (different streams, or different host threads on one device) race on it:
 *     serialise them.
 */
DSA_API int dsa_sparse_mla_noalloc(const uint16_t* q, const uint16_t* kv, const int32_t* idx,
                                   int B, int T, int S_max, int k, float softmax_scale,
                                   uint16_t* out, float* lse, dsa_stream_t stream);

/* Size in bytes of the fixed scratch array dsa_sparse_mla_noalloc uses (32 MiB). */
DSA_API size_t dsa_sparse_mla_noalloc_scratch_bytes(void);

/*
 * Paged caches (no counterpart on the pages: the block-table layout serving systems use for the
 * K-cache and the latent cache; the arithmetic is exactly that of the dense calls).
 *
 * A pool holds num_pages pages of page_size rows; sequence b's logical position s lives in row
 * block_table[b][s / page_size] * page_size + s % page_size of the pool. dsa_index_keys writes a
 * paged K-cache through its dst_row argument (dst_row = that pool row).
 *
 *   block_table  int32 [B][max_pages], page ids in [0, num_pages) for every page that holds a
 *                visible position (entries past a sequence's length are not read)
 *   page_size    a power of two, at least 64; S_max = max_pages * page_size is the logical capacity
 * A visible position whose page id is out of range sets DSA_ERR_DEVICE_BOUNDS (its key is
 * skipped: score left unwritten, attention weight zero).
 */

/* dsa_index_scores over a paged K-cache: k8_pool uint8 [num_pages*page_size][128],
 * k_scale_pool fp32 [num_pages*page_size]; everything else as dsa_index_scores. */
DSA_API int dsa_index_scores_paged(const uint8_t* q8, const float* q_scale, const float* w,
                                   const uint8_t* k8_pool, const float* k_scale_pool, int64_t num_pages,
                                   const int32_t* block_table, int max_pages, int page_size,
                                   const int32_t* q_pos, const int32_t* kv_len, int B, int T,
                                   float softmax_scale, float* scores, int64_t ld, uint32_t flags,
                                   dsa_stream_t stream);

/* dsa_sparse_mla over a paged latent cache: kv_pool bf16 [num_pages*page_size][576]; idx holds
 * logical positions (as dsa_topk writes them); everything else as dsa_sparse_mla (same
 * workspace size). */
DSA_API int dsa_sparse_mla_paged(const uint16_t* q, const uint16_t* kv_pool, int64_t num_pages,
                                 const int32_t* block_table, int max_pages, int page_size,
                                 const int32_t* idx, int B, int T, int k, float softmax_scale,
                                 uint16_t* out, float* lse, void* workspace, size_t ws_bytes,
                                 dsa_stream_t stream);

/*
 * Producers of the sparse-MLA inputs and the output absorption (absorbed MQA form). Source: the
 * "Similarities" page, MQA-decode excerpt (q_nope times wkv_b[:, :qk_nope_head_dim]; the latent
 * and rotary caches; the latent-weighted sum times wkv_b[:, -v_head_dim:]); the "Rotate first
 * features" page (MLA RoPE pairs features 2j and 2j+1, the interleaved layout). bf16 in and out,
 * fp32 arithmetic. Weights: head h's [128][512] matrix starts w_head_stride elements after head
 * h-1's (rows of 512 contiguous): w_uk = wkv_b, w_uv = wkv_b + 128*512, stride 256*512 for the
 * reference's wkv_b viewed as [128 heads][256][512]. Pointers 16-byte aligned; w_head_stride a
 * multiple of 8 and >= 128*512; rows >= 0 (0: nothing to do); rows >= 2^31 is rejected.
 */

/* q_out[t][h][0:512] = sum_d q_nope[t][h][d] * w_uk[h][d][0:512];
 * q_out[t][h][512:576] = interleaved RoPE_64 of q_pe[t][h] at pos[t] (rope_cs as dsa_index_keys).
 *   q_nope bf16 [rows][128][128], q_pe bf16 [rows][128][64], pos int32 [rows] in [0, max_pos),
 *   q_out bf16 [rows][128][576] -- the q argument of dsa_sparse_mla.
 * A position outside the table sets DSA_ERR_DEVICE_BOUNDS (that row's rotary part is zero). */
DSA_API int dsa_mla_q_absorb(const uint16_t* q_nope, const uint16_t* q_pe, const int32_t* pos,
                             const float* rope_cs, int max_pos, const uint16_t* w_uk, int64_t w_head_stride,
                             int64_t rows, uint16_t* q_out, dsa_stream_t stream);

/* Latent-cache write: kv_cache[dst_row[t]][0:512] = kv[t] (the normalised latent, copied) and
 * kv_cache[dst_row[t]][512:576] = interleaved RoPE_64 of k_pe[t] at pos[t].
 *   kv bf16 [rows][512], k_pe bf16 [rows][64], pos int32 [rows], dst_row int64 [rows] in
 *   [0, cache_rows), kv_cache bf16 [cache_rows][576] (dense [B][S_max][576] with row b*S_max+s, or a
 *   paged pool). A bad dst_row or position skips the row and sets DSA_ERR_DEVICE_BOUNDS. */
DSA_API int dsa_mla_kv_entry(const uint16_t* kv, const uint16_t* k_pe, const int32_t* pos,
                             const float* rope_cs, int max_pos, int64_t rows, const int64_t* dst_row,
                             uint16_t* kv_cache, int64_t cache_rows, dsa_stream_t stream);

/* out[t][h][0:128] = sum_c o[t][h][c] * w_uv[h][0:128][c].
 *   o bf16 [rows][128][512] (dsa_sparse_mla's out), out bf16 [rows][128][128]. */
DSA_API int dsa_mla_out_absorb(const uint16_t* o, const uint16_t* w_uv, int64_t w_head_stride, int64_t rows,
                               uint16_t* out, dsa_stream_t stream);

/* Bytes of device scratch dsa_sparse_mla needs for this shape (0 when it needs none). */
DSA_API size_t dsa_sparse_mla_workspace_size(int B, int T, int k);

/*
 * dsa_sparse_mla_heads - dsa_sparse_mla over a head shard: the query heads of one rank when the
 * 128 attention heads are split across ranks ("RoPE coefficients" page, MLA init excerpt: each
 * rank keeps n_local_heads = n_heads / world_size heads; the selected indices are the same on
 * every rank, which the Indexer.forward excerpt of "Rotate first features" broadcasts from rank 0).
 *   heads  64 (a two-way split) or 128 (the whole set: the same as dsa_sparse_mla)
 *   q      bf16 [B][T][heads][576];  out bf16 [B][T][heads][512];  lse fp32 [B][T][heads] or NULL
 *   kv, idx, softmax_scale, workspace: as dsa_sparse_mla, the workspace sized by
 *          dsa_sparse_mla_heads_workspace_size(B, T, k, heads)
 * The result for head h of the shard is that of dsa_sparse_mla for the same query row. A 64-head
 * shard runs one CTA per (query, key split) instead of a pair: its score rows fill half the TMEM
 * lanes, and the other half accumulates the second half of the output features.
 * Returns DSA_ERR_INVALID_ARG for any other head count; errors otherwise as dsa_sparse_mla.
 */
DSA_API int dsa_sparse_mla_heads(const uint16_t* q, const uint16_t* kv, const int32_t* idx,
                                 int B, int T, int S_max, int k, int heads, float softmax_scale,
                                 uint16_t* out, float* lse, void* workspace, size_t ws_bytes,
                                 dsa_stream_t stream);

/* Bytes of device scratch dsa_sparse_mla_heads needs (0 when none, or for an invalid shape). */
DSA_API size_t dsa_sparse_mla_heads_workspace_size(int B, int T, int k, int heads);

/*
 * dsa_get_device_status - synchronises `stream`, returns the first error recorded by a kernel
 * since the last call (DSA_OK if none) and clears it. DSA_ERR_CUDA if the sync itself fails.
 */
DSA_API int dsa_get_device_status(dsa_stream_t stream);

/*
 * Where a DSA_ERR_TIMEOUT came from. Every wait inside a kernel is bounded (one second of device
 * time); the first one that gives up records, next to the code, its site (one of the codes
 * below: high nibble = kernel, low nibble = the barrier waited on), the CTA index and how long
 * it waited.
 */
#define DSA_SITE_SCORES_Q 0x11          /* index scores: MMA waits for the query tile (TMA)      */
#define DSA_SITE_SCORES_K_FULL 0x12     /* index scores: MMA waits for a key tile (TMA)          */
#define DSA_SITE_SCORES_K_EMPTY 0x13    /* index scores: TMA waits for a free key stage          */
#define DSA_SITE_SCORES_ACC_FULL 0x14   /* index scores: epilogue waits for an accumulator       */
#define DSA_SITE_SCORES_ACC_EMPTY 0x15  /* index scores: MMA waits for a drained accumulator     */
#define DSA_SITE_MLA_Q 0x21             /* sparse MLA: MMA waits for Q (TMA + TMEM copy)         */
#define DSA_SITE_MLA_KV_FULL 0x22       /* sparse MLA: MMA waits for a gathered KV tile          */
#define DSA_SITE_MLA_KV_EMPTY 0x23      /* sparse MLA: gather waits for a free KV stage          */
#define DSA_SITE_MLA_S_FULL 0x24        /* sparse MLA: softmax waits for a score tile            */
#define DSA_SITE_MLA_P_FULL 0x25        /* sparse MLA: MMA waits for probabilities               */
#define DSA_SITE_MLA_P_EMPTY 0x26       /* sparse MLA: softmax waits for P V before rescaling O  */
#define DSA_SITE_MLA_O_FULL 0x27        /* sparse MLA: epilogue waits for the last P V           */
#define DSA_SITE_SELFTEST 0x31          /* dsa_selftest_wait_timeout                             */
#define DSA_SITE_ABSORB_W 0x41          /* MLA absorption: MMA waits for the resident weights    */
#define DSA_SITE_ABSORB_A_FULL 0x42     /* MLA absorption: MMA waits for an activation stage     */
#define DSA_SITE_ABSORB_A_EMPTY 0x43    /* MLA absorption: TMA waits for a free stage            */
#define DSA_SITE_ABSORB_ACC_FULL 0x44   /* MLA absorption: epilogue waits for an accumulator     */
#define DSA_SITE_ABSORB_ACC_EMPTY 0x45  /* MLA absorption: MMA waits for a drained accumulator   */

/*
 * dsa_get_error_detail - the detail recorded with the last non-OK code that
 * dsa_get_device_status returned on this device: *site (DSA_SITE_*, 0 if the error was not a
 * timeout), *block (CTA index) and *wait_us (how long the wait lasted). Any pointer may be NULL.
 * Returns DSA_OK, or DSA_ERR_CUDA if the device cannot be queried. Host only, no sync.
 */
DSA_API int dsa_get_error_detail(int* site, int* block, int* wait_us);

/*
 * dsa_selftest_wait_timeout - exercises the bounded-wait error path (no counterpart in the
 * method; it exists so failure detection can be tested without hanging or faulting a GPU).
 * Launches one CTA on `stream` that waits on a shared-memory barrier nothing arrives on; the
 * wait gives up after its bound and records DSA_ERR_TIMEOUT with site DSA_SITE_SELFTEST, which
 * dsa_get_device_status then returns. The CUDA context stays usable. Returns DSA_OK once
 * launched, DSA_ERR_UNSUPPORTED / DSA_ERR_CUDA otherwise.
 */
DSA_API int dsa_selftest_wait_timeout(dsa_stream_t stream);

/* Human-readable name of a status code (static string). */
DSA_API const char* dsa_status_string(int code);

/* 1 if the current device is sm_100 (B200 class) and the library's kernels can run on it. */
DSA_API int dsa_device_supported(void);

/* Library version string. */
DSA_API const char* dsa_version(void);

#ifdef __cplusplus
}
#endif

#endif /* DSA_H_ */
