// C ABI of libdsa: argument validation, the device status word, and dispatch to the kernels.
// Declarations and contracts: include/dsa.h.
#include <cuda.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include <algorithm>
#include <mutex>

#include "common.cuh"
#include "dsa.h"
#include "kernels.h"

namespace {

// Status block: code, then (for a timeout) site, CTA index, wait length in microseconds.
__device__ int g_dsa_status[4] = {0, 0, 0, 0};

// A barrier nothing arrives on, waited on with the kernels' own bounded wait.
__global__ void selftest_wait_kernel(int* status) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    abort_flag = 0;
    dsa::mbar_init(&bar, 1);
    dsa::fence_barrier_init();
  }
  __syncthreads();
  dsa::mbar_wait(&bar, 0, &abort_flag, status, DSA_SITE_SELFTEST);
}

constexpr int kMaxDevices = 64;

typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long*);

// The driver's context queries, looked up once through the runtime (the library does not link
// libcuda directly).
struct ContextQueries {
  CtxGetCurrentFn get_current = nullptr;
  CtxGetIdFn get_id = nullptr;
};
const ContextQueries& context_queries() {
  static ContextQueries q;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult r;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &r) == cudaSuccess &&
        r == cudaDriverEntryPointSuccess)
      q.get_current = reinterpret_cast<CtxGetCurrentFn>(p);
    p = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &r) == cudaSuccess &&
        r == cudaDriverEntryPointSuccess)
      q.get_id = reinterpret_cast<CtxGetIdFn>(p);
  });
  return q;
}

struct DeviceCache {
  uint64_t ctx = 0;            // id of the context the addresses below belong to (0: not set up)
  bool supported = false;
  int sms = 0;
  int* status = nullptr;
  int detail[3] = {0, 0, 0};   // site, block, wait_us of the last error read back
};
DeviceCache g_dev[kMaxDevices];
std::mutex g_mu;

// The status word's device address belongs to the context it was looked up in: when the device's
// context is re-created (for instance after cudaDeviceReset) it is looked up again.
DeviceCache* device_cache() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  DeviceCache& c = g_dev[dev];
  const uint64_t ctx = dsa_host::current_context_id();
  if (c.ctx == 0 || c.ctx != ctx) {
    std::lock_guard<std::mutex> lk(g_mu);
    if (c.ctx == 0 || c.ctx != ctx) {
      cudaDeviceProp prop;
      if (cudaGetDeviceProperties(&prop, dev) != cudaSuccess) return nullptr;
      c.supported = prop.major == 10 && prop.minor == 0;
      c.sms = prop.multiProcessorCount;
      void* addr = nullptr;
      if (cudaGetSymbolAddress(&addr, g_dsa_status) != cudaSuccess) return nullptr;
      c.status = static_cast<int*>(addr);
      c.ctx = dsa_host::current_context_id();     // the lookup made the device's context current
    }
  }
  return &c;
}

// Common prologue: device is sm_100 and the status word is reachable.
int prologue(int** status) {
  DeviceCache* c = device_cache();
  if (!c) return DSA_ERR_CUDA;
  if (!c->supported) return DSA_ERR_UNSUPPORTED;
  *status = c->status;
  return DSA_OK;
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

}  // namespace

namespace dsa_host {

uint64_t current_context_id() {
  const ContextQueries& q = context_queries();
  if (!q.get_current || !q.get_id) return 0;
  CUcontext ctx = nullptr;
  if (q.get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) return 0;
  unsigned long long id = 0;
  if (q.get_id(ctx, &id) != CUDA_SUCCESS) return 0;
  return (uint64_t)id + 1;
}

bool needs_setup(uint64_t* seen, int* dev_out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) dev = 0;
  if (dev_out) *dev_out = dev;
  if (dev < 0 || dev >= kMaxDevices) return true;
  const uint64_t ctx = current_context_id();
  return ctx == 0 || seen[dev] != ctx;
}

void mark_setup(uint64_t* seen) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return;
  seen[dev] = current_context_id();
}

int* status_word() {
  DeviceCache* c = device_cache();
  return c ? c->status : nullptr;
}

int check_launch() { return cudaGetLastError() == cudaSuccess ? DSA_OK : DSA_ERR_CUDA; }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int device_sm_count() {
  DeviceCache* c = device_cache();
  return (c && c->sms > 0) ? c->sms : 148;
}

int resident_ctas_per_sm(const void* func, int threads, int dyn_smem, int tmem_cols) {
  cudaFuncAttributes a;
  int dev = 0, smem_sm = 0, regs_sm = 0, threads_sm = 0, blocks_sm = 0, reserved = 0;
  if (cudaFuncGetAttributes(&a, func) != cudaSuccess || cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&smem_sm, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&regs_sm, cudaDevAttrMaxRegistersPerMultiprocessor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&threads_sm, cudaDevAttrMaxThreadsPerMultiProcessor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&blocks_sm, cudaDevAttrMaxBlocksPerMultiprocessor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&reserved, cudaDevAttrReservedSharedMemoryPerBlock, dev) != cudaSuccess)
    return 0;
  const int warps = (threads + 31) / 32;
  const int regs_cta = ((a.numRegs + 7) / 8 * 8) * 32 * warps;      // registers are allocated per warp, 8 at a time
  int n = blocks_sm;
  n = std::min(n, smem_sm / std::max(1, dyn_smem + (int)a.sharedSizeBytes + reserved));
  n = std::min(n, regs_sm / std::max(1, regs_cta));
  n = std::min(n, threads_sm / std::max(1, warps * 32));
  if (tmem_cols > 0) n = std::min(n, 512 / tmem_cols);
  return std::max(n, 0);
}

bool encode_tensor_map_2d(CUtensorMap* map, CUtensorMapDataType dtype, void* base, uint64_t inner,
                          uint64_t outer, uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer,
                          CUtensorMapSwizzle swizzle) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {inner, outer};
  const cuuint64_t strides[1] = {row_bytes};
  const cuuint32_t box[2] = {box_inner, box_outer};
  const cuuint32_t estr[2] = {1, 1};
  return fn(map, dtype, 2, base, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool encode_tensor_map_3d(CUtensorMap* map, CUtensorMapDataType dtype, void* base, const uint64_t dims[3],
                          const uint64_t strides[2], const uint32_t box[3], CUtensorMapSwizzle swizzle) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t d[3] = {dims[0], dims[1], dims[2]};
  const cuuint64_t st[2] = {strides[0], strides[1]};
  const cuuint32_t bx[3] = {box[0], box[1], box[2]};
  const cuuint32_t estr[3] = {1, 1, 1};
  return fn(map, dtype, 3, base, d, st, bx, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace dsa_host

// ------------------------------------------------------------------------------------------------
// Host-side RoPE table: YaRN frequencies of the "RoPE coefficients" precompute excerpt; the
// correction range and linear ramp follow the YaRN paper (their bodies are omitted on the page).
// ------------------------------------------------------------------------------------------------
namespace {

double yarn_correction_dim(double rotations, int dim, double base, double max_pos) {
  return dim * log(max_pos / (rotations * 2.0 * M_PI)) / (2.0 * log(base));
}

void yarn_freqs(double out[DSA_ROPE_PAIRS]) {
  const int dim = 2 * DSA_ROPE_PAIRS;            // qk_rope_head_dim = 64
  const double base = 10000.0, factor = 40.0;
  const double beta_fast = 32.0, beta_slow = 1.0, original = 4096.0;
  const int max_seq_len = 16384;
  double low = floor(yarn_correction_dim(beta_fast, dim, base, original));
  double high = ceil(yarn_correction_dim(beta_slow, dim, base, original));
  if (low < 0) low = 0;
  if (high > dim - 1) high = dim - 1;
  if (low == high) high += 0.001;
  for (int i = 0; i < DSA_ROPE_PAIRS; ++i) {
    const double f = 1.0 / pow(base, (2.0 * i) / dim);
    double ramp = (i - low) / (high - low);
    ramp = ramp < 0 ? 0 : (ramp > 1 ? 1 : ramp);
    const double smooth = 1.0 - ramp;
    out[i] = (max_seq_len > original) ? f / factor * (1.0 - smooth) + f * smooth : f;
  }
}

}  // namespace

extern "C" {

int dsa_rope_table(float* table, int max_pos) {
  if (!table || max_pos < 1 || max_pos > DSA_MAX_POS) return DSA_ERR_INVALID_ARG;
  double f[DSA_ROPE_PAIRS];
  yarn_freqs(f);
  float f32[DSA_ROPE_PAIRS];
  for (int i = 0; i < DSA_ROPE_PAIRS; ++i) f32[i] = (float)f[i];
  for (int p = 0; p < max_pos; ++p) {
    for (int i = 0; i < DSA_ROPE_PAIRS; ++i) {
      const float ang = (float)p * f32[i];           // fp32 product, as the page's float32 outer
      table[((size_t)p * DSA_ROPE_PAIRS + i) * 2 + 0] = (float)cos((double)ang);
      table[((size_t)p * DSA_ROPE_PAIRS + i) * 2 + 1] = (float)sin((double)ang);
    }
  }
  return DSA_OK;
}

// The argument checks of dsa_index_keys (no launch): DSA_OK, or DSA_ERR_INVALID_ARG.
static int index_keys_args(const void* x, int x_dtype, int64_t rows, int heads, const int32_t* pos,
                           const float* rope_cs, int max_pos, uint32_t flags, const uint8_t* out_fp8,
                           const float* out_scale, const int64_t* dst_row) {
  if (rows < 0 || heads < 1 || heads > 4096 || max_pos < 1 || max_pos > DSA_MAX_POS ||
      (flags & ~DSA_HADAMARD) != 0 || (x_dtype != DSA_F32 && x_dtype != DSA_BF16))
    return DSA_ERR_INVALID_ARG;
  if (rows == 0) return DSA_OK;
  if (!x || !pos || !rope_cs || !out_fp8 || !out_scale) return DSA_ERR_INVALID_ARG;
  if (!dsa_host::aligned16(x) || !dsa_host::aligned16(rope_cs) || !dsa_host::aligned16(out_fp8) ||
      !dsa_host::aligned16(out_scale) || (dst_row && !dsa_host::aligned16(dst_row)) ||
      !dsa_host::aligned16(pos))
    return DSA_ERR_INVALID_ARG;
  return DSA_OK;
}

int dsa_index_keys(const void* x, int x_dtype, int64_t rows, int heads, const int32_t* pos, const float* rope_cs,
                   int max_pos, uint32_t flags, uint8_t* out_fp8, float* out_scale,
                   const int64_t* dst_row, dsa_stream_t stream) {
  int rc = index_keys_args(x, x_dtype, rows, heads, pos, rope_cs, max_pos, flags, out_fp8, out_scale, dst_row);
  if (rc != DSA_OK || rows == 0) return rc;
  int* status;
  rc = prologue(&status);
  if (rc != DSA_OK) return rc;
  return dsa::launch_index_keys(x, x_dtype, rows, heads, pos, rope_cs, max_pos, flags, out_fp8, out_scale,
                                dst_row, (cudaStream_t)stream, status);
}

int dsa_index_qk(const void* kx, int64_t k_rows, const int32_t* k_pos, const int64_t* k_dst_row,
                 uint8_t* k_out_fp8, float* k_out_scale, const void* qx, int64_t q_rows, int q_heads,
                 const int32_t* q_pos, uint8_t* q_out_fp8, float* q_out_scale, int x_dtype,
                 const float* rope_cs, int max_pos, uint32_t flags, dsa_stream_t stream) {
  int rc = index_keys_args(kx, x_dtype, k_rows, 1, k_pos, rope_cs, max_pos, flags, k_out_fp8, k_out_scale,
                           k_dst_row);
  if (rc != DSA_OK) return rc;
  rc = index_keys_args(qx, x_dtype, q_rows, q_heads, q_pos, rope_cs, max_pos, flags, q_out_fp8, q_out_scale,
                       nullptr);
  if (rc != DSA_OK) return rc;
  if (k_rows == 0 && q_rows == 0) return DSA_OK;
  int* status;
  rc = prologue(&status);
  if (rc != DSA_OK) return rc;
  return dsa::launch_index_qk(kx, k_rows, k_pos, k_dst_row, k_out_fp8, k_out_scale, qx, q_rows, q_heads, q_pos,
                              q_out_fp8, q_out_scale, x_dtype, rope_cs, max_pos, flags, (cudaStream_t)stream,
                              status);
}

int dsa_index_scores(const uint8_t* q8, const float* q_scale, const float* w, const uint8_t* k8,
                     const float* k_scale, const int32_t* q_pos, const int32_t* kv_len, int B, int T,
                     int S_max, float softmax_scale, float* scores, int64_t ld, uint32_t flags,
                     dsa_stream_t stream) {
  if (B < 1 || T < 1 || S_max < 1 || ld < S_max || (ld & 3) != 0 || (flags & ~DSA_FILL_MASKED) != 0 ||
      !(softmax_scale > 0.f) || !isfinite(softmax_scale))
    return DSA_ERR_INVALID_ARG;
  if ((int64_t)B * T * 64 > 0x7fffffffLL || (int64_t)B * S_max > 0x7fffffffLL) return DSA_ERR_INVALID_ARG;
  if (!q8 || !q_scale || !w || !k8 || !k_scale || !q_pos || !kv_len || !scores) return DSA_ERR_INVALID_ARG;
  const void* ptrs[] = {q8, q_scale, w, k8, k_scale, q_pos, kv_len, scores};
  for (const void* p : ptrs)
    if (!dsa_host::aligned16(p)) return DSA_ERR_INVALID_ARG;
  int* status;
  int rc = prologue(&status);
  if (rc != DSA_OK) return rc;
  return dsa::launch_index_scores(q8, q_scale, w, k8, k_scale, q_pos, kv_len, B, T, S_max, softmax_scale,
                                  scores, ld, flags, (cudaStream_t)stream, status);
}

int dsa_index_topk(const uint8_t* q8, const float* q_scale, const float* w, const uint8_t* k8,
                   const float* k_scale, const int32_t* q_pos, const int32_t* kv_len, int B, int T, int S_max,
                   float softmax_scale, int k, uint32_t flags, int32_t* idx, dsa_stream_t stream) {
  if (B < 1 || T < 1 || S_max < 1 || S_max > DSA_TOPK_MAX_ROW || k < 1 || flags != 0 || !(softmax_scale > 0.f) ||
      !isfinite(softmax_scale))
    return DSA_ERR_INVALID_ARG;
  if ((int64_t)B * T * 64 > 0x7fffffffLL || (int64_t)B * S_max > 0x7fffffffLL ||
      (int64_t)B * T * 8 > 0x7fffffffLL)
    return DSA_ERR_INVALID_ARG;
  if (!q8 || !q_scale || !w || !k8 || !k_scale || !q_pos || !kv_len || !idx) return DSA_ERR_INVALID_ARG;
  const void* ptrs[] = {q8, q_scale, w, k8, k_scale, q_pos, kv_len, idx};
  for (const void* p : ptrs)
    if (!dsa_host::aligned16(p)) return DSA_ERR_INVALID_ARG;
  int* status;
  int rc = prologue(&status);
  if (rc != DSA_OK) return rc;
  return dsa::launch_index_topk(q8, q_scale, w, k8, k_scale, q_pos, kv_len, B, T, S_max, softmax_scale, k, idx,
                                (cudaStream_t)stream, status);
}

int dsa_topk(const float* scores, int64_t ld, const int32_t* q_pos, const int32_t* kv_len, int B, int T,
             int k, uint32_t flags, int32_t* idx, dsa_stream_t stream) {
  if (B < 1 || T < 1 || k < 1 || ld < 1 || (ld & 3) != 0 || (flags & ~DSA_SORTED) != 0) return DSA_ERR_INVALID_ARG;
  if ((flags & DSA_SORTED) && k > DSA_TOPK_SORT_MAX) return DSA_ERR_INVALID_ARG;
  if ((int64_t)B * T > 0x7fffffffLL) return DSA_ERR_INVALID_ARG;
  if (!scores || !q_pos || !kv_len || !idx) return DSA_ERR_INVALID_ARG;
  if (!dsa_host::aligned16(scores) || !dsa_host::aligned16(q_pos) || !dsa_host::aligned16(kv_len) ||
      !dsa_host::aligned16(idx))
    return DSA_ERR_INVALID_ARG;
  int* status;
  int rc = prologue(&status);
  if (rc != DSA_OK) return rc;
  return dsa::launch_topk(scores, ld, q_pos, kv_len, B, T, k, flags, idx, (cudaStream_t)stream, status);
}

size_t dsa_sparse_mla_workspace_size(int B, int T, int k) {
  if (B < 1 || T < 1 || k < 1) return 0;
  return dsa::sparse_mla_workspace_size(B, T, k, DSA_MLA_HEADS);
}

size_t dsa_sparse_mla_heads_workspace_size(int B, int T, int k, int heads) {
  if (B < 1 || T < 1 || k < 1 || (heads != 64 && heads != DSA_MLA_HEADS)) return 0;
  return dsa::sparse_mla_workspace_size(B, T, k, heads);
}

static int sparse_mla_checked(const uint16_t* q, const uint16_t* kv, const int32_t* idx, int B, int T, int S_max,
                              int k, int heads, float softmax_scale, uint16_t* out, float* lse, void* workspace,
                              size_t ws_bytes, dsa_stream_t stream, uint32_t flags = 0) {
  if ((flags & ~DSA_Q_READY) != 0) return DSA_ERR_INVALID_ARG;
  if (B < 1 || T < 1 || S_max < 1 || k < 1 || !(softmax_scale > 0.f) || !isfinite(softmax_scale))
    return DSA_ERR_INVALID_ARG;
  if ((int64_t)B * T * 2 * 1024 > 0x7fffffffLL) return DSA_ERR_INVALID_ARG;
  if (!q || !kv || !idx || !out) return DSA_ERR_INVALID_ARG;
  if (!dsa_host::aligned16(q) || !dsa_host::aligned16(kv) || !dsa_host::aligned16(idx) ||
      !dsa_host::aligned16(out) || (lse && !dsa_host::aligned16(lse)) ||
      (workspace && !dsa_host::aligned16(workspace)))
    return DSA_ERR_INVALID_ARG;
  int* status;
  int rc = prologue(&status);
  if (rc != DSA_OK) return rc;
  return dsa::launch_sparse_mla(q, kv, idx, B, T, S_max, k, heads, softmax_scale, out, lse, workspace, ws_bytes,
                                (flags & DSA_Q_READY) != 0, (cudaStream_t)stream, status);
}

int dsa_sparse_mla(const uint16_t* q, const uint16_t* kv, const int32_t* idx, int B, int T, int S_max,
                   int k, float softmax_scale, uint16_t* out, float* lse, void* workspace,
                   size_t ws_bytes, dsa_stream_t stream) {
  return sparse_mla_checked(q, kv, idx, B, T, S_max, k, DSA_MLA_HEADS, softmax_scale, out, lse, workspace, ws_bytes,
                            stream);
}

int dsa_sparse_mla_ex(const uint16_t* q, const uint16_t* kv, const int32_t* idx, int B, int T, int S_max, int k,
                      float softmax_scale, uint16_t* out, float* lse, void* workspace, size_t ws_bytes,
                      uint32_t flags, dsa_stream_t stream) {
  return sparse_mla_checked(q, kv, idx, B, T, S_max, k, DSA_MLA_HEADS, softmax_scale, out, lse, workspace, ws_bytes,
                            stream, flags);
}

int dsa_sparse_mla_heads(const uint16_t* q, const uint16_t* kv, const int32_t* idx, int B, int T, int S_max, int k,
                         int heads, float softmax_scale, uint16_t* out, float* lse, void* workspace, size_t ws_bytes,
                         dsa_stream_t stream) {
  if (heads != 64 && heads != DSA_MLA_HEADS) return DSA_ERR_INVALID_ARG;
  return sparse_mla_checked(q, kv, idx, B, T, S_max, k, heads, softmax_scale, out, lse, workspace, ws_bytes, stream);
}

static bool weights_ok(const uint16_t* w, int64_t w_head_stride) {
  return w && dsa_host::aligned16(w) && w_head_stride >= 128 * 512 && w_head_stride % 8 == 0 &&
         w_head_stride <= ((int64_t)1 << 40);
}

int dsa_mla_q_absorb(const uint16_t* q_nope, const uint16_t* q_pe, const int32_t* pos, const float* rope_cs,
                     int max_pos, const uint16_t* w_uk, int64_t w_head_stride, int64_t rows, uint16_t* q_out,
                     dsa_stream_t stream) {
  if (rows < 0 || rows >= 0x80000000LL || max_pos < 1 || !weights_ok(w_uk, w_head_stride)) return DSA_ERR_INVALID_ARG;
  if (!q_nope || !q_pe || !pos || !rope_cs || !q_out) return DSA_ERR_INVALID_ARG;
  const void* ptrs[] = {q_nope, q_pe, pos, rope_cs, q_out};
  for (const void* p : ptrs)
    if (!dsa_host::aligned16(p)) return DSA_ERR_INVALID_ARG;
  if (rows == 0) return DSA_OK;
  int* status;
  int rc = prologue(&status);
  if (rc != DSA_OK) return rc;
  return dsa::launch_mla_q_absorb(q_nope, q_pe, pos, rope_cs, max_pos, w_uk, w_head_stride, rows, q_out,
                                  (cudaStream_t)stream, status);
}

int dsa_mla_kv_entry(const uint16_t* kv, const uint16_t* k_pe, const int32_t* pos, const float* rope_cs,
                     int max_pos, int64_t rows, const int64_t* dst_row, uint16_t* kv_cache, int64_t cache_rows,
                     dsa_stream_t stream) {
  if (rows < 0 || rows >= 0x80000000LL || max_pos < 1 || cache_rows < 1) return DSA_ERR_INVALID_ARG;
  if (!kv || !k_pe || !pos || !rope_cs || !dst_row || !kv_cache) return DSA_ERR_INVALID_ARG;
  const void* ptrs[] = {kv, k_pe, pos, rope_cs, dst_row, kv_cache};
  for (const void* p : ptrs)
    if (!dsa_host::aligned16(p)) return DSA_ERR_INVALID_ARG;
  if (rows == 0) return DSA_OK;
  int* status;
  int rc = prologue(&status);
  if (rc != DSA_OK) return rc;
  return dsa::launch_mla_kv_entry(kv, k_pe, pos, rope_cs, max_pos, rows, dst_row, kv_cache, cache_rows,
                                  (cudaStream_t)stream, status);
}

int dsa_mla_out_absorb(const uint16_t* o, const uint16_t* w_uv, int64_t w_head_stride, int64_t rows, uint16_t* out,
                       dsa_stream_t stream) {
  if (rows < 0 || rows >= 0x80000000LL || !weights_ok(w_uv, w_head_stride)) return DSA_ERR_INVALID_ARG;
  if (!o || !out || !dsa_host::aligned16(o) || !dsa_host::aligned16(out)) return DSA_ERR_INVALID_ARG;
  if (rows == 0) return DSA_OK;
  int* status;
  int rc = prologue(&status);
  if (rc != DSA_OK) return rc;
  return dsa::launch_mla_out_absorb(o, w_uv, w_head_stride, rows, out, (cudaStream_t)stream, status);
}

// Shared checks of the paged-cache arguments: page_size a power of two >= 64; page ids are int32
// and pool rows index int32.
static bool paged_args_ok(int64_t num_pages, const int32_t* block_table, int max_pages, int page_size) {
  if (num_pages < 1 || max_pages < 1 || page_size < 64 || (page_size & (page_size - 1)) != 0) return false;
  if (num_pages * page_size > 0x7fffffffLL || (int64_t)max_pages * page_size > 0x7fffffffLL) return false;
  return block_table != nullptr && (reinterpret_cast<uintptr_t>(block_table) & 3) == 0;
}

int dsa_index_scores_paged(const uint8_t* q8, const float* q_scale, const float* w, const uint8_t* k8_pool,
                           const float* k_scale_pool, int64_t num_pages, const int32_t* block_table, int max_pages,
                           int page_size, const int32_t* q_pos, const int32_t* kv_len, int B, int T,
                           float softmax_scale, float* scores, int64_t ld, uint32_t flags, dsa_stream_t stream) {
  if (!paged_args_ok(num_pages, block_table, max_pages, page_size)) return DSA_ERR_INVALID_ARG;
  const int64_t S_max = (int64_t)max_pages * page_size;
  if (B < 1 || T < 1 || ld < S_max || (ld & 3) != 0 || (flags & ~DSA_FILL_MASKED) != 0 ||
      !(softmax_scale > 0.f) || !isfinite(softmax_scale))
    return DSA_ERR_INVALID_ARG;
  if ((int64_t)B * T * 64 > 0x7fffffffLL) return DSA_ERR_INVALID_ARG;
  if (!q8 || !q_scale || !w || !k8_pool || !k_scale_pool || !q_pos || !kv_len || !scores) return DSA_ERR_INVALID_ARG;
  const void* ptrs[] = {q8, q_scale, w, k8_pool, k_scale_pool, q_pos, kv_len, scores};
  for (const void* p : ptrs)
    if (!dsa_host::aligned16(p)) return DSA_ERR_INVALID_ARG;
  int* status;
  int rc = prologue(&status);
  if (rc != DSA_OK) return rc;
  return dsa::launch_index_scores_paged(q8, q_scale, w, k8_pool, k_scale_pool, num_pages, block_table, max_pages,
                                        page_size, q_pos, kv_len, B, T, softmax_scale, scores, ld, flags,
                                        (cudaStream_t)stream, status);
}

int dsa_sparse_mla_paged(const uint16_t* q, const uint16_t* kv_pool, int64_t num_pages, const int32_t* block_table,
                         int max_pages, int page_size, const int32_t* idx, int B, int T, int k, float softmax_scale,
                         uint16_t* out, float* lse, void* workspace, size_t ws_bytes, dsa_stream_t stream) {
  if (!paged_args_ok(num_pages, block_table, max_pages, page_size)) return DSA_ERR_INVALID_ARG;
  if (B < 1 || T < 1 || k < 1 || !(softmax_scale > 0.f) || !isfinite(softmax_scale)) return DSA_ERR_INVALID_ARG;
  if ((int64_t)B * T * 2 * 1024 > 0x7fffffffLL) return DSA_ERR_INVALID_ARG;
  if (!q || !kv_pool || !idx || !out) return DSA_ERR_INVALID_ARG;
  if (!dsa_host::aligned16(q) || !dsa_host::aligned16(kv_pool) || !dsa_host::aligned16(idx) ||
      !dsa_host::aligned16(out) || (lse && !dsa_host::aligned16(lse)) ||
      (workspace && !dsa_host::aligned16(workspace)))
    return DSA_ERR_INVALID_ARG;
  int* status;
  int rc = prologue(&status);
  if (rc != DSA_OK) return rc;
  return dsa::launch_sparse_mla_paged(q, kv_pool, num_pages, block_table, max_pages, page_size, idx, B, T, k,
                                      softmax_scale, out, lse, workspace, ws_bytes, (cudaStream_t)stream, status);
}

int dsa_get_device_status(dsa_stream_t stream) {
  DeviceCache* c = device_cache();
  if (!c) return DSA_ERR_CUDA;
  if (cudaStreamSynchronize((cudaStream_t)stream) != cudaSuccess) return DSA_ERR_CUDA;
  int v[4] = {0, 0, 0, 0};
  if (cudaMemcpy(v, c->status, sizeof(v), cudaMemcpyDeviceToHost) != cudaSuccess) return DSA_ERR_CUDA;
  if (v[0] != 0) {
    c->detail[0] = v[0] == DSA_ERR_TIMEOUT ? v[1] : 0;
    c->detail[1] = v[0] == DSA_ERR_TIMEOUT ? v[2] : 0;
    c->detail[2] = v[0] == DSA_ERR_TIMEOUT ? v[3] : 0;
    const int zero[4] = {0, 0, 0, 0};
    if (cudaMemcpy(c->status, zero, sizeof(zero), cudaMemcpyHostToDevice) != cudaSuccess) return DSA_ERR_CUDA;
  }
  return v[0];
}

int dsa_get_error_detail(int* site, int* block, int* wait_us) {
  DeviceCache* c = device_cache();
  if (!c) return DSA_ERR_CUDA;
  if (site) *site = c->detail[0];
  if (block) *block = c->detail[1];
  if (wait_us) *wait_us = c->detail[2];
  return DSA_OK;
}

int dsa_selftest_wait_timeout(dsa_stream_t stream) {
  int* status;
  int rc = prologue(&status);
  if (rc != DSA_OK) return rc;
  selftest_wait_kernel<<<1, 32, 0, (cudaStream_t)stream>>>(status);
  return dsa_host::check_launch();
}

const char* dsa_status_string(int code) {
  switch (code) {
    case DSA_OK: return "DSA_OK";
    case DSA_ERR_INVALID_ARG: return "DSA_ERR_INVALID_ARG";
    case DSA_ERR_UNSUPPORTED: return "DSA_ERR_UNSUPPORTED";
    case DSA_ERR_CUDA: return "DSA_ERR_CUDA";
    case DSA_ERR_TIMEOUT: return "DSA_ERR_TIMEOUT";
    case DSA_ERR_DEVICE_BOUNDS: return "DSA_ERR_DEVICE_BOUNDS";
    case DSA_ERR_WORKSPACE: return "DSA_ERR_WORKSPACE";
    default: return "DSA_ERR_UNKNOWN";
  }
}

int dsa_device_supported(void) {
  DeviceCache* c = device_cache();
  return (c && c->supported) ? 1 : 0;
}

const char* dsa_version(void) { return "dsa-b200 0.1.0"; }

}  // extern "C"
