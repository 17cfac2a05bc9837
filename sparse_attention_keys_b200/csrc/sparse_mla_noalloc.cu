// dsa_sparse_mla_noalloc: dsa_sparse_mla for callers that cannot allocate device memory.
//
// dsa_sparse_mla needs a scratch buffer for its split-KV partial results, which the caller
// normally allocates and passes in. Some callers cannot do that: code embedded in a host
// framework whose memory manager owns every device allocation (a raw cudaMalloc would bypass
// its accounting or exceed its pool cap), or a latency-critical serving loop that must not call
// cudaMalloc/cudaFree because those can synchronise the whole device. This entry point takes
// the scratch from a fixed array compiled into the library instead, so the call allocates
// nothing. The caller still owns and passes every input and output buffer.
//
// The array below is kNoAllocScratchBytes (32 MiB) of device memory that every GPU which loads
// the library keeps until the process exits. Host code cannot use the array's name as a device
// address (on the host it names a stand-in object), so the device address is looked up once per
// device with cudaGetSymbolAddress while that device is current, and passed to the kernels.
#include <cuda_runtime.h>
#include <math.h>

#include <mutex>

#include "common.cuh"
#include "dsa.h"
#include "kernels.h"

namespace {

constexpr size_t kNoAllocScratchBytes = size_t(32) << 20;

static __device__ __align__(256) unsigned char g_mla_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
void* g_scratch_addr[kMaxDevices] = {nullptr};
std::mutex g_scratch_mu;

// Device address of g_mla_scratch on the current device (set up on the first call per device).
int scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return DSA_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_scratch_mu);
  if (g_scratch_addr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_mla_scratch) != cudaSuccess || p == nullptr) return DSA_ERR_CUDA;
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return DSA_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

extern "C" {

DSA_API size_t dsa_sparse_mla_noalloc_scratch_bytes(void) { return kNoAllocScratchBytes; }

DSA_API int dsa_sparse_mla_noalloc(const uint16_t* q, const uint16_t* kv, const int32_t* idx, int B, int T,
                                   int S_max, int k, float softmax_scale, uint16_t* out, float* lse,
                                   dsa_stream_t stream) {
  if (B < 1 || T < 1 || S_max < 1 || k < 1 || !(softmax_scale > 0.f) || !isfinite(softmax_scale))
    return DSA_ERR_INVALID_ARG;
  if ((int64_t)B * T * 2 * 1024 > 0x7fffffffLL) return DSA_ERR_INVALID_ARG;
  if (!q || !kv || !idx || !out) return DSA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(kv) || !aligned16(idx) || !aligned16(out) || (lse && !aligned16(lse)))
    return DSA_ERR_INVALID_ARG;
  if (!dsa_device_supported()) return DSA_ERR_UNSUPPORTED;
  const size_t need = dsa::sparse_mla_workspace_size(B, T, k);
  if (need > kNoAllocScratchBytes) return DSA_ERR_WORKSPACE;   // shape needs more than the fixed array
  int* status = dsa_host::status_word();
  if (!status) return DSA_ERR_CUDA;
  void* scratch = nullptr;
  const int rc = scratch_address(&scratch);
  if (rc != DSA_OK) return rc;
  return dsa::launch_sparse_mla(q, kv, idx, B, T, S_max, k, softmax_scale, out, lse, scratch,
                                kNoAllocScratchBytes, (cudaStream_t)stream, status);
}

}  // extern "C"
