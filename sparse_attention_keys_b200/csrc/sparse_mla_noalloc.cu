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
// address (on the host it names a stand-in object), so the device address is looked up with
// cudaGetSymbolAddress while the device is current, once per device context (again if the
// context is re-created, e.g. after cudaDeviceReset), and passed to the kernels. Argument checks
// and the launch are those of dsa_sparse_mla itself, which this call forwards to.
#include <cuda_runtime.h>

#include <mutex>

#include "common.cuh"
#include "dsa.h"
#include "kernels.h"

namespace {

constexpr size_t kNoAllocScratchBytes = size_t(32) << 20;

static __device__ __align__(256) unsigned char g_mla_scratch[kNoAllocScratchBytes];

uint64_t g_scratch_ctx[dsa_host::kMaxSetupDevices] = {};   // context each address below belongs to
void* g_scratch_addr[dsa_host::kMaxSetupDevices] = {nullptr};
std::mutex g_scratch_mu;

// Device address of g_mla_scratch in the current device's context (looked up on the first call
// in each context).
int scratch_address(void** out) {
  int dev = 0;
  std::lock_guard<std::mutex> lk(g_scratch_mu);
  if (dsa_host::needs_setup(g_scratch_ctx, &dev)) {
    if (dev < 0 || dev >= dsa_host::kMaxSetupDevices) return DSA_ERR_CUDA;
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_mla_scratch) != cudaSuccess || p == nullptr) return DSA_ERR_CUDA;
    g_scratch_addr[dev] = p;
    dsa_host::mark_setup(g_scratch_ctx);
  }
  *out = g_scratch_addr[dev];
  return *out ? DSA_OK : DSA_ERR_CUDA;
}

}  // namespace

extern "C" {

DSA_API size_t dsa_sparse_mla_noalloc_scratch_bytes(void) { return kNoAllocScratchBytes; }

DSA_API int dsa_sparse_mla_noalloc(const uint16_t* q, const uint16_t* kv, const int32_t* idx, int B, int T,
                                   int S_max, int k, float softmax_scale, uint16_t* out, float* lse,
                                   dsa_stream_t stream) {
  if (B < 1 || T < 1 || k < 1) return DSA_ERR_INVALID_ARG;
  if (dsa_sparse_mla_workspace_size(B, T, k) > kNoAllocScratchBytes)
    return DSA_ERR_WORKSPACE;                          // the shape needs more than the fixed array
  if (!dsa_device_supported()) return DSA_ERR_UNSUPPORTED;
  void* scratch = nullptr;
  const int rc = scratch_address(&scratch);
  if (rc != DSA_OK) return rc;
  return dsa_sparse_mla(q, kv, idx, B, T, S_max, k, softmax_scale, out, lse, scratch, kNoAllocScratchBytes,
                        stream);
}

}  // extern "C"
