// hsa_decode_step_noalloc: the decode step with its scratch in a static
// device array instead of a caller-provided workspace, for callers that
// cannot allocate device memory when they decode.
#include <mutex>

#include "hsa.h"
#include "kernels.cuh"

namespace {

// One copy per device that loads the library, alive until the process exits.
__device__ __align__(256) unsigned char g_noalloc_scratch[HSA_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
void* g_scratch_ptr[kMaxDevices];
std::mutex g_scratch_mu;

// Device address of this device's array. In host code the array's name only
// stands in for the symbol; its device address has to be looked up, once per
// device, with that device current.
int scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return HSA_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return HSA_ERR_CUDA;
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return HSA_OK;
}

}  // namespace

extern "C" int hsa_decode_step_noalloc(const hsa_params* p, int32_t batch, int64_t capacity,
                                       int32_t* ctx_len, hsa_bf16* k_idx_cache, hsa_bf16* K_cache,
                                       hsa_bf16* V_cache, float* ksum_cache,
                                       const hsa_bf16* q_idx_new, const hsa_bf16* k_idx_new,
                                       const hsa_bf16* Q_new, const hsa_bf16* K_new,
                                       const hsa_bf16* V_new, hsa_bf16* O, int32_t* indices_out,
                                       cudaStream_t stream) {
  size_t need = 0;
  if (int e = hsa_decode_workspace_size(p, batch, capacity, &need)) return e;
  if (need > HSA_NOALLOC_SCRATCH_BYTES) return HSA_ERR_WORKSPACE;
  void* scratch = nullptr;
  if (int e = scratch_address(&scratch)) return e;
  // Every scratch region of the decode step is written before it is read
  // within the step, so stale contents from an earlier call are harmless.
  return hsa_decode_step(p, batch, capacity, ctx_len, k_idx_cache, K_cache, V_cache, ksum_cache,
                         q_idx_new, k_idx_new, Q_new, K_new, V_new, O, indices_out, scratch,
                         HSA_NOALLOC_SCRATCH_BYTES, stream);
}
