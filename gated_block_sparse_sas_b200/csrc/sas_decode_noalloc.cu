// Allocation-free decode: sas_decode with its scratch in a fixed device array that lives
// inside this library, so the caller passes only inputs and outputs.
//
// Who needs this: callers that cannot call cudaMalloc (or any allocator) around a decode
// step -- e.g. an inference runtime whose memory pool has already reserved the device
// memory, a plugin invoked from another framework's step where an extra allocation could
// fail or force a device-wide synchronisation, or a latency-critical loop that must not
// touch the allocator at all. They get the same kernels as sas_decode; only the origin of
// the scratch differs.
//
// Cost and limits: every GPU that loads this library holds kNoAllocScratchBytes of device
// memory for the scratch until the process exits. A problem whose scratch need (the size
// sas_decode_workspace_size reports) exceeds that is rejected with SAS_ERR_UNSUPPORTED.
// All calls on a device share the one array: calls whose kernels overlap on the GPU (two
// streams, or two threads) race on it, so serialise them. The array keeps whatever the
// previous call left; the decode kernels write every scratch element they later read, and
// the one word that must start at zero -- the error word, the array's first int32 -- is
// cleared by each call on its stream (cudaMemsetAsync, which allocates nothing).
// sas_decode_noalloc_error_word hands out that word's device address so the caller can read
// the status of its last call.
//
// The address of the array is looked up once per device ordinal and cached. The stream must
// belong to the current device, and a cudaDeviceReset of that device (which would reload the
// module at a new address) is not supported while the library stays loaded.
#include <mutex>

#include "sas_common.cuh"
#include "sas_kernels.h"

namespace sas {

constexpr size_t kNoAllocScratchBytes = (size_t)8 << 20;   // 8 MiB per device

static __device__ __align__(256) unsigned char g_decode_scratch[kNoAllocScratchBytes];

static std::mutex g_scratch_mu;
static void* g_scratch_addr[256] = {};   // device address of g_decode_scratch, per ordinal

// The device address of the scratch on the current device. The host-side name
// g_decode_scratch is only a stand-in for the symbol, never a device pointer, so the
// address is looked up once per device (with that device current) and cached.
static sas_status scratch_on_current_device(void** out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) {
    set_error("sas_decode_noalloc: cudaGetDevice failed: %s", cudaGetErrorString(e));
    return SAS_ERR_CUDA;
  }
  if (dev < 0 || dev >= 256) {
    set_error("sas_decode_noalloc: device ordinal %d out of range", dev);
    return SAS_ERR_UNSUPPORTED;
  }
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (g_scratch_addr[dev] == nullptr) {
    void* ptr = nullptr;
    e = cudaGetSymbolAddress(&ptr, g_decode_scratch);
    if (e != cudaSuccess || ptr == nullptr) {
      set_error("sas_decode_noalloc: cudaGetSymbolAddress failed: %s", cudaGetErrorString(e));
      return SAS_ERR_CUDA;
    }
    g_scratch_addr[dev] = ptr;
  }
  *out = g_scratch_addr[dev];
  return SAS_OK;
}

}  // namespace sas

extern "C" sas_status sas_decode_noalloc(const sas_decode_problem* p, const void* q,
                                         const void* q_nope, const void* k_cache,
                                         const void* v_cache, const void* gate_key_cache,
                                         const float* cur_pool, const void* wq,
                                         const float* qnorm_w, const void* wk,
                                         const float* knorm_w, void* o, int32_t* idx_out,
                                         float* logg_out, cudaStream_t stream) {
  size_t need = 0;
  const sas_status st = sas_decode_workspace_size(p, &need);   // also validates p
  if (st != SAS_OK) return st;
  if (need > sas::kNoAllocScratchBytes) {
    sas::set_error("sas_decode_noalloc: this problem needs %zu bytes of scratch but the "
                   "built-in scratch holds %zu; use sas_decode with a caller workspace",
                   need, sas::kNoAllocScratchBytes);
    return SAS_ERR_UNSUPPORTED;
  }
  void* scratch = nullptr;
  const sas_status s2 = sas::scratch_on_current_device(&scratch);
  if (s2 != SAS_OK) return s2;
  return sas_decode(p, q, q_nope, k_cache, v_cache, gate_key_cache, cur_pool, wq, qnorm_w, wk,
                    knorm_w, o, idx_out, logg_out, scratch, sas::kNoAllocScratchBytes, stream);
}

extern "C" sas_status sas_decode_noalloc_error_word(const int32_t** word) {
  if (word == nullptr) {
    sas::set_error("sas_decode_noalloc_error_word: word is NULL");
    return SAS_ERR_INVALID_ARG;
  }
  void* scratch = nullptr;
  const sas_status st = sas::scratch_on_current_device(&scratch);
  if (st != SAS_OK) return st;
  *word = static_cast<const int32_t*>(scratch);   // word 0 of the scratch: the error code
  return SAS_OK;
}
