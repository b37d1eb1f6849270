// noalloc.cu -- semkv_quantize for callers that cannot allocate device memory.
//
// semkv_quantize needs a caller-provided workspace (the per-token slot array
// and the per-sequence high counts).  Some callers have no way to provide one:
// an inference engine that has handed all device memory to its own pool
// allocator, or a plugin host that forbids cudaMalloc on its hot path.  This
// entry point gives them the same computation with the workspace taken from a
// fixed array in this file's device memory instead.
//
// The array is a file-scope __device__ object, so every GPU that loads the
// library holds SEMKV_NOALLOC_SCRATCH_BYTES of it until the process exits.
// Host code cannot use the array's name as a device address; its address is
// looked up once per device with cudaGetSymbolAddress, with that device
// current, on the first call made on the device.
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>

#include "../../include/semkv.h"

namespace {

constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_quant_scratch[SEMKV_NOALLOC_SCRATCH_BYTES];

std::mutex g_setup_mutex;
void *g_scratch_addr[kMaxDevices] = {};

// Device address of g_quant_scratch on the current device (set up once per device).
semkv_status scratch_address(void **out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return SEMKV_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_setup_mutex);
  if (g_scratch_addr[dev] == nullptr) {
    void *p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_quant_scratch);
    if (e != cudaSuccess || p == nullptr) return SEMKV_ERR_CUDA;
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return SEMKV_OK;
}

}  // namespace

extern "C" semkv_status semkv_quantize_noalloc(semkv_cache *c, const uint16_t *k, const uint16_t *v,
                                               int32_t T_max, const int32_t *seq_len,
                                               const uint8_t *mask, uint32_t *status, void *stream) {
  if (c == nullptr || c->B <= 0 || T_max <= 0) return SEMKV_ERR_INVALID_ARG;
  const size_t need = semkv_quantize_workspace_size(c->B, T_max);
  if (need == 0) return SEMKV_ERR_INVALID_ARG;
  if (need > (size_t)SEMKV_NOALLOC_SCRATCH_BYTES) return SEMKV_ERR_WORKSPACE;   // B*T_max too large
  void *scratch = nullptr;
  const semkv_status s = scratch_address(&scratch);
  if (s != SEMKV_OK) return s;
  // every entry the kernels read is written first by this call (slot of each
  // live token, high count of each sequence), so nothing needs clearing
  return semkv_quantize(c, k, v, T_max, seq_len, mask, scratch, (size_t)SEMKV_NOALLOC_SCRATCH_BYTES,
                        status, stream);
}
