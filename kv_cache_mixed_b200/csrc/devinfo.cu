// devinfo.cu -- per-device host caches for the launchers: the SM count, the
// dynamic shared-memory attributes of each kernel and its occupancy.  Each is
// queried from the runtime once per (device, kernel) instead of on every call,
// which matters for the many small launches of the generation path.
#include <cuda.h>
#include <cuda_runtime.h>

#include <map>
#include <mutex>
#include <tuple>

#include "internal.h"

namespace semkv {

namespace {
std::mutex g_mu;
std::map<int, int> g_sms;                                              // device -> SMs
std::map<std::pair<int, const void *>, int> g_smem;                    // (device, kernel) -> bytes set
std::map<std::tuple<int, const void *, int, int>, int> g_occ;          // (device, kernel, threads, smem) -> CTAs/SM
}  // namespace

int device_sm_count() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 1;
  std::lock_guard<std::mutex> lock(g_mu);
  auto it = g_sms.find(dev);
  if (it != g_sms.end()) return it->second;
  int sms = 0;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms < 1) sms = 1;
  g_sms[dev] = sms;
  return sms;
}

cudaError_t prepare_kernel(const void *fn, int smem_bytes) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(g_mu);
  auto key = std::make_pair(dev, fn);
  auto it = g_smem.find(key);
  if (it != g_smem.end() && it->second >= smem_bytes) return cudaSuccess;
  e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_bytes);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(fn, cudaFuncAttributePreferredSharedMemoryCarveout, cudaSharedmemCarveoutMaxShared);
  if (e != cudaSuccess) return e;
  g_smem[key] = smem_bytes;
  return cudaSuccess;
}

// cuTensorMapEncodeTiled from the driver, looked up once through the runtime
// (the library links the runtime only)
typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

cudaError_t encode_tensor_map_f16(CUtensorMap *map, const void *base, int rank, const uint64_t *dims,
                                  const uint64_t *strides_bytes, const uint32_t *box, bool swizzle128) {
  static EncodeTiledFn fn = nullptr;
  {
    std::lock_guard<std::mutex> lock(g_mu);
    if (!fn) {
      void *f = nullptr;
      cudaDriverEntryPointQueryResult q;
      cudaError_t e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q);
      if (e != cudaSuccess) return e;
      if (q != cudaDriverEntryPointSuccess || !f) return cudaErrorNotSupported;
      fn = reinterpret_cast<EncodeTiledFn>(f);
    }
  }
  cuuint64_t gd[5], gs[4];
  cuuint32_t bx[5], es[5];
  for (int i = 0; i < rank; ++i) {
    gd[i] = dims[i];
    bx[i] = box[i];
    es[i] = 1;
    if (i + 1 < rank) gs[i] = strides_bytes[i];
  }
  const CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, (cuuint32_t)rank, const_cast<void *>(base), gd, gs, bx,
                        es, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        swizzle128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

cudaError_t kernel_occupancy(const void *fn, int threads, int smem_bytes, int *ctas_per_sm) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(g_mu);
  auto key = std::make_tuple(dev, fn, threads, smem_bytes);
  auto it = g_occ.find(key);
  if (it != g_occ.end()) {
    *ctas_per_sm = it->second;
    return cudaSuccess;
  }
  int nb = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&nb, fn, threads, smem_bytes);
  if (e != cudaSuccess) return e;
  if (nb < 1) nb = 1;
  g_occ[key] = nb;
  *ctas_per_sm = nb;
  return cudaSuccess;
}

}  // namespace semkv
