// append.cu -- copy newly generated tokens into the FP16 block (SemKV, Fig. 6:
// new tokens are held back and quantized block-exactly, the most recent
// partial block stays FP16 during decoding).
#include "common.cuh"
#include "internal.h"

namespace semkv {

// rows = B*Lyr*H*take of K and V; one thread per 16-byte chunk; plus the scores
__global__ void buffer_append_kernel(const uint16_t *__restrict__ k_new,
                                     const uint16_t *__restrict__ v_new,
                                     const float *__restrict__ score_new, int n_total, int i0,
                                     int take, int slabs, int B, int block, int buf_len,
                                     uint16_t *__restrict__ bk, uint16_t *__restrict__ bv,
                                     float *__restrict__ bscore) {
  const int64_t nchunk = (int64_t)slabs * take * 16;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < 2 * nchunk;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int kv = i >= nchunk;
    const int64_t j = kv ? i - nchunk : i;
    const int ch = (int)(j & 15);
    const int64_t rt = j >> 4;                 // slab * take + t
    const int t = (int)(rt % take);
    const int64_t slab = rt / take;
    const uint4 *src = reinterpret_cast<const uint4 *>((kv ? v_new : k_new) +
                                                       (slab * n_total + i0 + t) * kD) + ch;
    uint4 *dst = reinterpret_cast<uint4 *>((kv ? bv : bk) + (slab * block + buf_len + t) * kD) + ch;
    *dst = *src;
  }
  const int64_t tid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (tid < (int64_t)B * take) {
    const int b = (int)(tid / take), t = (int)(tid % take);
    bscore[(int64_t)b * block + buf_len + t] = score_new[(int64_t)b * n_total + i0 + t];
  }
}

cudaError_t launch_buffer_append(const semkv_cache &c, const uint16_t *k_new,
                                 const uint16_t *v_new, const float *score_new, int n_total,
                                 int i0, int take, cudaStream_t st) {
  if (take <= 0) return cudaSuccess;
  const int slabs = c.B * c.n_layers * c.H;
  const int64_t work = 2ll * slabs * take * 16;
  int64_t blocks = (work + 255) / 256;
  const int64_t minb = ((int64_t)c.B * take + 255) / 256;
  if (blocks < minb) blocks = minb;
  if (blocks > 4096) blocks = 4096;
  buffer_append_kernel<<<(unsigned)blocks, 256, 0, st>>>(k_new, v_new, score_new, n_total, i0, take,
                                                          slabs, c.B, c.block, c.buf_len, c.buf_k,
                                                          c.buf_v, c.buf_score);
  return cudaGetLastError();
}

}  // namespace semkv
