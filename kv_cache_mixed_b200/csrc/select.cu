// select.cu -- per-prompt top-r selection (SemKV, Fig. 2: rank within each
// prompt, no normalisation needed; Fig. 4: the top-r get the high level, no
// score threshold is estimated).
//
// One CTA per sequence.  Scores map to order-preserving 32-bit keys (-0 made
// +0 first); an MSB-first 8-bit radix select finds the key K* of the
// ceil(r*len)-th largest score using shared-memory histograms (integer counts,
// so the result does not depend on the order of the atomic adds); tokens with
// key > K* are high, and among keys == K* the lowest token indices are taken,
// found with a block-wide scan in index order.  Bit-exact and deterministic.
#include "common.cuh"
#include "internal.h"

namespace semkv {

constexpr int SEL_THREADS = 1024;
constexpr int SEL_SMEM_KEYS = 49152;          // sequences up to this length keep keys in smem

__device__ __forceinline__ uint32_t order_key(float s) {
  const float f = __fadd_rn(s, 0.0f);          // -0 -> +0
  const uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__global__ void __launch_bounds__(SEL_THREADS)
select_kernel(const float *__restrict__ score, int64_t score_bstride,
              const int32_t *__restrict__ seq_len, int len_const, int T_max, int r_ppm,
              uint8_t *__restrict__ mask, int64_t mask_bstride, uint32_t *status, int cache_keys) {
  extern __shared__ uint32_t keys[];
  __shared__ uint32_t hist[256];
  __shared__ int sh_scan[33];
  __shared__ uint32_t sh_bucket, sh_above;
  __shared__ int sh_nan;

  const int b = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const float *sc = score + (int64_t)b * score_bstride;
  uint8_t *mk = mask + (int64_t)b * mask_bstride;
  int len = seq_len ? seq_len[b] : len_const;
  if (len < 0 || len > T_max) {
    if (tid == 0) set_flag(status, SEMKV_FLAG_SEQLEN);
    for (int t = tid; t < T_max; t += SEL_THREADS) mk[t] = 0;
    return;
  }
  for (int t = len + tid; t < T_max; t += SEL_THREADS) mk[t] = 0;
  const int64_t nh64 = ((int64_t)r_ppm * len + 999999) / 1000000;
  const int n_high = (int)nh64;

  if (tid == 0) sh_nan = 0;
  __syncthreads();
  const bool cached = cache_keys && len <= SEL_SMEM_KEYS;
  {
    int nan_seen = 0;
    for (int t = tid; t < len; t += SEL_THREADS) {
      const float s = sc[t];
      nan_seen |= isnan(s);
      if (cached) keys[t] = order_key(s);
    }
    if (__any_sync(0xffffffffu, nan_seen) && lane == 0) sh_nan = 1;
  }
  __syncthreads();
  if (sh_nan && tid == 0) set_flag(status, SEMKV_FLAG_NONFINITE);
  if (n_high == 0 || n_high == len) {
    const uint8_t v = n_high == 0 ? 0 : 1;
    for (int t = tid; t < len; t += SEL_THREADS) mk[t] = v;
    return;
  }
  auto key_at = [&](int t) -> uint32_t { return cached ? keys[t] : order_key(sc[t]); };

  // ---- radix select: K* = the n_high-th largest key
  uint32_t prefix = 0;
  uint32_t k = (uint32_t)n_high;      // rank (1-based) of K* among keys matching the prefix
  uint32_t cnt_eq = 0;
#pragma unroll 1
  for (int pass = 0; pass < 4; ++pass) {
    const int shift = 24 - 8 * pass;
    for (int i = tid; i < 256; i += SEL_THREADS) hist[i] = 0;
    __syncthreads();
    const uint32_t hmask = pass == 0 ? 0u : (0xFFFFFFFFu << (shift + 8));
    for (int t = tid; t < len; t += SEL_THREADS) {
      const uint32_t key = key_at(t);
      if ((key & hmask) == prefix) atomicAdd(&hist[(key >> shift) & 255u], 1u);
    }
    __syncthreads();
    if (warp == 0) {
      // lane l owns bins 255-8l .. 248-8l (descending)
      uint32_t h[8], s = 0;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        h[j] = hist[255 - 8 * lane - j];
        s += h[j];
      }
      uint32_t incl = s;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      const uint32_t hit = __ballot_sync(0xffffffffu, incl >= k);
      const int lstar = __ffs(hit) - 1;   // k <= total, so some lane hits
      if (lane == lstar) {
        uint32_t above = incl - s;
        int bucket = 255 - 8 * lane;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          if (above + h[j] >= k) {
            bucket = 255 - 8 * lane - j;
            break;
          }
          above += h[j];
        }
        sh_bucket = (uint32_t)bucket;
        sh_above = above;
      }
    }
    __syncthreads();
    const uint32_t bucket = sh_bucket;
    k -= sh_above;
    prefix |= bucket << shift;
    cnt_eq = hist[bucket];
    __syncthreads();
  }
  const uint32_t kstar = prefix;

  if (k == cnt_eq) {
    // every key equal to K* is taken: no ordering needed
    for (int t = tid; t < len; t += SEL_THREADS) mk[t] = key_at(t) >= kstar ? 1 : 0;
    return;
  }
  // ---- ties at K*: take the k lowest token indices among keys == K*
  uint32_t carry = 0;
  for (int base = 0; base < len; base += 4 * SEL_THREADS) {
    const int t0 = base + 4 * tid;
    uint32_t kk[4];
    int eq = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      kk[i] = (t0 + i < len) ? key_at(t0 + i) : 0u;
      eq += (t0 + i < len) && kk[i] == kstar;
    }
    // block exclusive scan of eq
    int x = eq;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      int y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    if (lane == 31) sh_scan[warp] = x;
    __syncthreads();
    if (warp == 0) {
      int tt = sh_scan[lane];
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        int y = __shfl_up_sync(0xffffffffu, tt, o);
        if (lane >= o) tt += y;
      }
      sh_scan[lane] = tt;
      if (lane == 31) sh_scan[32] = tt;
    }
    __syncthreads();
    uint32_t rank = carry + (uint32_t)(x - eq + (warp ? sh_scan[warp - 1] : 0));
    const uint32_t total = (uint32_t)sh_scan[32];
    __syncthreads();
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int t = t0 + i;
      if (t < len) {
        uint8_t v = kk[i] > kstar ? 1 : 0;
        if (kk[i] == kstar) {
          v = rank < k ? 1 : 0;
          ++rank;
        }
        mk[t] = v;
      }
    }
    carry += total;
  }
}

cudaError_t launch_select(const float *score, int64_t score_bstride, const int32_t *seq_len,
                          int len_const, int B, int T_max, int r_ppm, uint8_t *mask,
                          int64_t mask_bstride, uint32_t *status, cudaStream_t st) {
  const int cache = T_max <= SEL_SMEM_KEYS ? 1 : 0;
  const size_t smem = cache ? (size_t)T_max * 4 : 0;
  cudaError_t e = prepare_kernel(reinterpret_cast<const void *>(select_kernel), SEL_SMEM_KEYS * 4);   // once per device
  if (e != cudaSuccess) return e;
  select_kernel<<<B, SEL_THREADS, smem, st>>>(score, score_bstride, seq_len, len_const, T_max,
                                              r_ppm, mask, mask_bstride, status, cache);
  return cudaGetLastError();
}

}  // namespace semkv
