// select.cu -- per-prompt top-r selection (SemKV, Fig. 2: rank within each
// prompt, no normalisation needed; Fig. 4: the top-r get the high level, no
// score threshold is estimated).
//
// One cluster of 8 CTAs per sequence; CTA c of the cluster owns the tokens
// [c*seg, (c+1)*seg) of the sequence.  Scores map to order-preserving 32-bit
// keys (-0 made +0 first), kept in each CTA's shared memory; an MSB-first 8-bit
// radix select finds the key K* of the ceil(r*len)-th largest score: each pass
// every CTA builds the histogram of its own keys (integer counts, so the order
// of the atomic adds does not matter), the cluster barrier publishes them, and
// every CTA sums the 8 histograms through distributed shared memory and finds
// the same bucket.  Tokens with key > K* are high; among keys == K* the lowest
// token indices are taken: a CTA starts its in-order scan of its own ties after
// the tie counts of the CTAs before it.  Bit-exact and deterministic.
#include <cooperative_groups.h>

#include "common.cuh"
#include "internal.h"

namespace semkv {

namespace cg = cooperative_groups;

constexpr int SEL_CLUSTER = 8;                // CTAs per sequence (a portable cluster size)
constexpr int SEL_THREADS = 512;
constexpr int SEL_SEG_KEYS = 16384;           // a CTA keeps up to this many keys in shared memory

__device__ __forceinline__ uint32_t order_key(float s) {
  const float f = __fadd_rn(s, 0.0f);          // -0 -> +0
  const uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__global__ void __cluster_dims__(SEL_CLUSTER, 1, 1) __launch_bounds__(SEL_THREADS)
select_kernel(const float *__restrict__ score, int64_t score_bstride,
              const int32_t *__restrict__ seq_len, int len_const, int T_max, int r_ppm,
              uint8_t *__restrict__ mask, int64_t mask_bstride, uint32_t *status, int cache_keys) {
  extern __shared__ uint32_t keys[];
  __shared__ uint32_t hist[256];               // this CTA's counts (read by the whole cluster)
  __shared__ uint32_t tot[256];                // the cluster's counts
  __shared__ int sh_scan[33];
  __shared__ uint32_t sh_bucket, sh_above, sh_eq;
  __shared__ int sh_nan;

  cg::cluster_group cluster = cg::this_cluster();
  const int rank = (int)cluster.block_rank();
  const int b = blockIdx.y;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const float *sc = score + (int64_t)b * score_bstride;
  uint8_t *mk = mask + (int64_t)b * mask_bstride;
  int len = seq_len ? seq_len[b] : len_const;
  // (every CTA of a cluster sees the same length, so all take the same branches
  // below: the cluster barriers are reached by all or by none)
  if (len < 0 || len > T_max) {
    if (tid == 0 && rank == 0) set_flag(status, SEMKV_FLAG_SEQLEN);
    for (int t = rank * SEL_THREADS + tid; t < T_max; t += SEL_CLUSTER * SEL_THREADS) mk[t] = 0;
    return;
  }
  for (int t = len + rank * SEL_THREADS + tid; t < T_max; t += SEL_CLUSTER * SEL_THREADS) mk[t] = 0;
  const int64_t nh64 = ((int64_t)r_ppm * len + 999999) / 1000000;
  const int n_high = (int)nh64;
  const int seg = (len + SEL_CLUSTER - 1) / SEL_CLUSTER;
  const int lo = min(len, rank * seg), hi = min(len, lo + seg);

  if (tid == 0) sh_nan = 0;
  __syncthreads();
  const bool cached = cache_keys != 0;
  {
    int nan_seen = 0;
    for (int t = lo + tid; t < hi; t += SEL_THREADS) {
      const float s = sc[t];
      nan_seen |= isnan(s);
      if (cached) keys[t - lo] = order_key(s);
    }
    if (__any_sync(0xffffffffu, nan_seen) && lane == 0) sh_nan = 1;
  }
  __syncthreads();
  if (sh_nan && tid == 0) set_flag(status, SEMKV_FLAG_NONFINITE);
  if (n_high == 0 || n_high == len) {
    const uint8_t v = n_high == 0 ? 0 : 1;
    for (int t = lo + tid; t < hi; t += SEL_THREADS) mk[t] = v;
    return;
  }
  auto key_at = [&](int t) -> uint32_t { return cached ? keys[t - lo] : order_key(sc[t]); };

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
    for (int t = lo + tid; t < hi; t += SEL_THREADS) {
      const uint32_t key = key_at(t);
      if ((key & hmask) == prefix) atomicAdd(&hist[(key >> shift) & 255u], 1u);
    }
    cluster.sync();                    // every CTA's histogram is complete
    for (int i = tid; i < 256; i += SEL_THREADS) {
      uint32_t c = 0;
#pragma unroll
      for (int r = 0; r < SEL_CLUSTER; ++r) c += *cluster.map_shared_rank(&hist[i], r);
      tot[i] = c;
    }
    __syncthreads();
    if (warp == 0) {
      // lane l owns bins 255-8l .. 248-8l (descending)
      uint32_t h[8], s = 0;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        h[j] = tot[255 - 8 * lane - j];
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
    cnt_eq = tot[bucket];
    cluster.sync();                    // every CTA has read the histograms: they may be reset
  }
  const uint32_t kstar = prefix;

  if (k == cnt_eq) {
    // every key equal to K* is taken: no ordering needed
    for (int t = lo + tid; t < hi; t += SEL_THREADS) mk[t] = key_at(t) >= kstar ? 1 : 0;
    return;
  }
  // ---- ties at K*: the k lowest token indices among keys == K*.  This CTA's
  // ties come after those of the CTAs before it in the cluster.
  {
    int eq = 0;
    for (int t = lo + tid; t < hi; t += SEL_THREADS) eq += key_at(t) == kstar;
#pragma unroll
    for (int o = 16; o; o >>= 1) eq += __shfl_xor_sync(0xffffffffu, eq, o);
    if (tid == 0) sh_eq = 0;
    __syncthreads();
    if (lane == 0) atomicAdd(&sh_eq, (uint32_t)eq);
  }
  cluster.sync();                      // every CTA's tie count is published
  uint32_t carry = 0;
  for (int r = 0; r < rank; ++r) carry += *cluster.map_shared_rank(&sh_eq, r);
  for (int base = lo; base < hi; base += 4 * SEL_THREADS) {
    const int t0 = base + 4 * tid;
    uint32_t kk[4];
    int eq = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      kk[i] = (t0 + i < hi) ? key_at(t0 + i) : 0u;
      eq += (t0 + i < hi) && kk[i] == kstar;
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
      int tt = lane < SEL_THREADS / 32 ? sh_scan[lane] : 0;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        int y = __shfl_up_sync(0xffffffffu, tt, o);
        if (lane >= o) tt += y;
      }
      if (lane < SEL_THREADS / 32) sh_scan[lane] = tt;
      if (lane == 31) sh_scan[32] = tt;
    }
    __syncthreads();
    uint32_t rk = carry + (uint32_t)(x - eq + (warp ? sh_scan[warp - 1] : 0));
    const uint32_t total = (uint32_t)sh_scan[32];
    __syncthreads();
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int t = t0 + i;
      if (t < hi) {
        uint8_t v = kk[i] > kstar ? 1 : 0;
        if (kk[i] == kstar) {
          v = rk < k ? 1 : 0;
          ++rk;
        }
        mk[t] = v;
      }
    }
    carry += total;
  }
  cluster.sync();                      // no CTA leaves while another may read its tie count
}

cudaError_t launch_select(const float *score, int64_t score_bstride, const int32_t *seq_len,
                          int len_const, int B, int T_max, int r_ppm, uint8_t *mask,
                          int64_t mask_bstride, uint32_t *status, cudaStream_t st) {
  const int seg_max = (T_max + SEL_CLUSTER - 1) / SEL_CLUSTER;
  const int cache = seg_max <= SEL_SEG_KEYS ? 1 : 0;
  const size_t smem = cache ? (size_t)seg_max * 4 : 0;
  cudaError_t e = prepare_kernel(reinterpret_cast<const void *>(select_kernel), SEL_SEG_KEYS * 4);   // once per device
  if (e != cudaSuccess) return e;
  if (B > 0)
    select_kernel<<<dim3(SEL_CLUSTER, B), SEL_THREADS, smem, st>>>(score, score_bstride, seq_len, len_const, T_max,
                                                                   r_ppm, mask, mask_bstride, status, cache);
  return cudaGetLastError();
}

}  // namespace semkv
