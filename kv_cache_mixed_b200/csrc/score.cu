// score.cu -- per-token importance scores of one scoring layer (SemKV, Fig. 2).
//
// key_l2: the "key-norm" indicator (SemKV, Table 3): L2 norm of the token's key
//   over every KV head of the scoring layer, in one fixed fp32 order (lane
//   partials over dims 4l..4l+3, xor butterfly 16..1, heads in order, IEEE
//   sqrt), so the GPU result is one definite IEEE value.
//
// attn_mass: the attention indicator (SemKV, Table 1 "Attn.", Fig. 10: its
//   recomputation grows with T): s_j = sum over query heads and the last w
//   window rows of softmax_j(q . k_j / sqrt(D)), causal.  Two passes over K on
//   tensor cores (mma.sync m16n8k16, fp16 in, fp32 accumulate): pass 1 finds
//   every row's max and sum of exponentials (online, split over T chunks,
//   merged by a small kernel), pass 2 recomputes the logits and sums the
//   normalised probabilities down each key column.  Column sums are reduced in
//   a fixed order (warp shuffles, then warps, then KV heads), so the score is
//   deterministic.
#include "common.cuh"
#include "internal.h"

namespace semkv {

// ============================================================ key L2
constexpr int KL2_WARPS = 8;

__global__ void __launch_bounds__(KL2_WARPS * 32)
key_l2_kernel(const uint16_t *__restrict__ k, int64_t kbs, const int32_t *__restrict__ seq_len,
              int B, int T_max, int H, FastDiv divT, float *__restrict__ score, uint32_t *status) {
  const int lane = threadIdx.x & 31;
  const uint32_t ntok = (uint32_t)B * (uint32_t)T_max;
  const uint32_t w0 = blockIdx.x * KL2_WARPS + (threadIdx.x >> 5);
  const uint32_t nw = gridDim.x * KL2_WARPS;
  for (uint32_t tok = w0; tok < ntok; tok += nw) {
    const uint32_t b = divT.div(tok);
    const int t = (int)(tok - b * (uint32_t)T_max);
    const int len = seq_len[b];
    if (len < 0 || len > T_max) {
      if (lane == 0) {
        score[tok] = 0.0f;
        if (t == 0) set_flag(status, SEMKV_FLAG_SEQLEN);
      }
      continue;
    }
    if (t >= len) {
      if (lane == 0) score[tok] = 0.0f;
      continue;
    }
    const uint16_t *base = k + (int64_t)b * kbs + (int64_t)t * kD + 4 * lane;
    float acc = 0.0f;
    for (int g0 = 0; g0 < H; g0 += 8) {
      uint2 v[8];
#pragma unroll
      for (int j = 0; j < 8; ++j)
        if (g0 + j < H) v[j] = __ldg(reinterpret_cast<const uint2 *>(base + (int64_t)(g0 + j) * T_max * kD));
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        if (g0 + j >= H) break;
        const float2 a = __half22float2(*reinterpret_cast<const __half2 *>(&v[j].x));
        const float2 c = __half22float2(*reinterpret_cast<const __half2 *>(&v[j].y));
        float p = __fadd_rn(__fadd_rn(__fmul_rn(a.x, a.x), __fmul_rn(a.y, a.y)),
                            __fadd_rn(__fmul_rn(c.x, c.x), __fmul_rn(c.y, c.y)));
#pragma unroll
        for (int s = 16; s >= 1; s >>= 1) p = __fadd_rn(p, __shfl_xor_sync(0xffffffffu, p, s));
        acc = __fadd_rn(acc, p);
      }
    }
    if (lane == 0) {
      const float r = __fsqrt_rn(acc);
      if (!isfinite(r)) set_flag(status, SEMKV_FLAG_NONFINITE);
      score[tok] = r;
    }
  }
}

cudaError_t launch_score_key_l2(const uint16_t *k, int64_t k_bstride, const int32_t *seq_len,
                                int B, int T_max, int H, float *score, uint32_t *status,
                                cudaStream_t st) {
  int dev = 0, sms = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t ntok = (int64_t)B * T_max;
  int64_t want = (ntok + KL2_WARPS - 1) / KL2_WARPS;
  int64_t cap = (int64_t)sms * 8;
  int grid = (int)(want < cap ? want : cap);
  if (grid < 1) grid = 1;
  key_l2_kernel<<<grid, KL2_WARPS * 32, 0, st>>>(k, k_bstride, seq_len, B, T_max, H,
                                                  FastDiv((uint32_t)T_max), score, status);
  return cudaGetLastError();
}

// ============================================================ attention mass
constexpr int AM_WARPS = 8;
constexpr int AM_ROWS = AM_WARPS * 32;         // window rows per CTA row block (2 M-tiles per warp)
constexpr int AM_TILE = 64;                    // keys per smem tile
constexpr float kLog2e = 1.4426950408889634f;

struct AttnParams {
  const uint16_t *k;
  int64_t kbs;
  const uint16_t *q;        // [B][H_q][w][D]
  const int32_t *seq_len;
  int B, T_max, H, H_q, G, w;
  int Rg;                   // rows per KV head = G*w
  int nrb;                  // row blocks per KV head
  int nchunk;               // pass-1 T chunks
  float c1;                 // log2(e)/sqrt(D)
  float2 *part;             // [B][H_q*w][nchunk] (m, l) pass-1 partials
  float2 *stats;            // [B][H_q*w] (M, 1/Z)
  float *score;
  uint32_t *status;
};

// Load one 64-key tile of head g (tokens t0..t0+63, zero beyond T_max) into
// smem with a 16-byte-chunk xor swizzle (chunk' = chunk ^ (row & 7)).
__device__ __forceinline__ void am_load_tile(uint4 *sm, const uint16_t *kg, int t0, int T_max) {
  for (int i = threadIdx.x; i < AM_TILE * 16; i += AM_WARPS * 32) {
    const int r = i >> 4, c = i & 15;
    uint4 *dst = sm + r * 16 + (c ^ (r & 7));
    const int t = t0 + r;
    if (t < T_max) cp_async16(dst, kg + (int64_t)t * kD + c * 8);
    else *dst = make_uint4(0, 0, 0, 0);
  }
}

// A fragments (window rows of this warp) for one KV head: 2 M-tiles x 8 k-steps x 4 regs.
__device__ __forceinline__ void am_load_q(uint32_t (&qa)[2][8][4], const AttnParams &p, int b,
                                          int g, int rb, int warp, int lane) {
  const int r = lane >> 2, c = lane & 3;
#pragma unroll
  for (int mt = 0; mt < 2; ++mt) {
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
      const int rr = rb * AM_ROWS + warp * 32 + mt * 16 + r + 8 * hh;   // row within the head group
      const bool ok = rr < p.Rg;
      const int h = g * p.G + (ok ? rr / p.w : 0), i = ok ? rr % p.w : 0;
      const uint32_t *qrow = reinterpret_cast<const uint32_t *>(
          p.q + (((int64_t)b * p.H_q + h) * p.w + i) * kD);
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) {
        qa[mt][ks][hh] = ok ? __ldg(qrow + ks * 8 + c) : 0u;          // dims 16ks+2c, +1
        qa[mt][ks][2 + hh] = ok ? __ldg(qrow + ks * 8 + 4 + c) : 0u;  // dims 16ks+8+2c, +1
      }
    }
  }
}

// S = Q K^T for this warp's 32 rows and 32 keys (sub-tile st of the 64-key tile)
__device__ __forceinline__ void am_logits(float (&acc)[2][4][4], const uint32_t (&qa)[2][8][4],
                                          const uint4 *sm, int st, int lane) {
#pragma unroll
  for (int mt = 0; mt < 2; ++mt)
#pragma unroll
    for (int nt = 0; nt < 4; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[mt][nt][e] = 0.0f;
#pragma unroll
  for (int ks = 0; ks < 8; ++ks) {
#pragma unroll
    for (int np = 0; np < 2; ++np) {
      // matrices: (keys n0..+7, dims lo), (n0.., dims hi), (n0+8.., lo), (n0+8.., hi)
      const int mi = lane >> 3, ri = lane & 7;
      const int row = st * 32 + np * 16 + (mi >> 1) * 8 + ri;
      const int chunk = ks * 2 + (mi & 1);
      uint32_t bf[4];
      ldmatrix_x4(bf, sm + row * 16 + (chunk ^ (row & 7)));
#pragma unroll
      for (int mt = 0; mt < 2; ++mt) {
        mma_16816(acc[mt][np * 2], qa[mt][ks][0], qa[mt][ks][1], qa[mt][ks][2], qa[mt][ks][3],
                  bf[0], bf[1]);
        mma_16816(acc[mt][np * 2 + 1], qa[mt][ks][0], qa[mt][ks][1], qa[mt][ks][2],
                  qa[mt][ks][3], bf[2], bf[3]);
      }
    }
  }
}

// pass 1: grid (nchunk, H*nrb, B)
__global__ void __launch_bounds__(AM_WARPS * 32, 1) attn_rowstats_kernel(const AttnParams p) {
  __shared__ __align__(16) uint4 sm[2][AM_TILE * 16];
  const int chunk = blockIdx.x, g = blockIdx.y / p.nrb, rb = blockIdx.y % p.nrb, b = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, r = lane >> 2, c = lane & 3;
  const int len = p.seq_len[b];
  if (len < 0 || len > p.T_max) return;   // flagged by pass 2
  const int ntile = (len + AM_TILE - 1) / AM_TILE;
  const int tb = (int)((int64_t)ntile * chunk / p.nchunk), te = (int)((int64_t)ntile * (chunk + 1) / p.nchunk);
  const uint16_t *kg = p.k + (int64_t)b * p.kbs + (int64_t)g * p.T_max * kD;

  uint32_t qa[2][8][4];
  am_load_q(qa, p, b, g, rb, warp, lane);
  // row positions: rows r, r+8 of each M-tile
  int pos[2][2];
#pragma unroll
  for (int mt = 0; mt < 2; ++mt)
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
      const int rr = rb * AM_ROWS + warp * 32 + mt * 16 + r + 8 * hh;
      pos[mt][hh] = rr < p.Rg ? len - p.w + rr % p.w : -1;   // -1: dead row
    }
  float m[2][2], l[2][2];
#pragma unroll
  for (int mt = 0; mt < 2; ++mt)
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
      m[mt][hh] = -INFINITY;
      l[mt][hh] = 0.0f;
    }

  if (tb < te) {
    am_load_tile(sm[0], kg, tb * AM_TILE, p.T_max);
    cp_async_commit();
  }
  for (int ti = tb; ti < te; ++ti) {
    const int buf = (ti - tb) & 1;
    if (ti + 1 < te) am_load_tile(sm[buf ^ 1], kg, (ti + 1) * AM_TILE, p.T_max);
    cp_async_commit();
    cp_async_wait<1>();
    __syncthreads();
#pragma unroll 1
    for (int st = 0; st < 2; ++st) {
      float acc[2][4][4];
      am_logits(acc, qa, sm[buf], st, lane);
      const int j0 = ti * AM_TILE + st * 32;
#pragma unroll
      for (int mt = 0; mt < 2; ++mt)
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          float v[8];
          float mx = -INFINITY;
#pragma unroll
          for (int nt = 0; nt < 4; ++nt)
#pragma unroll
            for (int e = 0; e < 2; ++e) {
              const int j = j0 + nt * 8 + 2 * c + e;
              const float s = acc[mt][nt][hh * 2 + e] * p.c1;
              v[nt * 2 + e] = j <= pos[mt][hh] ? s : -INFINITY;
              mx = fmaxf(mx, v[nt * 2 + e]);
            }
          mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
          mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
          const float mn = fmaxf(m[mt][hh], mx);
          if (mn == -INFINITY) continue;
          float sum = 0.0f;
#pragma unroll
          for (int e = 0; e < 8; ++e) sum += ex2_approx(v[e] - mn);
          l[mt][hh] = l[mt][hh] * ex2_approx(m[mt][hh] - mn) + sum;
          m[mt][hh] = mn;
        }
    }
    __syncthreads();
  }
  // reduce l over the quad and write partials
#pragma unroll
  for (int mt = 0; mt < 2; ++mt)
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
      float lv = l[mt][hh];
      lv += __shfl_xor_sync(0xffffffffu, lv, 1);
      lv += __shfl_xor_sync(0xffffffffu, lv, 2);
      const int rr = rb * AM_ROWS + warp * 32 + mt * 16 + r + 8 * hh;
      if (c == 0 && rr < p.Rg) {
        const int row = (g * p.G + rr / p.w) * p.w + rr % p.w;      // h*w + i
        p.part[((int64_t)b * p.H_q * p.w + row) * p.nchunk + chunk] = make_float2(m[mt][hh], lv);
      }
    }
}

// merge pass-1 partials: one thread per window row
__global__ void attn_merge_kernel(const AttnParams p) {
  const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const int64_t nrows = (int64_t)p.B * p.H_q * p.w;
  if (idx >= nrows) return;
  const float2 *pp = p.part + idx * p.nchunk;
  float M = -INFINITY;
  for (int c = 0; c < p.nchunk; ++c) M = fmaxf(M, pp[c].x);
  float Z = 0.0f;
  if (M != -INFINITY)
    for (int c = 0; c < p.nchunk; ++c)
      if (pp[c].x != -INFINITY) Z += pp[c].y * ex2_approx(pp[c].x - M);
  p.stats[idx] = make_float2(M, Z > 0.0f ? 1.0f / Z : 0.0f);
}

// pass 2: grid (ceil(T_max/64), B); each CTA sums 64 key columns over every
// window row of every query head, KV heads in order.
__global__ void __launch_bounds__(AM_WARPS * 32, 1) attn_colsum_kernel(const AttnParams p) {
  __shared__ __align__(16) uint4 sm[AM_TILE * 16];
  __shared__ float colpart[AM_WARPS][AM_TILE];
  const int tile = blockIdx.x, b = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, r = lane >> 2, c = lane & 3;
  const int len = p.seq_len[b];
  const int t0 = tile * AM_TILE;
  float *out = p.score + (int64_t)b * p.T_max;
  if (len < 0 || len > p.T_max) {
    if (threadIdx.x < AM_TILE && t0 + (int)threadIdx.x < p.T_max) out[t0 + threadIdx.x] = 0.0f;
    if (threadIdx.x == 0 && tile == 0) set_flag(p.status, SEMKV_FLAG_SEQLEN);
    return;
  }
  if (t0 >= len) {
    if (threadIdx.x < AM_TILE && t0 + (int)threadIdx.x < p.T_max) out[t0 + threadIdx.x] = 0.0f;
    return;
  }
  float total = 0.0f;   // thread j < 64 accumulates column j
  for (int g = 0; g < p.H; ++g) {
    const uint16_t *kg = p.k + (int64_t)b * p.kbs + (int64_t)g * p.T_max * kD;
    __syncthreads();
    am_load_tile(sm, kg, t0, p.T_max);
    cp_async_commit();
    for (int rb = 0; rb < p.nrb; ++rb) {
      uint32_t qa[2][8][4];
      am_load_q(qa, p, b, g, rb, warp, lane);
      float M[2][2], iZ[2][2];
      int pos[2][2];
#pragma unroll
      for (int mt = 0; mt < 2; ++mt)
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          const int rr = rb * AM_ROWS + warp * 32 + mt * 16 + r + 8 * hh;
          if (rr < p.Rg) {
            const int row = (g * p.G + rr / p.w) * p.w + rr % p.w;
            const float2 s = p.stats[(int64_t)b * p.H_q * p.w + row];
            M[mt][hh] = s.x;
            iZ[mt][hh] = s.y;
            pos[mt][hh] = len - p.w + rr % p.w;
          } else {
            M[mt][hh] = 0.0f;
            iZ[mt][hh] = 0.0f;
            pos[mt][hh] = -1;
          }
        }
      cp_async_wait<0>();
      __syncthreads();
#pragma unroll 1
      for (int st = 0; st < 2; ++st) {
        float acc[2][4][4];
        am_logits(acc, qa, sm, st, lane);
        float col[4][2];
#pragma unroll
        for (int nt = 0; nt < 4; ++nt) col[nt][0] = col[nt][1] = 0.0f;
#pragma unroll
        for (int mt = 0; mt < 2; ++mt)
#pragma unroll
          for (int hh = 0; hh < 2; ++hh)
#pragma unroll
            for (int nt = 0; nt < 4; ++nt)
#pragma unroll
              for (int e = 0; e < 2; ++e) {
                const int j = t0 + st * 32 + nt * 8 + 2 * c + e;
                const float s = acc[mt][nt][hh * 2 + e] * p.c1;
                const float pr = (j <= pos[mt][hh] && iZ[mt][hh] > 0.0f)
                                     ? ex2_approx(s - M[mt][hh]) * iZ[mt][hh] : 0.0f;
                col[nt][e] += pr;
              }
        // reduce over the 8 row groups (lanes with the same c)
#pragma unroll
        for (int nt = 0; nt < 4; ++nt)
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            float v = col[nt][e];
            v += __shfl_xor_sync(0xffffffffu, v, 4);
            v += __shfl_xor_sync(0xffffffffu, v, 8);
            v += __shfl_xor_sync(0xffffffffu, v, 16);
            if (r == 0) colpart[warp][st * 32 + nt * 8 + 2 * c + e] = v;
          }
      }
      __syncthreads();
      if (threadIdx.x < AM_TILE) {
        float s = 0.0f;
#pragma unroll
        for (int wi = 0; wi < AM_WARPS; ++wi) s += colpart[wi][threadIdx.x];
        total += s;
      }
      __syncthreads();
    }
  }
  if (threadIdx.x < AM_TILE) {
    const int j = t0 + threadIdx.x;
    if (j < p.T_max) out[j] = j < len ? total : 0.0f;
  }
}

size_t attn_mass_ws_bytes(int B, int T_max, int H, int H_q, int w) {
  (void)H;
  const int64_t rows = (int64_t)B * H_q * w;
  const int ntile = (T_max + AM_TILE - 1) / AM_TILE;
  const int nchunk = ntile < 64 ? ntile : 64;
  return (size_t)(rows * nchunk * sizeof(float2) + rows * sizeof(float2) + 256);
}

cudaError_t launch_score_attn_mass(const uint16_t *k, int64_t k_bstride, const uint16_t *q_win,
                                   const int32_t *seq_len, int B, int T_max, int H, int H_q,
                                   int w, float *score, void *ws, uint32_t *status,
                                   cudaStream_t st) {
  AttnParams p;
  p.k = k;
  p.kbs = k_bstride;
  p.q = q_win;
  p.seq_len = seq_len;
  p.B = B;
  p.T_max = T_max;
  p.H = H;
  p.H_q = H_q;
  p.G = H_q / H;
  p.w = w;
  p.Rg = p.G * w;
  p.nrb = (p.Rg + AM_ROWS - 1) / AM_ROWS;
  const int ntile = (T_max + AM_TILE - 1) / AM_TILE;
  int dev = 0, sms = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  int want = (2 * sms + H * p.nrb * B - 1) / (H * p.nrb * B);
  p.nchunk = want < 1 ? 1 : (want > ntile ? ntile : (want > 64 ? 64 : want));
  p.c1 = kLog2e / sqrtf((float)kD);
  const int64_t rows = (int64_t)B * H_q * w;
  const int nchunk_ws = ntile < 64 ? ntile : 64;
  p.part = reinterpret_cast<float2 *>(ws);
  p.stats = reinterpret_cast<float2 *>(reinterpret_cast<char *>(ws) + rows * nchunk_ws * sizeof(float2));
  p.score = score;
  p.status = status;
  attn_rowstats_kernel<<<dim3(p.nchunk, H * p.nrb, B), AM_WARPS * 32, 0, st>>>(p);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  attn_merge_kernel<<<(unsigned)((rows + 255) / 256), 256, 0, st>>>(p);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  attn_colsum_kernel<<<dim3(ntile, B), AM_WARPS * 32, 0, st>>>(p);
  return cudaGetLastError();
}

}  // namespace semkv
