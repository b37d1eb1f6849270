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
//   tensor cores (fp16 in, fp32 accumulate): pass 1 finds every row's max and
//   sum of exponentials (online, split over T chunks, merged by a small
//   kernel), pass 2 recomputes the logits and sums the normalised
//   probabilities down each key column.  Window groups of up to 256 rows per
//   KV head run on tcgen05 with TMEM accumulators (attn_umma_kernel); wider
//   groups on mma.sync m16n8k16.  Column sums are reduced in a fixed order, so
//   the score is deterministic.
#include "common.cuh"
#include "internal.h"
#include "umma.cuh"

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
  const int sms = device_sm_count();
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

// merge pass-1 partials: one warp per window row, lanes over the T chunks
// (nchunk <= 64), reduced by a fixed shuffle tree
__global__ void __launch_bounds__(256) attn_merge_kernel(const AttnParams p) {
  const int64_t row = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  const int64_t nrows = (int64_t)p.B * p.H_q * p.w;
  if (row >= nrows) return;
  const float2 *pp = p.part + row * p.nchunk;
  const float2 a = lane < p.nchunk ? pp[lane] : make_float2(-INFINITY, 0.0f);
  const float2 c = lane + 32 < p.nchunk ? pp[lane + 32] : make_float2(-INFINITY, 0.0f);
  float M = fmaxf(a.x, c.x);
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
  float Z = 0.0f;
  if (M != -INFINITY) {
    if (a.x != -INFINITY) Z += a.y * ex2_approx(a.x - M);
    if (c.x != -INFINITY) Z += c.y * ex2_approx(c.x - M);
  }
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) Z += __shfl_xor_sync(0xffffffffu, Z, o);
  if (lane == 0) p.stats[row] = make_float2(M, Z > 0.0f ? 1.0f / Z : 0.0f);
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

// ---- both passes on the 5th-generation tensor cores (tcgen05, TMEM accumulators)
// CTA = (key chunk, KV head g, sequence b): 16 epilogue warps and one producer
// warp.  The Np <= 256 window rows of g's query heads stay in shared memory.
// The producer's lane 0 loads the 128-key tiles as two 128-byte-swizzled TMA
// tensor boxes (dims 0..63 and 64..127) into a 4-slot ring and issues each
// tile's MMAs into one of two TMEM accumulators (tile i into accumulator i%2,
// once the epilogue warps have released it).  Each epilogue warp waits for the
// tile's accumulator, reads its TMEM lanes (quadrant warp % 4) and releases the
// accumulator with one arrival: no CTA-wide barrier per tile, so a warp runs on
// to the next tile as soon as its MMAs are done, and the warps' exp2 bursts
// spread out instead of meeting.
//   pass 1: D[rows][keys] = Q_g[rows] . K^T  (two M=128 halves of rows, N=128):
//           each thread owns one row and one 64-key half of every tile, keeps an
//           online (max, sum of exp2) over its chunk, and writes one partial per
//           (row, chunk, key half);
//   pass 2: D[keys][rows] = K . Q_g^T  (M=128 keys, N=Np): each thread owns one
//           key and one quarter of the rows (warps w, w+4, w+8, w+12) and sums
//           exp2(s*c1 - M'_r), M'_r = M_r + log2(Z_r); one partial per (head,
//           row quarter, key), summed in order by attn_headsum_kernel.
constexpr int UA_EPI_WARPS = 16;
constexpr int UA_THREADS = (UA_EPI_WARPS + 1) * 32;   // + the producer warp
constexpr int UA_RQ = 4;                          // pass-2 row quarters (head partials per key)
constexpr int UA_KEYS = 128;
constexpr int UA_MAXN = 256;
constexpr int UA_NST = 4;                         // key tiles in the ring
constexpr int UA_QBYTES = UA_MAXN * 256;
constexpr int UA_KBYTES = UA_KEYS * 256;
constexpr int UA_OFF_Q = 0;
constexpr int UA_OFF_K = UA_QBYTES;
constexpr int UA_OFF_M = UA_OFF_K + UA_NST * UA_KBYTES;          // float [256] M'_r (pass 2)
// mbarriers: [2] accumulator full (MMA commit), [2] accumulator free (16 warp
// arrivals), [UA_NST] key tile landed (TMA)
constexpr int UA_OFF_BAR = UA_OFF_M + UA_MAXN * 4;
constexpr int UA_OFF_SLOT = UA_OFF_BAR + (4 + UA_NST) * 8;
constexpr int UA_SMEM = UA_OFF_SLOT + 16 + 1024;
constexpr int kUmmaWait = 1 << 22;
static_assert(UA_OFF_K % 1024 == 0 && UA_KBYTES % 1024 == 0, "operand blocks must be 1024-byte aligned");

__device__ __forceinline__ void mbar_arrive_one(uint64_t *bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];\n" ::"r"(smem_u32(bar)) : "memory");
}

template <int PASS>
__global__ void __launch_bounds__(UA_THREADS, 1) attn_umma_kernel(const AttnParams p, int Np, int nchunk,
                                                                   float *head_part,
                                                                   const __grid_constant__ CUtensorMap kmap) {
  extern __shared__ uint8_t smem_raw[];
  // 1024-byte alignment by an offset from the shared base, so that the compiler
  // still sees shared-memory pointers (plain shared loads, not generic ones)
  uint8_t *smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const int chunk = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const bool producer = warp == UA_EPI_WARPS;
  const int quarter = warp & 3;                    // TMEM lane quadrant of this warp
  const int half = (warp >> 2) & 1, kh = warp >> 3; // pass 1: row half, key half of the tile
  const int rq = warp >> 2;                        // pass 2: row quarter
  const int len = p.seq_len[b];
  if (len < 0 || len > p.T_max) return;            // flagged by the head-sum / merge kernels
  const int ntile = (len + UA_KEYS - 1) / UA_KEYS;
  const int tb = (int)((int64_t)ntile * chunk / nchunk), te = (int)((int64_t)ntile * (chunk + 1) / nchunk);
  const int n = te - tb;                           // this CTA's tiles; local tile i = tb + i

  float *Ms = reinterpret_cast<float *>(smem + UA_OFF_M);
  uint64_t *full = reinterpret_cast<uint64_t *>(smem + UA_OFF_BAR);    // [2]
  uint64_t *freeb = full + 2;                                           // [2]
  uint64_t *tbars = full + 4;                                           // [UA_NST]
  uint32_t *slot = reinterpret_cast<uint32_t *>(smem + UA_OFF_SLOT);
  const uint32_t sbase = smem_u32(smem);
  if (warp == 0) tmem_alloc(slot, 512);
  if (tid == 0) {
    mbar_init(&full[0], 1);
    mbar_init(&full[1], 1);
    mbar_init(&freeb[0], UA_EPI_WARPS);
    mbar_init(&freeb[1], UA_EPI_WARPS);
#pragma unroll
    for (int s = 0; s < UA_NST; ++s) mbar_init(&tbars[s], 1);
    fence_mbar_init();
  }
  // resident window rows of head g (zero past Rg), and pass 2's row constants
  {
    const uint16_t *qg = p.q + ((int64_t)b * p.H_q + g * p.G) * p.w * kD;
    for (int i = tid; i < Np * 16; i += UA_THREADS) {
      const int r = i >> 4, c = i & 15;
      const bool ok = r < p.Rg;
      cp_async16_zfill(smem + UA_OFF_Q + sw128_offset(r, c, Np), qg + (ok ? (int64_t)r * kD + c * 8 : 0), ok);
    }
    if (PASS == 2) {
      for (int r = tid; r < Np; r += UA_THREADS) {
        float m = INFINITY;                          // rows that contribute nothing
        if (r < p.Rg) {
          const float2 st = p.stats[(int64_t)b * p.H_q * p.w + g * p.Rg + r];
          if (st.y > 0.0f) m = st.x - __log2f(st.y);     // st.y = 1/Z
        }
        Ms[r] = m;
      }
    }
    cp_async_commit();
    cp_async_wait<0>();
    fence_proxy_async_smem();                      // the window rows feed the tensor cores
  }
  __syncthreads();
  const uint32_t tmem = *slot;
  tc_fence_after();
  const uint32_t qa = sbase + UA_OFF_Q;
  bool lost = false;

  if (producer) {
    if (lane == 0) {
      uint32_t tpend = 0;                          // slots with a load in flight
      int tstaged[UA_NST];                         // the local tile last loaded into each slot
      auto stage = [&](int i) {                    // local tile i into slot i % UA_NST
        if (i < n) {
          const int sl = i % UA_NST;
          uint8_t *kd = smem + UA_OFF_K + sl * UA_KBYTES;
          const int t0 = (tb + i) * UA_KEYS;
          mbar_expect_tx(&tbars[sl], UA_KBYTES);
          tma_load_4d(kd, &kmap, 0, t0, g, b, &tbars[sl]);
          tma_load_4d(kd + UA_KEYS * 128, &kmap, 64, t0, g, b, &tbars[sl]);
          tpend |= 1u << sl;
          tstaged[sl] = i;
        }
      };
      for (int i = 0; i < UA_NST; ++i) stage(i);
      int issued = 0;                              // MMAs issued (local tiles 0 .. issued-1)
      for (int i = 0; i < n; ++i) {
        const int sl = i % UA_NST, ab = i & 1;
        // the tile's keys have landed, and the accumulator's last tile (i-2)
        // has been read by all 16 epilogue warps
        if (!mbar_wait(&tbars[sl], (i / UA_NST) & 1, kUmmaWait)) { lost = true; break; }
        tpend &= ~(1u << sl);
        if (i >= 2 && !mbar_wait(&freeb[ab], ((i - 2) >> 1) & 1, kUmmaWait)) { lost = true; break; }
        tc_fence_after();
        const uint32_t ka = sbase + UA_OFF_K + sl * UA_KBYTES;
        const uint32_t acc = tmem + ab * 256;
        if (PASS == 1) {
          const uint32_t idesc = umma_idesc_f16(128, UA_KEYS);
          for (int hf = 0; hf * 128 < Np; ++hf) {
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) {
              const uint32_t off = (ks & 3) * 32;
              const uint64_t adesc = umma_desc_sw128(qa + (ks >> 2) * (Np * 128) + hf * 128 * 128 + off);
              const uint64_t bdesc = umma_desc_sw128(ka + (ks >> 2) * (UA_KEYS * 128) + off);
              umma_f16(acc + hf * 128, adesc, bdesc, idesc, ks > 0 ? 1u : 0u);
            }
          }
        } else {
          const uint32_t idesc = umma_idesc_f16(UA_KEYS, Np);
#pragma unroll
          for (int ks = 0; ks < 8; ++ks) {
            const uint32_t off = (ks & 3) * 32;
            const uint64_t adesc = umma_desc_sw128(ka + (ks >> 2) * (UA_KEYS * 128) + off);
            const uint64_t bdesc = umma_desc_sw128(qa + (ks >> 2) * (Np * 128) + off);
            umma_f16(acc, adesc, bdesc, idesc, ks > 0 ? 1u : 0u);
          }
        }
        umma_commit(&full[ab]);
        issued = i + 1;
        // the slot of tile i-1 is free once its MMAs are done: load tile i+3 there
        if (i >= 1) {
          if (!mbar_wait(&full[(i - 1) & 1], ((i - 1) >> 1) & 1, kUmmaWait)) { lost = true; break; }
          stage(i - 1 + UA_NST);
        }
      }
      if (lost) {
        // drain: wait, with the full bound, for the commits of the MMAs issued
        // (the last two) and for every key tile load still in flight, before
        // TMEM and shared memory are freed
        set_flag(p.status, SEMKV_FLAG_TIMEOUT);
        for (int i = issued - 2 < 0 ? 0 : issued - 2; i < issued; ++i)
          mbar_wait(&full[i & 1], (i >> 1) & 1, kUmmaWait);
        for (int sl = 0; sl < UA_NST; ++sl)
          if ((tpend >> sl) & 1u) mbar_wait(&tbars[sl], (tstaged[sl] / UA_NST) & 1, kUmmaWait);
      }
    }
  } else {
    // epilogue warps
    const int row = half * 128 + quarter * 32 + lane;
    const int pos = (PASS == 1 && row < p.Rg) ? len - p.w + row % p.w : -1;
    float m_run = -INFINITY, l_run = 0.0f;
    const int ncol_q = Np / UA_RQ;                 // pass 2: rows per row quarter (a multiple of 16)
    for (int i = 0; i < n; ++i) {
      const int ab = i & 1;
      if (!mbar_wait(&full[ab], (i >> 1) & 1, kUmmaWait)) {
        lost = true;
        break;
      }
      tc_fence_after();
      const int t0 = (tb + i) * UA_KEYS;
      const bool edge = t0 + UA_KEYS - 1 > len - p.w;
      if (PASS == 1) {
        if (half * 128 < Np) {
          const uint32_t la = tmem + ab * 256 + half * 128 + kh * 64 + ((uint32_t)(quarter * 32) << 16);
          // raw logits of this row for its 64 keys (c1 > 0: the max commutes with the scaling)
          float v[64];
#pragma unroll
          for (int cb = 0; cb < 2; ++cb) tmem_ld32(la + cb * 32, *reinterpret_cast<uint32_t(*)[32]>(&v[cb * 32]));
          tmem_ld_wait();
          if (edge) {
            const int lim = pos - t0 - kh * 64;      // keys t0 + 64 kh + j with j > lim are masked
#pragma unroll
            for (int j = 0; j < 64; ++j) v[j] = j <= lim ? v[j] : -INFINITY;
          }
          // two 32-key halves, each an online update: the max of the second half
          // is independent of the first half's exp2, so the two interleave
#pragma unroll
          for (int hk = 0; hk < 2; ++hk) {
            const float *vh = v + 32 * hk;
            float mr = vh[0];
#pragma unroll
            for (int j = 1; j < 31; j += 2) mr = fmax3_nan(mr, vh[j], vh[j + 1]);
            const float mx = fmax_nan(m_run, fmax_nan(mr, vh[31]) * p.c1);
            if (mx != -INFINITY) {
              float sum[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
              for (int j = 0; j < 32; ++j) sum[j & 3] += ex2_approx(__fmaf_rn(vh[j], p.c1, -mx));
              l_run = l_run * ex2_approx(m_run - mx) + ((sum[0] + sum[1]) + (sum[2] + sum[3]));
              m_run = mx;
            }
          }
        }
      } else {
        const int key = t0 + quarter * 32 + lane;
        const int c0 = rq * ncol_q;
        const uint32_t la = tmem + ab * 256 + c0 + ((uint32_t)(quarter * 32) << 16);
        float acc4[4] = {0.0f, 0.0f, 0.0f, 0.0f};
        for (int cb = 0; cb < ncol_q; cb += 64) {
          // (a load past the quarter reads columns of the next one, still inside
          // the 256-column accumulator, and they are not used)
          uint32_t u[64];
          tmem_ld32(la + cb, *reinterpret_cast<uint32_t(*)[32]>(&u[0]));
          tmem_ld32(la + cb + 32, *reinterpret_cast<uint32_t(*)[32]>(&u[32]));
          tmem_ld_wait();
          const int nc = ncol_q - cb < 64 ? ncol_q - cb : 64;     // a multiple of 16
          if (!edge) {
            const float4 *M4 = reinterpret_cast<const float4 *>(Ms + c0 + cb);
            auto col4 = [&](int j4) {
              const float4 m4 = M4[j4];
              acc4[0] += ex2_approx(__fmaf_rn(__uint_as_float(u[4 * j4 + 0]), p.c1, -m4.x));
              acc4[1] += ex2_approx(__fmaf_rn(__uint_as_float(u[4 * j4 + 1]), p.c1, -m4.y));
              acc4[2] += ex2_approx(__fmaf_rn(__uint_as_float(u[4 * j4 + 2]), p.c1, -m4.z));
              acc4[3] += ex2_approx(__fmaf_rn(__uint_as_float(u[4 * j4 + 3]), p.c1, -m4.w));
            };
            if (nc == 64) {
#pragma unroll
              for (int j4 = 0; j4 < 16; ++j4) col4(j4);
            } else {
#pragma unroll
              for (int j4 = 0; j4 < 16; ++j4) {
                if (j4 * 4 >= nc) break;
                col4(j4);
              }
            }
          } else {
#pragma unroll
            for (int j = 0; j < 64; ++j) {
              if (j >= nc) break;
              const int r = c0 + cb + j;
              const bool vis = r < p.Rg && key <= len - p.w + r % p.w;
              acc4[j & 3] += vis ? ex2_approx(__fmaf_rn(__uint_as_float(u[j]), p.c1, -Ms[r])) : 0.0f;
            }
          }
        }
        const float acc = (acc4[0] + acc4[1]) + (acc4[2] + acc4[3]);
        // one partial per (KV head, row quarter, key): no exchange between the
        // four warps of a key, the head-sum kernel adds the quarters in order
        if (key < p.T_max)
          head_part[(((int64_t)b * p.H + g) * UA_RQ + rq) * p.T_max + key] = key < len ? acc : 0.0f;
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_one(&freeb[ab]);   // this warp is done with the accumulator
    }
    if (PASS == 1) {
      if (half * 128 < Np && row < p.Rg) {
        const int hrow = (g * p.G + row / p.w) * p.w + row % p.w;    // h*w + i
        p.part[((int64_t)b * p.H_q * p.w + hrow) * p.nchunk + 2 * chunk + kh] = make_float2(m_run, l_run);
      }
    }
    if (lost && lane == 0) set_flag(p.status, SEMKV_FLAG_TIMEOUT);
  }
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, 512);
}

// score[b][j] = sum over KV heads and row halves, in order, of the column partials
__global__ void attn_headsum_kernel(const AttnParams p, const float *__restrict__ head_part) {
  const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= (int64_t)p.B * p.T_max) return;
  const int b = (int)(idx / p.T_max), j = (int)(idx % p.T_max);
  const int len = p.seq_len[b];
  if (len < 0 || len > p.T_max) {
    p.score[idx] = 0.0f;
    if (j == 0) set_flag(p.status, SEMKV_FLAG_SEQLEN);
    return;
  }
  float s = 0.0f;
  if (j < len) {
    // the partials in order; eight loads in flight before they are added
    const int np = UA_RQ * p.H;
    const float *hp = head_part + (int64_t)b * np * p.T_max + j;
    for (int g0 = 0; g0 < np; g0 += 8) {
      float v[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) v[i] = g0 + i < np ? __ldg(hp + (int64_t)(g0 + i) * p.T_max) : 0.0f;
#pragma unroll
      for (int i = 0; i < 8; ++i)
        if (g0 + i < np) s += v[i];
    }
  }
  p.score[idx] = s;
}

size_t attn_mass_ws_bytes(int B, int T_max, int H, int H_q, int w) {
  const int64_t rows = (int64_t)B * H_q * w;
  const int ntile = (T_max + AM_TILE - 1) / AM_TILE;
  const int nchunk = ntile < 64 ? ntile : 64;
  const size_t parts = (size_t)(rows * nchunk * sizeof(float2) + rows * sizeof(float2) + 256);
  return (parts + 255) / 256 * 256 + (size_t)B * H * UA_RQ * T_max * sizeof(float) + 256;
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
  const int sms = device_sm_count();
  p.c1 = kLog2e / sqrtf((float)kD);
  const int64_t rows = (int64_t)B * H_q * w;
  const int nchunk_ws = ntile < 64 ? ntile : 64;
  p.part = reinterpret_cast<float2 *>(ws);
  p.stats = reinterpret_cast<float2 *>(reinterpret_cast<char *>(ws) + rows * nchunk_ws * sizeof(float2));
  const size_t parts = (size_t)(rows * nchunk_ws * sizeof(float2) + rows * sizeof(float2) + 256);
  float *head_part = reinterpret_cast<float *>(reinterpret_cast<char *>(ws) + (parts + 255) / 256 * 256);
  p.score = score;
  p.status = status;
  cudaError_t e;
  const int Np = (p.Rg + 63) / 64 * 64;       // two column halves of whole 32-column loads
  if (Np <= UA_MAXN) {
    // tcgen05 path: one CTA per SM (all of TMEM), about one wave of CTAs;
    // pass 1 writes two partials per (row, chunk), so at most 32 chunks
    const int utiles = (T_max + UA_KEYS - 1) / UA_KEYS;
    int nch = sms / (H * B);                  // whole waves only
    nch = nch < 1 ? 1 : (nch > utiles ? utiles : (nch > 32 ? 32 : nch));
    p.nchunk = 2 * nch;
    // keys [B][H][T_max][128] fp16 as a 4-D tensor map (dims fastest first),
    // boxes of 64 dims x 128 keys landing 128-byte swizzled; it needs 16-byte
    // aligned keys and a batch stride of whole 16-byte units (both checked by
    // semkv_score)
    CUtensorMap kmap;
    {
      const uint64_t dims[4] = {(uint64_t)kD, (uint64_t)T_max, (uint64_t)H, (uint64_t)B};
      const uint64_t strides[3] = {(uint64_t)kD * 2, (uint64_t)T_max * kD * 2, (uint64_t)k_bstride * 2};
      const uint32_t box[4] = {64, (uint32_t)UA_KEYS, 1, 1};
      e = encode_tensor_map_f16(&kmap, k, 4, dims, strides, box, true);
      if (e != cudaSuccess) return e;
    }
    auto k1 = attn_umma_kernel<1>;
    auto k2 = attn_umma_kernel<2>;
    e = prepare_kernel(reinterpret_cast<const void *>(k1), UA_SMEM);
    if (e != cudaSuccess) return e;
    e = prepare_kernel(reinterpret_cast<const void *>(k2), UA_SMEM);
    if (e != cudaSuccess) return e;
    k1<<<dim3(nch, H, B), UA_THREADS, UA_SMEM, st>>>(p, Np, nch, head_part, kmap);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    attn_merge_kernel<<<(unsigned)((rows + 7) / 8), 256, 0, st>>>(p);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    k2<<<dim3(nch, H, B), UA_THREADS, UA_SMEM, st>>>(p, Np, nch, head_part, kmap);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    attn_headsum_kernel<<<(unsigned)(((int64_t)B * T_max + 255) / 256), 256, 0, st>>>(p, head_part);
    return cudaGetLastError();
  }
  // mma.sync path for window groups wider than 256 rows
  int want = (2 * sms + H * p.nrb * B - 1) / (H * p.nrb * B);
  p.nchunk = want < 1 ? 1 : (want > ntile ? ntile : (want > 64 ? 64 : want));
  attn_rowstats_kernel<<<dim3(p.nchunk, H * p.nrb, B), AM_WARPS * 32, 0, st>>>(p);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  attn_merge_kernel<<<(unsigned)((rows + 7) / 8), 256, 0, st>>>(p);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  attn_colsum_kernel<<<dim3(ntile, B), AM_WARPS * 32, 0, st>>>(p);
  return cudaGetLastError();
}

}  // namespace semkv
