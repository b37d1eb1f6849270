// decode.cu -- GQA decode attention over the mixed-precision cache (SemKV,
// Fig. 5: "the mixed-precision quantized KV cache used for decoding"; Fig. 6:
// the most recent partial block stays FP16 during decoding).
//
// Attention works in the code domain, so no row is ever dequantized:
//   q . khat_j = scale_j * (q . c_j) + mn_j * sum(q)
//   sum_j p_j vhat_j = sum_j (p_j scale_j) c_j + (sum_j p_j mn_j) * 1
// Both dot products run on tensor cores (mma.sync m16n8k16, f16 x f16 -> f32).
// Codes enter the tensor cores as raw f16 subnormal bit patterns c * 2^-24
// (exact), so a digit costs no conversion: unpacking a 32-bit word gives the
// digit in the low bits of a register and two digits packed in one register
// are already an f16x2 operand.  The 2^24 factor is folded into the scales.
//
// Digit extraction (any L in [2,16]): a word is split by constant divisors into
// parts of k digits with L^k small enough that, with F = v * ceil(2^32/L^k),
// each step t = F * L yields the next digit (most significant first) in the
// high 32 bits and the next F in the low 32 bits.  The part sizes below were
// checked exhaustively against repeated division for every part value.  For
// L <= 6 one step by L^2 yields two digits, turned into the f16x2 operand by a
// small shared-memory table.
//
// Work split: one pool class per launch (template on its L, and on whether
// the rows are Hadamard-rotated); CTA = 4 warps on a contiguous range of
// 16-token tiles of one (sequence, layer, KV head); each warp streams its
// tiles through a ring of bulk asynchronous copies (cp.async.bulk completing
// on mbarriers, bounded waits); online softmax in the log2 domain; the 4
// warps merge in shared memory and the CTA writes one partial (m, l, o[128])
// per query head.  The FP16 block gets its own small kernel and a last kernel
// merges all partials of a (sequence, layer, KV head) into the output.
//
// MMA shapes per 16-token tile: the logits put the 16 tokens on the MMA rows
// and the query heads on the 8 columns (one m16n8k16 per 16 head-dim slots);
// the values put 16 head-dim slots on the rows and the query heads on the
// columns, with P' moved into that operand layout by movmatrix.  With at most
// 4 query heads per KV head, columns 4..7 of the value MMA carry the low f16
// part of P', so one MMA takes both parts.
#include "common.cuh"
#include "internal.h"

namespace semkv {

constexpr int DEC_WARPS = 4;
constexpr int DEC_NST = 4;                  // tiles in flight per warp
constexpr int DEC_GMAX = 8;                 // query heads per KV head handled (M rows used)
constexpr int PART_STRIDE = 132;            // floats per partial: m, l, pad, pad, o[128]
constexpr float kLog2eF = 1.4426950408889634f;

// ---- digit split table: part sizes in digits, least significant part first
__host__ __device__ constexpr int split_part(int L, int i) {
  // {part0, part1, part2} per L; a 0 marks an unused part
  return L == 2 ? (i < 2 ? 16 : 0) : L == 3 ? (i < 2 ? 10 : 0) : L == 4 ? (i < 2 ? 8 : 0)
       : L == 5 ? (i == 0 ? 6 : i == 1 ? 7 : 0) : L == 6 ? (i < 2 ? 6 : 0)
       : L == 7 ? (i == 0 ? 3 : 4) : L == 8 ? (i < 2 ? 5 : 0) : L == 9 ? (i < 2 ? 5 : 0)
       : L == 10 ? (i == 0 ? 4 : i == 1 ? 5 : 0) : L == 11 ? 3 : (i < 2 ? 4 : 0);
}
__host__ __device__ constexpr int split_parts(int L) { return (L == 7 || L == 11) ? 3 : 2; }

// Pair path (L <= 6): one wide multiply by L^2 yields two digits at once,
// hi = c_{j+1} * L + c_j, and a shared-memory table of L^2 entries turns hi
// into the f16x2 operand (c_j, c_{j+1}).  Every part of these levels starts on
// an even digit and only the top part can have odd length, so with the word
// stride in slots rounded up to even (L = 5: 13 digits in 14 slots) every pair
// stays inside one part; an odd top part leads with one single-digit step.
__host__ __device__ constexpr bool use_pairs(int L) { return L <= 6; }

template <int L>
struct Geo {
  static constexpr int N = digits_per_word(L);       // digits per word
  static constexpr int W = words_per_row(L);         // words per row
  static constexpr int S = use_pairs(L) ? N + (N & 1) : N;   // slots per word
  static constexpr int WPG = (W + 3) / 4;            // words per lane group (lane % 4)
  static constexpr int KB = (WPG * S + 3) / 4;       // 16-slot k-blocks
  static constexpr int TILE_BYTES = 16 * W * 4 * 2 + 16 * 8 * 2;
  static_assert(split_part(L, 0) + split_part(L, 1) + split_part(L, 2) == N, "split must cover the word");
  static_assert(!use_pairs(L) || (split_part(L, 0) % 2 == 0 && (split_parts(L) == 2 || split_part(L, 1) % 2 == 0)),
                "pair path needs even parts below the top part");
};

// digit j (0 = least significant) of word w into dig[j0 + j].  Lr holds L at
// run time so that every digit step stays one wide multiply.
template <int L, int NDIG>
__device__ __forceinline__ void extract_word(uint32_t w, uint32_t (&dig)[NDIG], int j0, uint32_t Lr) {
  constexpr int NP = split_parts(L);
  uint32_t rest = w;
  int jb = j0;
#pragma unroll
  for (int pi = 0; pi < NP; ++pi) {
    const int k = split_part(L, pi);
    uint32_t v;
    if (pi < NP - 1) {
      const uint32_t P = (uint32_t)ipow(L, k);
      const uint32_t qq = rest / P;
      v = rest - qq * P;
      rest = qq;
    } else {
      v = rest;
    }
    const uint32_t M = (uint32_t)(((1ull << 32) + ipow(L, k) - 1) / ipow(L, k));
    uint32_t F = v * M;
#pragma unroll
    for (int d = k - 1; d >= 0; --d) {
      uint32_t lo, hi;
      mul_wide(F, Lr, lo, hi);
      dig[jb + d] = hi;
      F = lo;
    }
    jb += k;
  }
}

// pair path: f16x2 registers of slot pairs (j0 + 2m, j0 + 2m + 1) into pr[j0/2 + m]
template <int L, int NPR>
__device__ __forceinline__ void extract_word_pairs(uint32_t w, uint32_t (&pr)[NPR], int j0, uint32_t Lr,
                                                   uint32_t L2r, const uint32_t *lut) {
  constexpr int NP = split_parts(L);
  uint32_t rest = w;
  int jb = j0;
#pragma unroll
  for (int pi = 0; pi < NP; ++pi) {
    const int k = split_part(L, pi);
    uint32_t v;
    if (pi < NP - 1) {
      const uint32_t P = (uint32_t)ipow(L, k);
      const uint32_t qq = rest / P;
      v = rest - qq * P;
      rest = qq;
    } else {
      v = rest;
    }
    const uint32_t M = (uint32_t)(((1ull << 32) + ipow(L, k) - 1) / ipow(L, k));
    uint32_t F = v * M;
    if (k & 1) {                       // odd top part: its top digit alone, upper half zero
      uint32_t lo, hi;
      mul_wide(F, Lr, lo, hi);
      pr[(jb + k - 1) >> 1] = hi;
      F = lo;
    }
#pragma unroll
    for (int m = k / 2 - 1; m >= 0; --m) {
      uint32_t lo, hi;
      mul_wide(F, L2r, lo, hi);
      pr[(jb >> 1) + m] = lut[hi];
      F = lo;
    }
    jb += k;
  }
}

// The lane group c = lane % 4 owns words c*WPG .. c*WPG+WPG-1 of a token row.
// Its digit slot u = i*S + j (word i, digit j) sits in k-block u/4 at
// position u%4; positions 0,1 are one f16x2 register, 2,3 the other.
template <int L>
__device__ __forceinline__ void unpack_row(const uint32_t *wrow, int c, uint32_t Lr, uint32_t L2r,
                                           const uint32_t *lut, uint32_t (&reg)[Geo<L>::KB][2]) {
  using G = Geo<L>;
  constexpr int ND = G::KB * 4;
  // words past W of the row read the next bytes of the tile buffer: any 32-bit
  // value unpacks to digits in [0, L) and those slots carry q = 0 (K) or are
  // never written out (V), so no bounds check is needed
  const uint32_t *wr = wrow + c * G::WPG;
  if constexpr (use_pairs(L)) {
    uint32_t pr[ND / 2];
#pragma unroll
    for (int i = 0; i < G::WPG; ++i) extract_word_pairs<L, ND / 2>(wr[i], pr, i * G::S, Lr, L2r, lut);
#pragma unroll
    for (int u = (G::WPG * G::S) / 2; u < ND / 2; ++u) pr[u] = 0u;
#pragma unroll
    for (int kb = 0; kb < G::KB; ++kb) {
      reg[kb][0] = pr[2 * kb];
      reg[kb][1] = pr[2 * kb + 1];
    }
  } else {
    uint32_t dig[ND];
#pragma unroll
    for (int i = 0; i < G::WPG; ++i) extract_word<L, ND>(wr[i], dig, i * G::N, Lr);
#pragma unroll
    for (int u = G::WPG * G::N; u < ND; ++u) dig[u] = 0u;
#pragma unroll
    for (int kb = 0; kb < G::KB; ++kb) {
      reg[kb][0] = __byte_perm(dig[4 * kb], dig[4 * kb + 1], 0x5410);
      reg[kb][1] = __byte_perm(dig[4 * kb + 2], dig[4 * kb + 3], 0x5410);
    }
  }
}

// head-dim index of slot u of lane group c (or -1 for a padding slot)
template <int L>
__device__ __forceinline__ int slot_dim(int c, int u) {
  using G = Geo<L>;
  const int wi = c * G::WPG + u / G::S;
  const int j = u % G::S;
  const int d = wi * G::N + j;
  return (u < G::WPG * G::S && j < G::N && wi < G::W && d < kD) ? d : -1;
}

struct DecParams {
  // pool of this launch
  const uint32_t *kw, *vw;          // [B][Lyr][H][cap][W]
  const float2 *km, *vm;            // [B][Lyr][H][cap]
  const int32_t *count;             // [B]
  int cap;
  // cache geometry
  int B, Lyr, H, H_q, G, layer0, nL;
  const uint16_t *q;                // [B][nL][H_q][D]
  float c2;                         // sm_scale * log2(e)
  float *part;                      // [slabs][NU][G][PART_STRIDE]
  int NU, unit0, S;                 // units per slab, first unit of this launch, splits
  uint32_t *status;
  uint32_t Lrt;                     // the pool's level count (equals the template L)
  int rot;                          // rows stored Hadamard-rotated (needs G <= 4)
  int wait0;                        // polls of each warp's first copy wait (testing aid)
};

constexpr int kMergeBytes = DEC_WARPS * DEC_GMAX * kD * 4 + DEC_WARPS * DEC_GMAX * 3 * 4;
template <int L>
constexpr int kBarOff = (DEC_WARPS * DEC_NST * Geo<L>::TILE_BYTES > kMergeBytes)
                            ? DEC_WARPS * DEC_NST * Geo<L>::TILE_BYTES : kMergeBytes;
template <int L>
constexpr int kQOff = kBarOff<L> + DEC_WARPS * DEC_NST * 8;
static_assert(Geo<6>::TILE_BYTES % 16 == 0 && Geo<5>::TILE_BYTES % 16 == 0 && kMergeBytes % 16 == 0,
              "tile buffers must keep 16-byte alignment for bulk copies");
constexpr int kWaitLimit = 1 << 20;         // mbarrier polls before a copy is declared lost
constexpr int kLutBytes = 64 * 4;           // pair table, L*L <= 36 entries
template <int L>
constexpr int kQfragBytes = Geo<L>::KB * 32 * 8;   // q operand fragments, [kb][lane] x 2 words

template <int L, bool ROT>
__global__ void __launch_bounds__(DEC_WARPS * 32, 4)
decode_pool_kernel(const DecParams p) {
  using Gm = Geo<L>;
  constexpr int KB = Gm::KB, W = Gm::W;
  constexpr float kappa = (L == 2) ? 0.5f : 1.0f;       // keeps p*scale inside f16 range
  extern __shared__ __align__(16) uint8_t smem[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, r = lane >> 2, c = lane & 3;
  const int slab = blockIdx.x / p.S, split = blockIdx.x % p.S;
  const int h = slab % p.H, li = (slab / p.H) % p.nL, b = slab / (p.H * p.nL);
  const int64_t pslab = ((int64_t)b * p.Lyr + p.layer0 + li) * p.H + h;
  const int G = p.G;
  const uint32_t Lr = p.Lrt;                             // == L, opaque to the compiler
  const uint32_t L2r = Lr * Lr;

  // ---- shared memory: per-warp tile rings, their mbarriers, then the q rows
  uint8_t *ring = smem + warp * DEC_NST * Gm::TILE_BYTES;
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + kBarOff<L>) + warp * DEC_NST;
  uint32_t *lut = reinterpret_cast<uint32_t *>(smem + kQOff<L>);      // [L*L] digit pairs (pair path)
  uint2 *qfrag = reinterpret_cast<uint2 *>(smem + kQOff<L> + kLutBytes);            // [KB][32]
  float *qs = reinterpret_cast<float *>(smem + kQOff<L> + kLutBytes + kQfragBytes<L>);  // [G][128]
  if (lane == 0) {
#pragma unroll
    for (int s = 0; s < DEC_NST; ++s) mbar_init(&bars[s], 1);
    fence_mbar_init();
  }
  if (use_pairs(L))
    for (int i = threadIdx.x; i < L * L; i += DEC_WARPS * 32) lut[i] = (uint32_t)(i % L) | ((uint32_t)(i / L) << 16);
  for (int i = threadIdx.x; i < G * kD; i += DEC_WARPS * 32) {
    const int qh = i / kD, d = i % kD;
    const uint16_t hb = p.q[(((int64_t)b * p.nL + li) * p.H_q + h * G + qh) * kD + d];
    qs[i] = __half2float(__ushort_as_half(hb));
  }
  __syncthreads();
  if (ROT) {
    // q' = H q (unnormalised 128-point Hadamard, fp32): q . k = q' . (H k) / 128
    for (int h = 1; h < kD; h <<= 1) {
      for (int i = threadIdx.x; i < G * (kD / 2); i += DEC_WARPS * 32) {
        float *row = qs + (i / (kD / 2)) * kD;
        const int bi = i % (kD / 2), j = (bi / h) * 2 * h + bi % h;
        const float a = row[j], b = row[j + h];
        row[j] = __fadd_rn(a, b);
        row[j + h] = __fsub_rn(a, b);
      }
      __syncthreads();
    }
  }

  // ---- q fragments in slot order (kept in shared memory, one copy per CTA:
  // every warp uses the same fragments), and sum(q) * c2 for this lane's query r
  // With rotated rows q' is not an f16 value: columns 0..3 carry its f16
  // high part and columns 4..7 (G <= 4) its low part, q' - hi, so one MMA
  // gives the logit to about 2^-22 relative.
  float qsum = 0.0f;
  const bool qlo = ROT && r >= 4;
  const int rq = ROT ? (r & 3) : r;
#pragma unroll
  for (int kb = 0; kb < KB; ++kb) {
    uint32_t qv[2];
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
      float v[2];
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int d = slot_dim<L>(c, 4 * kb + 2 * hh + e);
        v[e] = (rq < G && d >= 0) ? qs[rq * kD + d] : 0.0f;
        qsum += qlo ? 0.0f : v[e];
        if (qlo) v[e] = __fsub_rn(v[e], __half2float(__float2half_rn(v[e])));
      }
      qv[hh] = pack_half2(v[0], v[1]);
    }
    if (warp == 0) qfrag[kb * 32 + lane] = make_uint2(qv[0], qv[1]);
  }
  __syncthreads();
  qsum += __shfl_xor_sync(0xffffffffu, qsum, 1);
  qsum += __shfl_xor_sync(0xffffffffu, qsum, 2);
  const float c2k = ROT ? p.c2 * (1.0f / 128.0f) : p.c2;     // rotated: q' . k' / 128
  const float qsc = qsum * c2k;
  const float kscale = c2k * 16777216.0f;              // 2^24: codes are c * 2^-24
  // This lane's two queries are the MMA columns 2c, 2c+1 of the logits.  With
  // G <= 4 the value MMA's columns 4..7 carry the low f16 part of P' for
  // queries 0..3, so lanes c >= 2 mirror the softmax of lane c-2 and one MMA
  // per k-block takes both parts.
  const bool pack_lo = G <= 4;
  const int qc0 = pack_lo ? ((2 * c) & 3) : 2 * c;
  const float qs0 = __shfl_sync(0xffffffffu, qsc, 4 * qc0);        // sum(q)*c2 lives in quad r
  const float qs1 = __shfl_sync(0xffffffffu, qsc, 4 * (qc0 + 1));

  // ---- this CTA's tiles
  const int n = min(p.count[b], p.cap);
  const int ntile = (n + 15) >> 4;
  const int tb = (int)((int64_t)ntile * split / p.S), te = (int)((int64_t)ntile * (split + 1) / p.S);
  const uint32_t *kw = p.kw + pslab * p.cap * W;
  const uint32_t *vw = p.vw + pslab * p.cap * W;
  const float2 *km = p.km + pslab * p.cap;
  const float2 *vm = p.vm + pslab * p.cap;

  // one lane streams the warp's tiles: 4 bulk copies (K words, V words, K meta,
  // V meta) completing on the slot's mbarrier
  constexpr uint32_t kWB = 64 * W;                    // bytes of 16 rows of words
  auto issue = [&](int tile, int slotix) {
    if (lane == 0 && tile < te) {
      uint8_t *dst = ring + slotix * Gm::TILE_BYTES;
      const int t0 = tile * 16;
      fence_proxy_async_smem();
      mbar_expect_tx(&bars[slotix], 2 * kWB + 256);
      bulk_g2s(dst, kw + (int64_t)t0 * W, kWB, &bars[slotix]);
      bulk_g2s(dst + kWB, vw + (int64_t)t0 * W, kWB, &bars[slotix]);
      bulk_g2s(dst + 2 * kWB, km + t0, 128, &bars[slotix]);
      bulk_g2s(dst + 2 * kWB + 128, vm + t0, 128, &bars[slotix]);
    }
  };

  float m_run[2] = {-INFINITY, -INFINITY}, l_run[2] = {0.0f, 0.0f}, mt_run[2] = {0.0f, 0.0f};
  float oacc[KB][4];
#pragma unroll
  for (int kb = 0; kb < KB; ++kb) oacc[kb][0] = oacc[kb][1] = oacc[kb][2] = oacc[kb][3] = 0.0f;

  // ring prologue
  int next = tb + warp;
#pragma unroll
  for (int s = 0; s < DEC_NST - 1; ++s) {
    issue(next, s);
    next += DEC_WARPS;
  }
  int slotix = 0;
  uint32_t parity = 0;                 // bit s: parity of the next phase of slot s
  bool lost = false;
  int tile = tb + warp;
  for (; tile < te; tile += DEC_WARPS) {
    issue(next, (slotix + DEC_NST - 1) % DEC_NST);
    next += DEC_WARPS;
    if (!mbar_wait(&bars[slotix], (parity >> slotix) & 1u, tile == tb + warp ? p.wait0 : kWaitLimit)) {
      lost = true;
      break;
    }
    parity ^= 1u << slotix;
    const uint8_t *tbuf = ring + slotix * Gm::TILE_BYTES;
    const uint32_t *sk = reinterpret_cast<const uint32_t *>(tbuf);
    const uint32_t *sv = reinterpret_cast<const uint32_t *>(tbuf + 64 * W);
    const float2 *skm = reinterpret_cast<const float2 *>(tbuf + 128 * W);
    const float2 *svm = reinterpret_cast<const float2 *>(tbuf + 128 * W + 128);
    const int t0 = tile * 16;

    // ---- logits S = C Q^T: tokens r, r+8 on the MMA rows, queries on the
    // columns; even and odd k-blocks accumulate apart (shorter MMA chain)
    float lg[4];                          // (token r, q0), (r, q1), (r+8, q0), (r+8, q1)
    {
      uint32_t ka[KB][2], kb8[KB][2];
      unpack_row<L>(sk + r * W, c, Lr, L2r, lut, ka);
      unpack_row<L>(sk + (8 + r) * W, c, Lr, L2r, lut, kb8);
      float sa[4] = {0.f, 0.f, 0.f, 0.f}, sb[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int kb = 0; kb < KB; ++kb) {
        const uint2 qb = qfrag[kb * 32 + lane];
        if (kb & 1) mma_16816(sb, ka[kb][0], kb8[kb][0], ka[kb][1], kb8[kb][1], qb.x, qb.y);
        else mma_16816(sa, ka[kb][0], kb8[kb][0], ka[kb][1], kb8[kb][1], qb.x, qb.y);
      }
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        float sv = sa[i] + sb[i];
        const float mirror = __shfl_xor_sync(0xffffffffu, sv, 2);
        if (ROT) sv = sv + mirror;                    // high + low part of q'
        else if (pack_lo && c >= 2) sv = mirror;
        const int tt = (i < 2) ? r : 8 + r;
        const float2 mm = skm[tt];
        const float v = __fmaf_rn(sv, mm.y * kscale, mm.x * ((i & 1) ? qs1 : qs0));
        lg[i] = (t0 + tt < n) ? v : -INFINITY;
      }
    }
    // ---- online softmax (log2 domain): max over the 16 tokens = over r
    float mx0 = fmaxf(lg[0], lg[2]), mx1 = fmaxf(lg[1], lg[3]);
#pragma unroll
    for (int o = 4; o <= 16; o <<= 1) {
      mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, o));
      mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, o));
    }
    const float mn0 = fmaxf(m_run[0], mx0), mn1 = fmaxf(m_run[1], mx1);
    if (__any_sync(0xffffffffu, (mn0 > m_run[0]) | (mn1 > m_run[1]))) {
      const float a0 = (mn0 > m_run[0]) ? ex2_approx(m_run[0] - mn0) : 1.0f;   // m_run=-inf -> 0
      const float a1 = (mn1 > m_run[1]) ? ex2_approx(m_run[1] - mn1) : 1.0f;
      l_run[0] *= a0;
      mt_run[0] *= a0;
      l_run[1] *= a1;
      mt_run[1] *= a1;
#pragma unroll
      for (int kb = 0; kb < KB; ++kb) {
        oacc[kb][0] *= a0;
        oacc[kb][1] *= a1;
        oacc[kb][2] *= a0;
        oacc[kb][3] *= a1;
      }
      m_run[0] = mn0;
      m_run[1] = mn1;
    }
    // P' = p * scale * kappa as an f16 pair hi + lo (hi = RN(P'), lo = RN(P' - hi)):
    // relative error 2^-22 instead of 2^-11 for a single f16
    uint32_t xh[2], xl[2];                // (token r | r+8): f16x2 of columns 2c, 2c+1
#pragma unroll
    for (int g2 = 0; g2 < 2; ++g2) {
      const int tt = g2 ? 8 + r : r;
      const bool ok = t0 + tt < n;
      const float2 vmm = svm[tt];
      float pw[2];
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const float pr = ok ? ex2_approx(lg[2 * g2 + e] - m_run[e]) : 0.0f;
        l_run[e] += pr;
        mt_run[e] += pr * vmm.x;
        pw[e] = pr * (vmm.y * kappa);
      }
      const __half2 hi = __floats2half2_rn(pw[0], pw[1]);
      const float2 hf = __half22float2(hi);
      const __half2 lo = __floats2half2_rn(pw[0] - hf.x, pw[1] - hf.y);
      xh[g2] = *reinterpret_cast<const uint32_t *>(&hi);
      xl[g2] = *reinterpret_cast<const uint32_t *>(&lo);
    }

    // ---- values: O^T += C^T P' (codes and P' transposed in registers)
    uint32_t vr0[KB][2], vr1[KB][2];
    unpack_row<L>(sv + r * W, c, Lr, L2r, lut, vr0);
    unpack_row<L>(sv + (8 + r) * W, c, Lr, L2r, lut, vr1);
    if (pack_lo) {
      // columns 0..3: hi parts (lanes c < 2), 4..7: lo parts (lanes c >= 2)
      const uint32_t b0 = movmatrix_t(c < 2 ? xh[0] : xl[0]);
      const uint32_t b1 = movmatrix_t(c < 2 ? xh[1] : xl[1]);
#pragma unroll
      for (int kb = 0; kb < KB; ++kb) {
        const uint32_t a0 = movmatrix_t(vr0[kb][0]);
        const uint32_t a1 = movmatrix_t(vr0[kb][1]);
        const uint32_t a2 = movmatrix_t(vr1[kb][0]);
        const uint32_t a3 = movmatrix_t(vr1[kb][1]);
        mma_16816(oacc[kb], a0, a1, a2, a3, b0, b1);
      }
    } else {
      const uint32_t bh0 = movmatrix_t(xh[0]), bh1 = movmatrix_t(xh[1]);
      const uint32_t bl0 = movmatrix_t(xl[0]), bl1 = movmatrix_t(xl[1]);
#pragma unroll
      for (int kb = 0; kb < KB; ++kb) {
        const uint32_t a0 = movmatrix_t(vr0[kb][0]);
        const uint32_t a1 = movmatrix_t(vr0[kb][1]);
        const uint32_t a2 = movmatrix_t(vr1[kb][0]);
        const uint32_t a3 = movmatrix_t(vr1[kb][1]);
        mma_16816(oacc[kb], a0, a1, a2, a3, bh0, bh1);
        mma_16816(oacc[kb], a0, a1, a2, a3, bl0, bl1);
      }
    }
    __syncwarp();
    slotix = (slotix + 1) % DEC_NST;
  }
  if (lost) {
    // a copy did not arrive in time: flag it, and give the copies still in
    // flight (tiles tile, tile+4, ... < next) a bounded chance to land before
    // this CTA's shared memory is released
    if (lane == 0) set_flag(p.status, SEMKV_FLAG_TIMEOUT);
    for (int t2 = tile, s2 = slotix; t2 < next && t2 < te; t2 += DEC_WARPS, s2 = (s2 + 1) % DEC_NST)
      mbar_wait(&bars[s2], (parity >> s2) & 1u, kWaitLimit);
  }

  // ---- totals of l and of the min term over the token rows (lanes r); with
  // packed low parts, lanes c >= 2 hold the low-part sums of queries 2c-4, 2c-3
#pragma unroll
  for (int o = 4; o <= 16; o <<= 1)
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      l_run[e] += __shfl_xor_sync(0xffffffffu, l_run[e], o);
      mt_run[e] += __shfl_xor_sync(0xffffffffu, mt_run[e], o);
    }
  if (pack_lo)
#pragma unroll
    for (int kb = 0; kb < KB; ++kb)
#pragma unroll
      for (int i = 0; i < 4; ++i) oacc[kb][i] += __shfl_xor_sync(0xffffffffu, oacc[kb][i], 2);
  const bool owner = !pack_lo || c < 2;

  // ---- merge the 4 warps in shared memory (reuses the ring)
  __syncthreads();
  float *wo = reinterpret_cast<float *>(smem);                        // [warps][GMAX][128]
  float *wst = wo + DEC_WARPS * DEC_GMAX * kD;                        // [warps][GMAX][3]
  if (owner && r == 0)
#pragma unroll
    for (int e = 0; e < 2; ++e)
      if (qc0 + e < G) {
        wst[(warp * DEC_GMAX + qc0 + e) * 3 + 0] = m_run[e];
        wst[(warp * DEC_GMAX + qc0 + e) * 3 + 1] = l_run[e];
        wst[(warp * DEC_GMAX + qc0 + e) * 3 + 2] = mt_run[e];
      }
  constexpr float unscale = 16777216.0f / kappa;
  if (owner)
#pragma unroll
    for (int kb = 0; kb < KB; ++kb) {
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        // slot r (hh=0) or 8+r (hh=1) of block kb belongs to lane group r/2, position (r%2) + 2hh
        const int d = slot_dim<L>(r >> 1, 4 * kb + 2 * hh + (r & 1));
        if (d >= 0) {
          if (qc0 < G) wo[(warp * DEC_GMAX + qc0) * kD + d] = oacc[kb][2 * hh] * unscale;
          if (qc0 + 1 < G) wo[(warp * DEC_GMAX + qc0 + 1) * kD + d] = oacc[kb][2 * hh + 1] * unscale;
        }
      }
    }
  __syncthreads();
  float *dst = p.part + ((int64_t)slab * p.NU + p.unit0 + split) * G * PART_STRIDE;
  for (int i = threadIdx.x; i < G * kD; i += DEC_WARPS * 32) {
    const int qh = i / kD, d = i % kD;
    float M = -INFINITY;
#pragma unroll
    for (int wi = 0; wi < DEC_WARPS; ++wi) M = fmaxf(M, wst[(wi * DEC_GMAX + qh) * 3]);
    float o = 0.0f, lsum = 0.0f;
    if (M != -INFINITY) {
#pragma unroll
      for (int wi = 0; wi < DEC_WARPS; ++wi) {
        const float mw = wst[(wi * DEC_GMAX + qh) * 3];
        if (mw == -INFINITY) continue;
        const float a = ex2_approx(mw - M);
        o += a * (wo[(wi * DEC_GMAX + qh) * kD + d] + wst[(wi * DEC_GMAX + qh) * 3 + 2]);
        lsum += a * wst[(wi * DEC_GMAX + qh) * 3 + 1];
      }
    }
    dst[qh * PART_STRIDE + 4 + d] = o;
    if (d == 0) {
      dst[qh * PART_STRIDE + 0] = M;
      dst[qh * PART_STRIDE + 1] = lsum;
    }
  }
}

// ---- FP16 block: one CTA of 128 threads per (sequence, layer, KV head)
struct BufParams {
  const uint16_t *bk, *bv;     // [B][Lyr][H][block][D]
  int block, buf_len;
  int B, Lyr, H, H_q, G, layer0, nL;
  const uint16_t *q;
  float c2;
  float *part;
  int NU, unit;
  int score_li;                // layer (relative to layer0) whose buffer logits are kept, or -1
  float *logit;                // [B][H_q][block] log2-domain logits of the FP16 tokens
};

// Logits: one warp per token, lane l holding dims 4l..4l+3, so each warp load
// is one whole 256-byte row; the G partial dots are reduced by xor shuffles.
// Values: thread = head dim, each V row read once (coalesced) for all G heads.
__global__ void __launch_bounds__(128) decode_buffer_kernel(const BufParams p) {
  __shared__ float qs[DEC_GMAX][kD];
  __shared__ float pr[DEC_GMAX][128];    // logits (log2 domain), then exp2(logit - max)
  __shared__ float red[DEC_GMAX][2];
  const int slab = blockIdx.x;
  const int h = slab % p.H, li = (slab / p.H) % p.nL, b = slab / (p.H * p.nL);
  const int64_t pslab = ((int64_t)b * p.Lyr + p.layer0 + li) * p.H + h;
  const int G = p.G, n = p.buf_len, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  for (int i = tid; i < G * kD; i += 128)
    qs[i / kD][i % kD] = __half2float(__ushort_as_half(
        p.q[(((int64_t)b * p.nL + li) * p.H_q + h * G + i / kD) * kD + i % kD]));
  __syncthreads();
  const uint16_t *kb = p.bk + pslab * p.block * kD;
  const uint16_t *vb = p.bv + pslab * p.block * kD;
  float qr[DEC_GMAX][4];
#pragma unroll
  for (int qh = 0; qh < DEC_GMAX; ++qh)
#pragma unroll
    for (int i = 0; i < 4; ++i) qr[qh][i] = qh < G ? qs[qh][4 * lane + i] : 0.0f;
  for (int t = warp; t < n; t += 4) {
    const uint2 u = *reinterpret_cast<const uint2 *>(kb + (int64_t)t * kD + 4 * lane);
    const float2 a = __half22float2(*reinterpret_cast<const __half2 *>(&u.x));
    const float2 c = __half22float2(*reinterpret_cast<const __half2 *>(&u.y));
#pragma unroll
    for (int qh = 0; qh < DEC_GMAX; ++qh) {
      if (qh >= G) break;
      float s = fmaf(qr[qh][3], c.y, fmaf(qr[qh][2], c.x, fmaf(qr[qh][1], a.y, qr[qh][0] * a.x)));
#pragma unroll
      for (int o = 16; o >= 1; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
      if (lane == 0) {
        pr[qh][t] = s * p.c2;
        if (li == p.score_li) p.logit[((int64_t)b * p.H_q + h * G + qh) * p.block + t] = s * p.c2;
      }
    }
  }
  __syncthreads();
  for (int qh = warp; qh < G; qh += 4) {
    float mx = -INFINITY;
    for (int t = lane; t < n; t += 32) mx = fmaxf(mx, pr[qh][t]);
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    float sum = 0.0f;
    for (int t = lane; t < n; t += 32) {
      const float e = ex2_approx(pr[qh][t] - mx);
      pr[qh][t] = e;
      sum += e;
    }
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
    if (lane == 0) {
      red[qh][0] = mx;
      red[qh][1] = sum;
    }
  }
  __syncthreads();
  float o[DEC_GMAX];
#pragma unroll
  for (int qh = 0; qh < DEC_GMAX; ++qh) o[qh] = 0.0f;
#pragma unroll 4
  for (int t = 0; t < n; ++t) {
    const float vv = __half2float(__ushort_as_half(vb[(int64_t)t * kD + tid]));
#pragma unroll
    for (int qh = 0; qh < DEC_GMAX; ++qh)
      if (qh < G) o[qh] = fmaf(pr[qh][t], vv, o[qh]);
  }
  float *dst = p.part + ((int64_t)slab * p.NU + p.unit) * G * PART_STRIDE;
#pragma unroll
  for (int qh = 0; qh < DEC_GMAX; ++qh) {
    if (qh >= G) break;
    dst[qh * PART_STRIDE + 4 + tid] = o[qh];
    if (tid == 0) {
      dst[qh * PART_STRIDE + 0] = n > 0 ? red[qh][0] : -INFINITY;
      dst[qh * PART_STRIDE + 1] = n > 0 ? red[qh][1] : 0.0f;
    }
  }
}

// ---- merge all partials of a (sequence, layer, KV head) for one query head:
// CTA = (slab, query head of the group), thread = head dim.  At the scoring
// layer, thread t < buf_len also writes the final softmax probability of
// FP16 token t (same normalisation as the output) for the score accumulation.
struct MergeAcc {
  int rot;                     // pool partials are in the rotated basis: o = (H o' / 128 + o_buf) / l
  int score_li, block, buf_len;
  const float *logit;          // [B][H_q][block]
  float *prob;                 // [B][H_q][block]
};

__global__ void __launch_bounds__(128) decode_merge_kernel(const float *__restrict__ part, int NU,
                                                           int G, int H, int nL, int H_q,
                                                           uint16_t *__restrict__ out, const MergeAcc acc) {
  __shared__ float ot[kD];
  const int slab = blockIdx.x / G, qh = blockIdx.x % G, d = threadIdx.x;
  const int h = slab % H, li = (slab / H) % nL, b = slab / (H * nL);
  const float *pq = part + (int64_t)slab * NU * G * PART_STRIDE + qh * PART_STRIDE;
  float M = -INFINITY;
  for (int u = 0; u < NU; ++u) M = fmaxf(M, pq[(int64_t)u * G * PART_STRIDE]);
  float o = 0.0f, l = 0.0f, ob = 0.0f;        // ob: the FP16 block's share (last unit)
  if (M != -INFINITY) {
    for (int u = 0; u < NU; ++u) {
      const float *pp = pq + (int64_t)u * G * PART_STRIDE;
      const float mu = pp[0];
      if (mu == -INFINITY) continue;
      const float a = ex2_approx(mu - M);
      if (acc.rot && u == NU - 1) ob = a * pp[4 + d];
      else o += a * pp[4 + d];
      l += a * pp[1];
    }
  }
  if (acc.rot) {                               // uniform per CTA
    ot[d] = o;
    __syncthreads();
    for (int hs = 1; hs < kD; hs <<= 1) {
      const float a = ot[d & ~hs], bb = ot[d | hs];
      __syncthreads();
      ot[d] = (d & hs) ? __fsub_rn(a, bb) : __fadd_rn(a, bb);
      __syncthreads();
    }
    o = __fmaf_rn(ot[d], 1.0f / 128.0f, ob);
  }
  const float res = l > 0.0f ? o / l : 0.0f;
  out[(((int64_t)b * nL + li) * H_q + h * G + qh) * kD + d] = __half_as_ushort(__float2half_rn(res));
  if (li == acc.score_li && d < acc.buf_len) {
    const int64_t ix = ((int64_t)b * H_q + h * G + qh) * acc.block + d;
    acc.prob[ix] = (l > 0.0f) ? ex2_approx(acc.logit[ix] - M) / l : 0.0f;
  }
}

// buf_score[b][t] += sum over the query heads, in order, of the probabilities
// of FP16 token t at the scoring layer
__global__ void decode_score_acc_kernel(const float *__restrict__ prob, int H_q, int block, int buf_len,
                                        float *__restrict__ buf_score) {
  const int b = blockIdx.x, t = threadIdx.x;
  if (t >= buf_len) return;
  float s = 0.0f;
  for (int j = 0; j < H_q; ++j) s += prob[((int64_t)b * H_q + j) * block + t];
  buf_score[(int64_t)b * block + t] += s;
}

// ---------------------------------------------------------------- host side
template <int L>
static int pool_smem_bytes(int G) {
  return kQOff<L> + kLutBytes + kQfragBytes<L> + G * kD * 4;
}

template <int L, bool ROT>
static cudaError_t launch_pool(const DecParams &p, int grid, cudaStream_t st) {
  const int smem = pool_smem_bytes<L>(p.G);
  cudaError_t e = prepare_kernel(reinterpret_cast<const void *>(decode_pool_kernel<L, ROT>),
                                 pool_smem_bytes<L>(DEC_GMAX));
  if (e != cudaSuccess) return e;
  decode_pool_kernel<L, ROT><<<grid, DEC_WARPS * 32, smem, st>>>(p);
  return cudaGetLastError();
}

template <bool ROT>
static cudaError_t launch_pool_rt(int L, const DecParams &p, int grid, cudaStream_t st) {
  switch (L) {
    case 2: return launch_pool<2, ROT>(p, grid, st);
    case 3: return launch_pool<3, ROT>(p, grid, st);
    case 4: return launch_pool<4, ROT>(p, grid, st);
    case 5: return launch_pool<5, ROT>(p, grid, st);
    case 6: return launch_pool<6, ROT>(p, grid, st);
    case 7: return launch_pool<7, ROT>(p, grid, st);
    case 8: return launch_pool<8, ROT>(p, grid, st);
    case 9: return launch_pool<9, ROT>(p, grid, st);
    case 10: return launch_pool<10, ROT>(p, grid, st);
    case 11: return launch_pool<11, ROT>(p, grid, st);
    case 12: return launch_pool<12, ROT>(p, grid, st);
    case 13: return launch_pool<13, ROT>(p, grid, st);
    case 14: return launch_pool<14, ROT>(p, grid, st);
    case 15: return launch_pool<15, ROT>(p, grid, st);
    case 16: return launch_pool<16, ROT>(p, grid, st);
    default: return cudaErrorInvalidValue;
  }
}

static cudaError_t launch_pool_any(int L, const DecParams &p, int grid, cudaStream_t st) {
  return p.rot ? launch_pool_rt<true>(L, p, grid, st) : launch_pool_rt<false>(L, p, grid, st);
}

// splits per slab for a pool of capacity cap (host knows only capacities)
static int pool_splits(const semkv_cache &c, int n_layers, int cap) {
  const int sms = device_sm_count();
  const int64_t slabs = (int64_t)c.B * n_layers * c.H;
  // about 1.75 waves of the 4 resident CTAs per SM, rounded to the nearest
  // split count: on the 32-layer prefill cache (256 slabs) 4 splits took
  // 0.584 ms against 0.666 (2), 0.675 (3), 0.616 (5), 0.627 (7), 0.614 (10)
  const int64_t target = (int64_t)sms * 7;
  int64_t S = (target + slabs / 2) / slabs;
  const int64_t max_by_tiles = (cap / 16 + 15) / 16;  // keep >= 16 tiles (4 per warp) per unit
  if (S > max_by_tiles) S = max_by_tiles;
  if (S < 1) S = 1;
  if (S > 64) S = 64;
  return (int)S;
}

size_t decode_ws_bytes(const semkv_cache &c, int n_layers) {
  const int Sh = pool_splits(c, n_layers, c.cap_high), Sl = pool_splits(c, n_layers, c.cap_low);
  const int64_t slabs = (int64_t)c.B * n_layers * c.H;
  const int G = c.H_q / c.H;
  const size_t parts = (size_t)(slabs * (Sh + Sl + 1) * G * PART_STRIDE * sizeof(float));
  return parts + 2 * (size_t)c.B * c.H_q * c.block * sizeof(float);
}

cudaError_t launch_decode(const semkv_cache &c, int layer0, int n_layers, int score_layer, const uint16_t *q,
                          uint16_t *out, float sm_scale, void *ws, uint32_t *status, cudaStream_t st) {
  const int Sh = pool_splits(c, n_layers, c.cap_high), Sl = pool_splits(c, n_layers, c.cap_low);
  const int NU = Sh + Sl + 1;
  const int slabs = c.B * n_layers * c.H;
  const int G = c.H_q / c.H;
  DecParams p;
  p.B = c.B;
  p.Lyr = c.n_layers;
  p.H = c.H;
  p.H_q = c.H_q;
  p.G = G;
  p.layer0 = layer0;
  p.nL = n_layers;
  p.q = q;
  p.c2 = sm_scale * kLog2eF;
  p.part = reinterpret_cast<float *>(ws);
  p.NU = NU;
  p.status = status;
  p.wait0 = first_wait_polls(kWaitLimit);
  cudaError_t e;
  // high pool
  p.kw = c.k_high; p.vw = c.v_high;
  p.km = reinterpret_cast<const float2 *>(c.k_high_meta);
  p.vm = reinterpret_cast<const float2 *>(c.v_high_meta);
  p.count = c.n_high; p.cap = c.cap_high; p.unit0 = 0; p.S = Sh; p.Lrt = (uint32_t)c.L_high;
  p.rot = c.rotate;
  e = launch_pool_any(c.L_high, p, slabs * Sh, st);
  if (e != cudaSuccess) return e;
  // low pool
  p.kw = c.k_low; p.vw = c.v_low;
  p.km = reinterpret_cast<const float2 *>(c.k_low_meta);
  p.vm = reinterpret_cast<const float2 *>(c.v_low_meta);
  p.count = c.n_low; p.cap = c.cap_low; p.unit0 = Sh; p.S = Sl; p.Lrt = (uint32_t)c.L_low;
  e = launch_pool_any(c.L_low, p, slabs * Sl, st);
  if (e != cudaSuccess) return e;
  // FP16 block
  BufParams bp;
  bp.bk = c.buf_k; bp.bv = c.buf_v; bp.block = c.block; bp.buf_len = c.buf_len;
  bp.B = c.B; bp.Lyr = c.n_layers; bp.H = c.H; bp.H_q = c.H_q; bp.G = G;
  bp.layer0 = layer0; bp.nL = n_layers; bp.q = q; bp.c2 = p.c2;
  bp.part = p.part; bp.NU = NU; bp.unit = Sh + Sl;
  // score accumulation at the scoring layer (relative index, -1 = none)
  const int score_li = (score_layer >= layer0 && score_layer < layer0 + n_layers && c.buf_len > 0)
                           ? score_layer - layer0 : -1;
  float *logit = reinterpret_cast<float *>(reinterpret_cast<char *>(ws) +
                                           (size_t)slabs * NU * G * PART_STRIDE * sizeof(float));
  float *prob = logit + (size_t)c.B * c.H_q * c.block;
  bp.score_li = score_li;
  bp.logit = logit;
  decode_buffer_kernel<<<slabs, 128, 0, st>>>(bp);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  MergeAcc ma;
  ma.rot = c.rotate;
  ma.score_li = score_li;
  ma.block = c.block;
  ma.buf_len = c.buf_len;
  ma.logit = logit;
  ma.prob = prob;
  decode_merge_kernel<<<slabs * G, 128, 0, st>>>(p.part, NU, G, c.H, n_layers, c.H_q, out, ma);
  e = cudaGetLastError();
  if (e != cudaSuccess || score_li < 0) return e;
  decode_score_acc_kernel<<<c.B, c.block, 0, st>>>(prob, c.H_q, c.block, c.buf_len, c.buf_score);
  return cudaGetLastError();
}

}  // namespace semkv
