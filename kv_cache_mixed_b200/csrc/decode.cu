// decode.cu -- GQA decode attention over the mixed-precision cache (SemKV,
// Fig. 5: "the mixed-precision quantized KV cache used for decoding"; Fig. 6:
// the most recent partial block stays FP16 during decoding).
//
// Attention works in the code domain, so no row is ever dequantized:
//   q . khat_j = scale_j * (q . c_j) + mn_j * sum(q)
//   sum_j p_j vhat_j = sum_j (p_j scale_j) c_j + (sum_j p_j mn_j) * 1
// Both dot products run on tensor cores (mma.sync m16n8k16, f16 x f16 -> f32).
// Two digits of one token sit in one f16x2 register, which is the operand
// format of the MMA, so a digit is never converted after it is extracted.
//
// Digit extraction, levels that are not powers of two: a word is cut by
// integer division into parts of k digits (L^k <= 1024), and two parts P are
// packed into one f16x2 register.  Then, on both halves at once, one f16 step
//     t = fma(X, c, K) = 1536 + floor(X' / L)     (X = 1024 + P first, then t)
// gives the next floor of the part (exact: every value is an integer below
// 2048, and (c, K) were chosen so that the rounding of X c + K lands on the
// floor for every part value, checked exhaustively), and
//     digit = X + fma(t, -L, 1536 L - B)     (B = X's bias, exact)
// peels one digit off.
//   Keys take the floors x_s = floor(P / L^s) themselves: the raw part P
// (s = 0) costs nothing and a later floor is the low 9 bits of t, one logic
// operation, so a step costs one f16x2 FMA and one logic operation for two
// slots.  The digits d_s = x_s - L x_(s+1) are recovered by linearity on the
// query side: slot s takes the coefficient q_s - L q_(s-1) (an f16 hi + lo
// pair in the spare MMA columns), once per CTA.
//   Values take the digits as normal f16 numbers.  The tensor cores add the
// products into the accumulator by truncation, aligned to its exponent; with
// subnormal value operands (v * 2^-24) the long value sums lost accuracy (the
// worst full-size output error rose from 3.6e-4 to 8e-4 rel-L2), although a
// single product of that size on its own comes out exact.
//   Levels that are powers of two (2, 4, 8, 16) take their digits straight
// out of the bit fields, placed 10 - log2 L bits up in an f16 subnormal
// pattern (d * 2^(10 - log2 L - 24), exact), with the power of two folded
// into the scales.  The pages' layout (groups in whole bits) feeds plain
// digits through the digit chain.
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
// columns, with the digits and P' moved into that operand layout by
// movmatrix.  With at most 4 query heads per KV head, columns 4..7 of the
// value MMA carry the low f16 part of P', so one MMA takes both parts.
#include <functional>

#include "common.cuh"
#include "internal.h"

namespace semkv {

constexpr int DEC_WARPS = 4;
constexpr int DEC_NST = 3;                  // 32-token tiles in flight per warp
constexpr int DEC_GMAX = 8;                 // query heads per KV head handled (M rows used)
constexpr int PART_STRIDE = 132;            // floats per partial: m, l, pad, pad, o[128]
constexpr float kLog2eF = 1.4426950408889634f;

__host__ __device__ constexpr bool is_pow2_level(int L) { return L == 2 || L == 4 || L == 8 || L == 16; }

// ---- f16 digit plan of a level that is not a power of two: part sizes in
// digits (least significant part first; consecutive parts share a register)
// and the f16 bit patterns of (c, K) for the first step (X = 1024 + P) and
// for the later steps (X = 1536 + P).
struct F16Plan {
  int np;
  int part[5];
  uint16_t c0, k0, c1, k1;
};
__host__ __device__ constexpr F16Plan f16_plan(int L) {
  return L == 3    ? F16Plan{4, {5, 5, 5, 5, 0}, 0x3553, 0x64ab, 0x3552, 0x6401}
         : L == 5  ? F16Plan{4, {4, 4, 3, 2, 0}, 0x3265, 0x6533, 0x3263, 0x64cd}
         : L == 6  ? F16Plan{4, {3, 3, 3, 3, 0}, 0x3155, 0x6555, 0x3153, 0x6500}
         : L == 7  ? F16Plan{4, {3, 3, 3, 2, 0}, 0x3094, 0x656d, 0x3093, 0x6524}
         : L == 9  ? F16Plan{5, {2, 2, 2, 2, 2}, 0x2f19, 0x658e, 0x2ee6, 0x655a}
         : L == 10 ? F16Plan{4, {3, 2, 2, 2, 0}, 0x2e68, 0x6599, 0x2e66, 0x6566}
         : L == 11 ? F16Plan{5, {2, 2, 2, 2, 1}, 0x2dc9, 0x65a3, 0x2da6, 0x6578}
         : L == 12 ? F16Plan{4, {2, 2, 2, 2, 0}, 0x2d58, 0x65aa, 0x2d26, 0x6584}
         : L == 13 ? F16Plan{4, {2, 2, 2, 2, 0}, 0x2ce9, 0x65b1, 0x2cc6, 0x658d}
         : L == 14 ? F16Plan{4, {2, 2, 2, 2, 0}, 0x2c98, 0x65b6, 0x2c66, 0x6596}
         : L == 15 ? F16Plan{4, {2, 2, 2, 2, 0}, 0x2c48, 0x65bb, 0x2c3b, 0x659a}
                   : F16Plan{0, {0, 0, 0, 0, 0}, 0, 0, 0, 0};
}
__host__ __device__ constexpr int plan_part(int L, int i) { return i < f16_plan(L).np ? f16_plan(L).part[i] : 0; }
__host__ __device__ constexpr int plan_regs(int L) { return (f16_plan(L).np + 1) / 2; }
__host__ __device__ constexpr int plan_steps(int L, int j) {
  return f16_plan(L).part[2 * j] > (2 * j + 1 < f16_plan(L).np ? f16_plan(L).part[2 * j + 1] : 0)
             ? f16_plan(L).part[2 * j]
             : f16_plan(L).part[2 * j + 1];
}
__host__ __device__ constexpr int plan_offset(int L, int i) {
  int o = 0;
  for (int m = 0; m < i; ++m) o += f16_plan(L).part[m];
  return o;
}

// f16x2 registers (digit pairs) one word yields
__host__ __device__ constexpr int word_regs(int L) {
  if (is_pow2_level(L)) return digits_per_word(L) / 2;
  int r = 0;
  for (int j = 0; j < plan_regs(L); ++j) r += plan_steps(L, j);
  return r;
}
// digit (within the word) in half `h` (0 = low, 1 = high) of register m, or -1 (padding)
__host__ __device__ constexpr int reg_digit(int L, int m, int h) {
  if (is_pow2_level(L)) return m + h * (digits_per_word(L) / 2);
  int base = 0;
  for (int j = 0; j < plan_regs(L); ++j) {
    const int st = plan_steps(L, j);
    if (m < base + st) {
      const int pi = 2 * j + h, s = m - base;
      if (pi >= f16_plan(L).np || s >= f16_plan(L).part[pi]) return -1;
      return plan_offset(L, pi) + s;
    }
    base += st;
  }
  return -1;
}

// step s (floor(P / L^s)) of the part in half `h` of register m, or -1
__host__ __device__ constexpr int reg_step(int L, int m, int h) {
  if (is_pow2_level(L)) return -1;
  int base = 0;
  for (int j = 0; j < plan_regs(L); ++j) {
    const int st = plan_steps(L, j);
    if (m < base + st) {
      const int pi = 2 * j + h, s = m - base;
      return (pi < f16_plan(L).np && s < f16_plan(L).part[pi]) ? s : -1;
    }
    base += st;
  }
  return -1;
}

template <int L>
struct Geo {
  static constexpr int N = digits_per_word(L);       // digits per word
  static constexpr int W = words_per_row(L);         // words per row
  static constexpr int S = 2 * word_regs(L);         // digit slots per word
  static constexpr int SP = (S + 3) / 4 * 4;         // slots per word, padded to whole k-block positions
  static constexpr int RPW = SP / 2;                 // f16x2 registers per word
  static constexpr int KPW = SP / 4;                 // k-blocks per word
  static constexpr int WPG = (W + 3) / 4;            // words per lane group (lane % 4)
  static constexpr int KB = WPG * KPW;               // 16-slot k-blocks
  static constexpr int TT = 32;                      // tokens per tile (two 16-token MMA blocks)
  static constexpr int TILE_BYTES = TT * W * 4 * 2 + TT * 8 * 2;
  // bit-field digits (powers of two) sit SH bits up in an f16 subnormal
  // pattern, d * 2^(SH-24), the highest place that keeps every digit below
  // 2^10, so the value products stay as large as the bit fields allow (see
  // the value digits above)
  static constexpr int SH = is_pow2_level(L) ? 10 - bits_for(L) : 0;
  // operand scales: keys take floors as subnormal patterns (x * 2^-24), values
  // take normal f16 digits (levels that are not powers of two)
  static constexpr float FAC_K = is_pow2_level(L) ? (float)(1 << (24 - SH)) : 16777216.0f;
  static constexpr float FAC_V = is_pow2_level(L) ? (float)(1 << (24 - SH)) : 1.0f;
};

__device__ __forceinline__ uint32_t hfma2(uint32_t a, uint32_t b, uint32_t c) {
  uint32_t d;
  asm("fma.rn.f16x2 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}
__device__ __forceinline__ uint32_t hadd2(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("add.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}
__host__ __device__ constexpr uint32_t h2dup(uint16_t b) { return (uint32_t)b | ((uint32_t)b << 16); }
// f16 bits of a small integer v (|v| < 2^15, exactly representable)
__host__ __device__ constexpr uint16_t f16_int_bits(int v) {
  int a = v < 0 ? -v : v;
  int e = 0;
  while ((a >> (e + 1)) != 0) ++e;                   // a in [2^e, 2^(e+1))
  const int mant = e >= 10 ? (a >> (e - 10)) & 0x3ff : (a << (10 - e)) & 0x3ff;
  return (uint16_t)((v < 0 ? 0x8000 : 0) | ((e + 15) << 10) | mant);
}

// ST f16 digit steps on the packed pair x = (1024 + Pa, 1024 + Pb): out[o0 + s]
// = (digit s of Pa, digit s of Pb), least significant first
template <int L, int ST, int NR>
__device__ __forceinline__ void f16_digit_steps(uint32_t x, uint32_t (&out)[NR], int o0) {
  constexpr uint32_t C0 = h2dup(f16_plan(L).c0), K0 = h2dup(f16_plan(L).k0);
  constexpr uint32_t C1 = h2dup(f16_plan(L).c1), K1 = h2dup(f16_plan(L).k1);
  constexpr uint32_t NEGL = h2dup(f16_int_bits(-L));
  constexpr uint32_t R0 = h2dup(f16_int_bits(1536 * L - 1024)), R1 = h2dup(f16_int_bits(1536 * L - 1536));
  constexpr uint32_t M1024 = h2dup(f16_int_bits(-1024)), M1536 = h2dup(f16_int_bits(-1536));
  if constexpr (ST == 1) {
    out[o0] = hadd2(x, M1024);
  } else {
    uint32_t t = hfma2(x, C0, K0);
    out[o0] = hadd2(x, hfma2(t, NEGL, R0));
#pragma unroll
    for (int s = 1; s < ST - 1; ++s) {
      const uint32_t t2 = hfma2(t, C1, K1);
      out[o0 + s] = hadd2(t, hfma2(t2, NEGL, R1));
      t = t2;
    }
    out[o0 + ST - 1] = hadd2(t, M1536);
  }
}

// ST floor steps on the packed pair xb = (Pa, Pb) (two parts below 1024 as
// raw 16-bit fields): out[o0 + s] = (floor(Pa / L^s), floor(Pb / L^s)) as f16
// subnormal patterns, s = 0 .. ST-1.  The chain is the digit chain's first
// half (X = 1024 + P, then t = 1536 + floor(P / L^s), exact); a floor below
// 512 is then the low 9 bits of t's pattern 0x6600 + floor, one logic
// operation.  Digits follow from the floors, d_s = x_s - L x_(s+1), which the
// key side applies to q once instead of to every token.
template <int L, int ST, int NR>
__device__ __forceinline__ void f16_floor_steps(uint32_t xb, uint32_t (&out)[NR], int o0) {
  constexpr uint32_t C0 = h2dup(f16_plan(L).c0), K0 = h2dup(f16_plan(L).k0);
  constexpr uint32_t C1 = h2dup(f16_plan(L).c1), K1 = h2dup(f16_plan(L).k1);
  out[o0] = xb;
  if constexpr (ST > 1) {
    uint32_t t = hfma2(xb | 0x64006400u, C0, K0);
    out[o0 + 1] = t & 0x01ff01ffu;
#pragma unroll
    for (int s = 2; s < ST; ++s) {
      t = hfma2(t, C1, K1);
      out[o0 + s] = t & 0x01ff01ffu;
    }
  }
}

// floor(x / D) for any 32-bit x, on the fp64 pipe instead of a 32-bit
// multiply-high: x is exact as the double 2^52 + x minus 2^52, inv >= 1/D is
// within 2^-49 of it (relative), so x * inv exceeds x / D by less than 1/D and
// one fma rounded toward zero onto 2^52 (unit last place 1) leaves
// floor(x / D) in the low word.  The integer pipe that the rest of the
// digit extraction loads is spared the word's widest multiply.
template <uint32_t D>
__device__ __forceinline__ uint32_t div_fp64(uint32_t x) {
  constexpr double inv = (1.0 / (double)D) * (1.0 + 0x1p-50);
  const double xd = __hiloint2double(0x43300000, (int)x) - 4503599627370496.0;
  return (uint32_t)__double2loint(__fma_rz(xd, inv, 4503599627370496.0));
}

// register pair J of a word (parts 2J, 2J+1) and the ones after it: the
// parts' floors (keys) or their digits (values); `rest` holds the
// word's digits from part 2J on
template <int L, int J, bool KEYS, int NR>
__device__ __forceinline__ void extract_regs(uint32_t rest, uint32_t (&out)[NR], int o) {
  if constexpr (J < plan_regs(L)) {
    constexpr int ka = plan_part(L, 2 * J), kb = plan_part(L, 2 * J + 1);
    uint32_t v = rest, next = 0;
    if constexpr (J < plan_regs(L) - 1) {
      constexpr uint32_t D = (uint32_t)ipow(L, ka + kb);
      next = div_fp64<D>(rest);
      v = rest - next * D;
    }
    uint32_t xb;
    if constexpr (kb > 0) {
      // (v mod L^ka) | (v div L^ka) << 16: the quotient by multiply-high is
      // exact because v < L^(ka+kb) and L^ka * L^(ka+kb) < 2^32
      constexpr uint32_t Da = (uint32_t)ipow(L, ka);
      const uint32_t q = __umulhi(v, (uint32_t)((0x100000000ull + Da - 1) / Da));
      xb = v + q * (65536u - Da);
    } else {
      xb = v;
    }
    constexpr int st = ka > kb ? ka : kb;
    if constexpr (KEYS) f16_floor_steps<L, st>(xb, out, o);
    else f16_digit_steps<L, st>(xb | 0x64006400u, out, o);
    extract_regs<L, J + 1, KEYS>(next, out, o + st);
  }
}

// the S/2 operand registers of word w, in slot order, into out[o0 ..]: bit
// fields as d << SH subnormal patterns (powers of two), else the parts' floors
// (keys) or digits (values)
template <int L, bool KEYS, int NR>
__device__ __forceinline__ void extract_word(uint32_t w, uint32_t (&out)[NR], int o0) {
  constexpr int SH = Geo<L>::SH;
  // bits [at, at + b) of w moved to bit `to`
  auto field = [&](int at, int to) -> uint32_t { return at >= to ? (w >> (at - to)) : (w << (to - at)); };
  if constexpr (L == 2 || L == 4 || L == 16) {
    constexpr int b = L == 2 ? 1 : (L == 4 ? 2 : 4);
    constexpr uint32_t msk = ((uint32_t)(L - 1) * 0x00010001u) << SH;
#pragma unroll
    for (int m = 0; m < 16 / b; ++m) out[o0 + m] = field(b * m, SH) & msk;          // digits m, m + 16/b
  } else if constexpr (L == 8) {
#pragma unroll
    for (int m = 0; m < 5; ++m)                                                       // digits m, m + 5
      out[o0 + m] = (field(3 * m, SH) & (7u << SH)) | (field(3 * m + 15, 16 + SH) & (7u << (16 + SH)));
  } else {
    extract_regs<L, 0, KEYS>(w, out, o0);
  }
}

// The lane group c = lane % 4 owns words c*WPG .. c*WPG+WPG-1 of a token row.
// Its digit slot u = i*SP + j (word i, slot j) sits in k-block u/4 at position
// u%4; positions 0,1 are one f16x2 register, 2,3 the other.  Word i alone
// fills k-blocks i*KPW .. i*KPW+KPW-1, so a word's registers can go to the
// tensor cores as soon as it is unpacked.  Words past W of the row read the
// next bytes of the tile buffer: every part of any 32-bit value stays a
// finite f16, and those slots carry q = 0 (K) or are never written out (V).
template <int L, bool KEYS>
__device__ __forceinline__ void unpack_word(uint32_t w, uint32_t (&reg)[Geo<L>::RPW]) {
  extract_word<L, KEYS, Geo<L>::RPW>(w, reg, 0);
#pragma unroll
  for (int u = Geo<L>::S / 2; u < Geo<L>::RPW; ++u) reg[u] = 0u;
}

// head-dim index of slot u of lane group c (or -1 for a padding slot)
template <int L>
__device__ __forceinline__ int slot_dim(int c, int u) {
  using G = Geo<L>;
  const int wi = c * G::WPG + u / G::SP;
  const int j = u % G::SP;
  const int dg = j < G::S ? reg_digit(L, j >> 1, j & 1) : -1;
  const int d = wi * G::N + dg;
  return (u < G::WPG * G::SP && dg >= 0 && wi < G::W && d < kD) ? d : -1;
}

// floor step of slot u of lane group c (levels that are not powers of two);
// slot u holds floor(P / L^s) of the part whose digit s is slot_dim(c, u)
template <int L>
__device__ __forceinline__ int slot_step(int c, int u) {
  using G = Geo<L>;
  const int j = u % G::SP;
  return j < G::S ? reg_step(L, j >> 1, j & 1) : -1;
}

// ---- the pages' layout (SEMKV_LAYOUT_PAGES): rows are bit streams of groups
// of g digits in b bits.  KIND 0: levels 2, 4, 16, whose stream is the word
// layout's (read as words); KIND 1: a group splits into two f16 parts (ka, kb)
// that share one register chain; KIND 2: a group is one part below 1024 and
// two groups share a chain; KIND 3: level 8, digits are 3-bit fields.  A block
// of groups (2, or 4 for KIND 2) fills whole k-blocks; the lane group c owns
// blocks c*BPG .. c*BPG+BPG-1 of a row.
template <int L>
struct PGeo {
  static constexpr int g = pages_g(L), b = pages_b(L), NGRP = pages_groups(L), R = pages_row_bits(L);
  static constexpr int TD = kD - (NGRP - 1) * g;                       // digits of the last group
  static constexpr int TB = bits_for(ipow(L, TD));                     // its bits
  static constexpr int KIND = (L == 2 || L == 4 || L == 16) ? 0 : L == 8 ? 3 : (ipow(L, g) <= 1024 ? 2 : 1);
  static constexpr int KA = (g + 1) / 2, KBP = g - KA;                 // KIND 1 parts
  static constexpr int RPGR = KIND == 3 ? 3 : KA;                      // registers per group (KIND 1, 3)
  static constexpr int GB = KIND == 2 ? 4 : 2;                         // groups per block
  static constexpr int RB = KIND == 2 ? 2 * g : 2 * RPGR;              // registers per block
  static constexpr int NBLK = (NGRP + GB - 1) / GB;
  static constexpr int BPG = (NBLK + 3) / 4;                           // blocks per lane group
  static constexpr int KB = BPG * RB / 2;                              // 16-slot k-blocks
  static constexpr int TT = 32;
  static constexpr int CW = ((TT * R + 31) / 32 + 16 + 3) / 4 * 4;     // staged stream words (+ copy slack)
  static constexpr int TILE_BYTES = 2 * CW * 4 + 2 * TT * 4;
  static constexpr float FAC = KIND == 3 ? 16777216.0f : 1.0f;
  static_assert(KIND == 0 || RB % 2 == 0, "a block must fill whole k-block positions");
  static_assert(!pages_supported(L) || KIND != 1 || (ipow(L, KA) <= 1024 && ipow(L, KA) * ipow(L, g) < (1ull << 32)),
                "KIND 1 parts");
};

// b-bit field at stream bit `pos` of the staged buffer (pos >= 0, b <= 20)
__device__ __forceinline__ uint32_t read_bits(const uint32_t *buf, int pos, int nbits) {
  const int w = pos >> 5;
  return __funnelshift_r(buf[w], buf[w + 1], pos & 31) & ((1u << nbits) - 1u);
}

// the RB digit-pair registers of block `blk` of the row whose stream starts at
// buffer bit `rowbit`.  Groups past the row's last one read the bits after it:
// every part stays below 2048, so those slots hold finite values, and they
// carry q = 0 (K) or are never written out (V).
template <int L>
__device__ __forceinline__ void unpack_block(const uint32_t *buf, int rowbit, int blk,
                                             uint32_t (&reg)[PGeo<L>::RB]) {
  using P = PGeo<L>;
  if constexpr (P::KIND == 1) {
#pragma unroll
    for (int q = 0; q < 2; ++q) {
      const int gi = blk * 2 + q;
      const uint32_t V = read_bits(buf, rowbit + gi * P::b, gi == P::NGRP - 1 ? P::TB : P::b);
      constexpr uint32_t Da = (uint32_t)ipow(L, P::KA);
      const uint32_t qq = __umulhi(V, (uint32_t)((0x100000000ull + Da - 1) / Da));
      f16_digit_steps<L, P::KA>((V + qq * (65536u - Da)) | 0x64006400u, reg, q * P::KA);
    }
  } else if constexpr (P::KIND == 2) {
#pragma unroll
    for (int ch = 0; ch < 2; ++ch) {
      const int g0 = blk * 4 + 2 * ch;
      const uint32_t V0 = read_bits(buf, rowbit + g0 * P::b, g0 == P::NGRP - 1 ? P::TB : P::b);
      const uint32_t V1 = read_bits(buf, rowbit + (g0 + 1) * P::b, g0 + 1 == P::NGRP - 1 ? P::TB : P::b);
      f16_digit_steps<L, P::g>((V0 | (V1 << 16)) | 0x64006400u, reg, ch * P::g);
    }
  } else if constexpr (P::KIND == 3) {
#pragma unroll
    for (int q = 0; q < 2; ++q) {
      const int gi = blk * 2 + q;
      const uint32_t V = read_bits(buf, rowbit + gi * P::b, gi == P::NGRP - 1 ? P::TB : P::b);
      reg[3 * q] = (V & 7u) | ((V << 13) & 0x70000u);              // digits 0, 1
      reg[3 * q + 1] = ((V >> 6) & 7u) | ((V << 7) & 0x70000u);    // digits 2, 3
      reg[3 * q + 2] = (V >> 12) & 7u;                              // digit 4
    }
  }
}

// head-dim index of slot u of lane group c in the pages' layout (or -1)
template <int L>
__device__ __forceinline__ int slot_dim_pages(int c, int u) {
  using P = PGeo<L>;
  const int blk = c * P::BPG + u / (2 * P::RB);
  const int j = u % (2 * P::RB), m = j >> 1, h = j & 1;
  int gi, dg, nd;
  if constexpr (P::KIND == 2) {
    gi = blk * 4 + 2 * (m / P::g) + h;
    dg = m % P::g;
    nd = gi == P::NGRP - 1 ? P::TD : P::g;
  } else if constexpr (P::KIND == 3) {
    gi = blk * 2 + m / 3;
    dg = 2 * (m % 3) + h;
    nd = gi == P::NGRP - 1 ? P::TD : P::g;
  } else {
    gi = blk * 2 + m / P::KA;
    const int s = m % P::KA;
    const int ka = (gi == P::NGRP - 1 && P::TD < P::KA) ? P::TD : P::KA;
    const int kb = (gi == P::NGRP - 1 ? P::TD : P::g) - ka;
    dg = h == 0 ? (s < ka ? s : -1) : (s < kb ? P::KA + s : -1);
    nd = gi == P::NGRP - 1 ? P::TD : P::g;
  }
  const int d = gi * P::g + dg;
  return (u < P::BPG * 2 * P::RB && gi < P::NGRP && dg >= 0 && dg < nd && d < kD) ? d : -1;
}

// slot map of either layout
template <int L, bool GROUPS>
__device__ __forceinline__ int slot_dim_any(int c, int u) {
  if constexpr (GROUPS) return slot_dim_pages<L>(c, u);
  else return slot_dim<L>(c, u);
}

// one pool class of a launch
struct PoolArgs {
  const uint32_t *kw, *vw;          // [B][Lyr][H][slab_words] (words: [cap][W]; pages: bit stream)
  const float2 *km, *vm;            // [B][Lyr][H][cap] (pages: __half2 per row)
  const int32_t *count;             // [B]
  int cap;
  int S, unit0;                     // splits per slab, first partial unit of this class
  int64_t slab_words;               // code words of one (sequence, layer, head) slab
};

struct DecParams {
  // the classes of this launch: CTAs [0, slabs*pool[0].S) take class 0, the
  // next slabs*pool[1].S take class 1 (pool[1].S = 0 when a launch has one class)
  PoolArgs pool[2];
  int slabs;
  // cache geometry
  int B, Lyr, H, H_q, G, layer0, nL;
  const uint16_t *q;                // [B][nL][H_q][D]
  float c2;                         // sm_scale * log2(e)
  float *part;                      // [slabs][NU][G][PART_STRIDE]
  int NU;                           // partial units per slab
  uint32_t *status;
  int rot;                          // rows stored Hadamard-rotated (needs G <= 4)
  int wait0;                        // polls of each warp's first copy wait (testing aid)
};

constexpr int kMergeBytes = DEC_WARPS * DEC_GMAX * kD * 4 + DEC_WARPS * DEC_GMAX * 3 * 4;
constexpr int kWaitLimit = 1 << 20;         // mbarrier polls before a copy is declared lost
// shared-memory layout of a pool CTA: per-warp tile rings, their mbarriers, the
// q fragments and the q rows
template <int L, bool PAGES, bool WIDE>
struct Lay {
  static constexpr bool GROUPS = PAGES && PGeo<L>::KIND != 0;          // read the pages' groups
  static constexpr int TILE = GROUPS ? PGeo<L>::TILE_BYTES : (PAGES ? Geo<L>::TT * Geo<L>::W * 8 + Geo<L>::TT * 8
                                                                     : Geo<L>::TILE_BYTES);
  static constexpr int KB = GROUPS ? PGeo<L>::KB : Geo<L>::KB;
  static constexpr bool FLOORS = !GROUPS && !is_pow2_level(L);        // key slots hold floors, not digits
  static constexpr int BAR = (DEC_WARPS * DEC_NST * TILE > kMergeBytes) ? DEC_WARPS * DEC_NST * TILE : kMergeBytes;
  static constexpr int QOFF = BAR + DEC_WARPS * DEC_NST * 8;
  // q operand fragments, [kb][lane] x 2 words; with floors and G > 4 a second
  // set holds the low f16 parts (they cannot ride in columns 4..7)
  static constexpr int QFRAG = KB * 32 * 8 * (FLOORS && WIDE ? 2 : 1);
  static_assert(TILE % 16 == 0 && kMergeBytes % 16 == 0, "tile buffers must keep 16-byte alignment for bulk copies");
};

// One CTA's share of one pool class: tiles [tb, te) of split `split` of slab
// `slab`.  WIDE: more than 4 query heads per KV head (G > 4).
template <int L, bool ROT, bool PAGES, bool WIDE>
__device__ __forceinline__ void pool_body(const DecParams &p, const PoolArgs &pa, int slab, int split,
                                          uint8_t *smem) {
  using Gm = Geo<L>;
  using Ly = Lay<L, PAGES, WIDE>;
  using Pg = PGeo<L>;
  constexpr bool GROUPS = Ly::GROUPS;            // the pages' groups (else 32-bit words)
  constexpr bool FLOORS = Ly::FLOORS;            // key slots hold floor(P / L^s), not digits
  constexpr int KB = Ly::KB, W = Gm::W;
  constexpr float FAC_K = GROUPS ? Pg::FAC : Gm::FAC_K;          // operand scales, keys and values
  constexpr float FAC_V = GROUPS ? Pg::FAC : Gm::FAC_V;
  constexpr float kappa = (L == 2) ? 0.5f : 1.0f;       // keeps p*scale inside f16 range
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, r = lane >> 2, c = lane & 3;
  const int h = slab % p.H, li = (slab / p.H) % p.nL, b = slab / (p.H * p.nL);
  const int64_t pslab = ((int64_t)b * p.Lyr + p.layer0 + li) * p.H + h;
  const int G = p.G;

  // ---- shared memory: per-warp tile rings, their mbarriers, then the q rows
  uint8_t *ring = smem + warp * DEC_NST * Ly::TILE;
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + Ly::BAR) + warp * DEC_NST;
  uint2 *qfrag = reinterpret_cast<uint2 *>(smem + Ly::QOFF);                          // [KB][32]
  float *qs = reinterpret_cast<float *>(smem + Ly::QOFF + Ly::QFRAG);                // [G][128]
  if (lane == 0) {
#pragma unroll
    for (int s = 0; s < DEC_NST; ++s) mbar_init(&bars[s], 1);
    fence_mbar_init();
  }
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
  // A slot's coefficient is q_d for a digit slot.  For a floor slot x_s of a
  // part it is q_d - L q_(d-1) for s >= 1 (d-1: the part's previous digit)
  // and q_d for s = 0, since sum_s q_s d_s = q_0 x_0 + sum_(s>=1) (q_s - L
  // q_(s-1)) x_s over a part's floors x_s = floor(P / L^s).
  // A coefficient that is not an f16 value (rotated rows, floor slots) goes as
  // an f16 pair hi + lo, to about 2^-22 relative: with G <= 4 columns 0..3
  // carry hi and columns 4..7 lo, so one MMA takes both; with G > 4 the lo
  // parts get MMAs of their own (second fragment set).
  // Otherwise, with G <= 4, columns 4..7 repeat the query heads of columns
  // 0..3, so every lane of a row gets the logits of its head pair.
  float qsum = 0.0f;
  constexpr bool lo_cols = (ROT || FLOORS) && !WIDE;
  constexpr bool lo_pass = FLOORS && WIDE;
  const bool qlo = lo_cols && r >= 4;
  const int rq = WIDE ? r : (r & 3);
#pragma unroll
  for (int kb = 0; kb < KB; ++kb) {
    uint32_t qv[2], ql[2];
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
      float v[2], vl[2];
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int u = 4 * kb + 2 * hh + e;
        const int d = slot_dim_any<L, GROUPS>(c, u);
        const bool ok = rq < G && d >= 0;
        const float qd = ok ? qs[rq * kD + d] : 0.0f;
        float cf = qd;
        if constexpr (FLOORS) {
          if (ok && slot_step<L>(c, u) > 0) cf = __fmaf_rn(-(float)L, qs[rq * kD + d - 1], qd);
        }
        qsum += qlo ? 0.0f : qd;
        vl[e] = __fsub_rn(cf, __half2float(__float2half_rn(cf)));
        v[e] = qlo ? vl[e] : cf;
      }
      qv[hh] = pack_half2(v[0], v[1]);
      ql[hh] = pack_half2(vl[0], vl[1]);
    }
    if (warp == 0) {
      qfrag[kb * 32 + lane] = make_uint2(qv[0], qv[1]);
      if constexpr (lo_pass) qfrag[(KB + kb) * 32 + lane] = make_uint2(ql[0], ql[1]);
    }
  }
  __syncthreads();
  qsum += __shfl_xor_sync(0xffffffffu, qsum, 1);
  qsum += __shfl_xor_sync(0xffffffffu, qsum, 2);
  const float c2k = ROT ? p.c2 * (1.0f / 128.0f) : p.c2;     // rotated: q' . k' / 128
  const float qsc = qsum * c2k;
  const float kscale = c2k * FAC_K;                    // key operands are v / FAC_K
  // This lane's two queries are the MMA columns 2c, 2c+1 of the logits.  With
  // G <= 4 columns 4..7 repeat heads 0..3 (or carry q''s low part when
  // rotated), so lane c >= 2 holds the same two heads as lane c-2 and the two
  // lanes split each tile's blocks; the value MMA's columns 4..7 carry the low
  // f16 part of P', so one MMA per k-block takes both parts.
  constexpr bool pack_lo = !WIDE;
  const int qc0 = pack_lo ? ((2 * c) & 3) : 2 * c;
  const float qs0 = __shfl_sync(0xffffffffu, qsc, 4 * qc0);        // sum(q)*c2 lives in quad r
  const float qs1 = __shfl_sync(0xffffffffu, qsc, 4 * (qc0 + 1));

  // ---- this CTA's tiles (32 tokens each)
  constexpr int TT = Gm::TT;
  constexpr int UPG = GROUPS ? Pg::BPG : Gm::WPG;     // units (words, or blocks of groups) per lane group
  constexpr int RPU = GROUPS ? Pg::RB : Gm::RPW;      // f16x2 registers per unit
  constexpr int KPU = RPU / 2;                        // k-blocks per unit
  // staged tile: K codes, V codes, K meta, V meta (meta: 8 B a row, 4 B in the pages' layout)
  constexpr int CWB = GROUPS ? Pg::CW * 4 : TT * W * 4;
  constexpr int MB = PAGES ? 4 : 8;
  const int n = min(pa.count[b], pa.cap);
  const int ntile = (n + TT - 1) / TT;
  const int tb = (int)((int64_t)ntile * split / pa.S), te = (int)((int64_t)ntile * (split + 1) / pa.S);
  const uint32_t *kw = pa.kw + pslab * pa.slab_words;
  const uint32_t *vw = pa.vw + pslab * pa.slab_words;
  const uint8_t *km = reinterpret_cast<const uint8_t *>(pa.km) + pslab * pa.cap * MB;
  const uint8_t *vm = reinterpret_cast<const uint8_t *>(pa.vm) + pslab * pa.cap * MB;

  // one lane streams the warp's tiles: 4 bulk copies (K words, V words, K meta,
  // V meta) completing on the slot's mbarrier.  Capacities are multiples of
  // 16, so the last tile of a slab may hold 16 rows: the copies stop at the
  // capacity, and the rows of the buffer past it are masked like rows past n.
  // In the pages' layout the tile's rows are stream bits [t0 R, (t0+nt) R): the
  // copy takes the 16-byte aligned words around them, and the tile's first row
  // starts at buffer bit (t0 R) mod 128.
  auto issue = [&](int tile, int slotix) {
    if (lane == 0 && tile < te) {
      uint8_t *dst = ring + slotix * Ly::TILE;
      const int t0 = tile * TT;
      const int nt = min(TT, pa.cap - t0);
      int64_t w0 = (int64_t)t0 * W;
      uint32_t wb = (uint32_t)nt * W * 4;
      if constexpr (GROUPS) {
        w0 = ((int64_t)t0 * Pg::R >> 5) & ~3ll;
        const int64_t w1 = ((((int64_t)(t0 + nt) * Pg::R + 31) >> 5) + 3) & ~3ll;
        wb = (uint32_t)(w1 - w0) * 4;
      }
      fence_proxy_async_smem();
      mbar_expect_tx(&bars[slotix], 2 * wb + 2 * (uint32_t)nt * MB);
      bulk_g2s(dst, kw + w0, wb, &bars[slotix]);
      bulk_g2s(dst + CWB, vw + w0, wb, &bars[slotix]);
      bulk_g2s(dst + 2 * CWB, km + (int64_t)t0 * MB, (uint32_t)nt * MB, &bars[slotix]);
      bulk_g2s(dst + 2 * CWB + TT * MB, vm + (int64_t)t0 * MB, (uint32_t)nt * MB, &bars[slotix]);
    }
  };

  float m_run[2] = {-INFINITY, -INFINITY}, l_run[2] = {0.0f, 0.0f}, mt_run[2] = {0.0f, 0.0f};
  float oacc[KB][4];
#pragma unroll
  for (int kb = 0; kb < KB; ++kb) oacc[kb][0] = oacc[kb][1] = oacc[kb][2] = oacc[kb][3] = 0.0f;
  // With G <= 4 the two 16-token blocks of a tile split the softmax: lanes
  // c < 2 take block 0, lanes c >= 2 block 1 (their MMA columns duplicate the
  // same query heads); with G > 4 every lane takes both blocks.
  const int nb = pack_lo ? 1 : 2;
  const int myblk = pack_lo ? (c >> 1) : 0;

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
    const uint8_t *tbuf = ring + slotix * Ly::TILE;
    const uint32_t *sk = reinterpret_cast<const uint32_t *>(tbuf);
    const uint32_t *sv = reinterpret_cast<const uint32_t *>(tbuf + CWB);
    const uint8_t *smk = tbuf + 2 * CWB, *smv = tbuf + 2 * CWB + TT * MB;
    // (min, scale) of staged row tt
    auto meta = [&](const uint8_t *base, int tt) -> float2 {
      if constexpr (PAGES) return __half22float2(reinterpret_cast<const __half2 *>(base)[tt]);
      else return reinterpret_cast<const float2 *>(base)[tt];
    };
    const int t0 = tile * TT;
    const bool full = t0 + TT <= n;
    const int rowbit0 = GROUPS ? (int)(((int64_t)t0 * Pg::R) & 127) : 0;
    // the f16x2 operand registers of unit i of staged row `row` (keys: the
    // parts' floors; values: digits)
    auto unpack = [&](bool keys, const uint32_t *buf, int row, int i, uint32_t (&regs)[RPU]) {
      if constexpr (GROUPS) {
        unpack_block<L>(buf, rowbit0 + row * Pg::R, c * UPG + i, regs);
      } else {
        if (keys) unpack_word<L, true>(buf[row * W + c * UPG + i], regs);
        else unpack_word<L, false>(buf[row * W + c * UPG + i], regs);
      }
    };
    constexpr bool KEYS = true, VALUES = false;

    // ---- logits S = C Q^T per 16-token block: tokens on the MMA rows (r, r+8),
    // query heads on the columns; each word goes to the tensor cores as soon
    // as it is unpacked
    float sacc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
    for (int i = 0; i < UPG; ++i) {
#pragma unroll
      for (int blk = 0; blk < 2; ++blk) {
        uint32_t ra[RPU], rb[RPU];
        unpack(KEYS, sk, blk * 16 + r, i, ra);
        unpack(KEYS, sk, blk * 16 + 8 + r, i, rb);
#pragma unroll
        for (int m = 0; m < KPU; ++m) {
          const uint2 qb = qfrag[(i * KPU + m) * 32 + lane];
          mma_16816(sacc[blk], ra[2 * m], rb[2 * m], ra[2 * m + 1], rb[2 * m + 1], qb.x, qb.y);
          if constexpr (lo_pass) {
            const uint2 qc = qfrag[(KB + i * KPU + m) * 32 + lane];
            mma_16816(sacc[blk], ra[2 * m], rb[2 * m], ra[2 * m + 1], rb[2 * m + 1], qc.x, qc.y);
          }
        }
      }
    }
    float lg[2][4];                       // per lane block j: (token r, q0), (r, q1), (r+8, q0), (r+8, q1)
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      if (j >= nb) break;
      float s4[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        float a0 = sacc[0][i], a1 = sacc[1][i];
        if constexpr (lo_cols) {                      // high + low part of the coefficients
          a0 += __shfl_xor_sync(0xffffffffu, a0, 2);
          a1 += __shfl_xor_sync(0xffffffffu, a1, 2);
        }
        s4[i] = (pack_lo ? myblk : j) ? a1 : a0;
      }
      const int tt = (pack_lo ? myblk : j) * 16 + r;
      const float2 m0 = meta(smk, tt), m1 = meta(smk, tt + 8);
      lg[j][0] = __fmaf_rn(s4[0], m0.y * kscale, m0.x * qs0);
      lg[j][1] = __fmaf_rn(s4[1], m0.y * kscale, m0.x * qs1);
      lg[j][2] = __fmaf_rn(s4[2], m1.y * kscale, m1.x * qs0);
      lg[j][3] = __fmaf_rn(s4[3], m1.y * kscale, m1.x * qs1);
      if (!full) {
        if (t0 + tt >= n) lg[j][0] = lg[j][1] = -INFINITY;
        if (t0 + tt + 8 >= n) lg[j][2] = lg[j][3] = -INFINITY;
      }
    }
    // ---- online softmax (log2 domain): max over the tile's tokens, shared
    // by the two lanes (c, c^2) of a head pair when they split the blocks
    float mx0 = fmaxf(lg[0][0], lg[0][2]), mx1 = fmaxf(lg[0][1], lg[0][3]);
    if (!pack_lo) {
      mx0 = fmaxf(mx0, fmaxf(lg[1][0], lg[1][2]));
      mx1 = fmaxf(mx1, fmaxf(lg[1][1], lg[1][3]));
    }
#pragma unroll
    for (int o = 4; o <= 16; o <<= 1) {
      mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, o));
      mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, o));
    }
    if (pack_lo) {
      mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
      mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
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
    uint32_t xh[2][2], xl[2][2];          // [lane block][token r | r+8]: f16x2 of this lane's two heads
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      if (j >= nb) break;
#pragma unroll
      for (int g2 = 0; g2 < 2; ++g2) {
        const int tt = (pack_lo ? myblk : j) * 16 + 8 * g2 + r;
        const bool ok = full || t0 + tt < n;
        // rows past the count hold whatever the pool memory held: keep them out
        const float2 vmm = ok ? meta(smv, tt) : make_float2(0.0f, 0.0f);
        float pw[2];
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const float pr = ok ? ex2_approx(lg[j][2 * g2 + e] - m_run[e]) : 0.0f;
          l_run[e] += pr;
          mt_run[e] += pr * vmm.x;
          pw[e] = pr * (vmm.y * kappa);
        }
        const __half2 hi = __floats2half2_rn(pw[0], pw[1]);
        const float2 hf = __half22float2(hi);
        const __half2 lo = __floats2half2_rn(pw[0] - hf.x, pw[1] - hf.y);
        xh[j][g2] = *reinterpret_cast<const uint32_t *>(&hi);
        xl[j][g2] = *reinterpret_cast<const uint32_t *>(&lo);
      }
    }
    // ---- B operands of the value MMAs: 8x8 matrices (rows = 8 tokens, columns
    // 0..3 the hi parts and 4..7 the lo parts of the query heads), transposed
    uint32_t bh[2][2], bl[2][2];          // [block][token r | r+8]
    if (pack_lo) {
#pragma unroll
      for (int g2 = 0; g2 < 2; ++g2) {
        // lane (r, c) supplies columns 2c, 2c+1: hi parts from the block-0 lane
        // of its head pair, lo parts from the partner lane c^2
        const uint32_t sxh = __shfl_xor_sync(0xffffffffu, xh[0][g2], 2);
        const uint32_t sxl = __shfl_xor_sync(0xffffffffu, xl[0][g2], 2);
        bh[0][g2] = movmatrix_t(c < 2 ? xh[0][g2] : sxl);
        bh[1][g2] = movmatrix_t(c < 2 ? sxh : xl[0][g2]);
      }
    } else {
#pragma unroll
      for (int j = 0; j < 2; ++j)
#pragma unroll
        for (int g2 = 0; g2 < 2; ++g2) {
          bh[j][g2] = movmatrix_t(xh[j][g2]);
          bl[j][g2] = movmatrix_t(xl[j][g2]);
        }
    }

    // ---- values: O^T += C^T P' (codes transposed in registers), word by word
#pragma unroll
    for (int i = 0; i < UPG; ++i) {
#pragma unroll
      for (int blk = 0; blk < 2; ++blk) {
        uint32_t ra[RPU], rb[RPU];
        unpack(VALUES, sv, blk * 16 + r, i, ra);
        unpack(VALUES, sv, blk * 16 + 8 + r, i, rb);
#pragma unroll
        for (int m = 0; m < KPU; ++m) {
          const int kb = i * KPU + m;
          const uint32_t a0 = movmatrix_t(ra[2 * m]);
          const uint32_t a1 = movmatrix_t(ra[2 * m + 1]);
          const uint32_t a2 = movmatrix_t(rb[2 * m]);
          const uint32_t a3 = movmatrix_t(rb[2 * m + 1]);
          mma_16816(oacc[kb], a0, a1, a2, a3, bh[blk][0], bh[blk][1]);
          if constexpr (!pack_lo) mma_16816(oacc[kb], a0, a1, a2, a3, bl[blk][0], bl[blk][1]);
        }
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
  if (pack_lo)          // lanes c and c^2 took the two blocks of every tile, with the same running max
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      l_run[e] += __shfl_xor_sync(0xffffffffu, l_run[e], 2);
      mt_run[e] += __shfl_xor_sync(0xffffffffu, mt_run[e], 2);
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
  constexpr float unscale = FAC_V / kappa;
  if (owner)
#pragma unroll
    for (int kb = 0; kb < KB; ++kb) {
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        // slot r (hh=0) or 8+r (hh=1) of block kb belongs to lane group r/2, position (r%2) + 2hh
        // (both candidate slots are compile-time, so the slot table folds away)
        const int dA = slot_dim_any<L, GROUPS>(r >> 1, 4 * kb + 2 * hh);
        const int dB = slot_dim_any<L, GROUPS>(r >> 1, 4 * kb + 2 * hh + 1);
        const int d = (r & 1) ? dB : dA;
        if (d >= 0) {
          if (qc0 < G) wo[(warp * DEC_GMAX + qc0) * kD + d] = oacc[kb][2 * hh] * unscale;
          if (qc0 + 1 < G) wo[(warp * DEC_GMAX + qc0 + 1) * kD + d] = oacc[kb][2 * hh + 1] * unscale;
        }
      }
    }
  __syncthreads();
  float *dst = p.part + ((int64_t)slab * p.NU + pa.unit0 + split) * G * PART_STRIDE;
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

// Both pool classes in one launch (LA: class 0 = high, LB: class 1 = low), so
// that the CTAs of the two pools fill the same waves; a launch with one class
// uses LA == LB.
template <int LA, int LB, bool ROT, bool PAGES, bool WIDE>
__global__ void __launch_bounds__(DEC_WARPS * 32, 4) decode_pool_kernel(const DecParams p) {
  extern __shared__ __align__(16) uint8_t smem[];
  // the FP16-block kernel after it reads nothing this kernel writes: let it start
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const int n0 = p.slabs * p.pool[0].S;
  const int cls = (int)blockIdx.x >= n0;
  const int i = cls ? (int)blockIdx.x - n0 : (int)blockIdx.x;
  const int S = p.pool[cls].S;
  if constexpr (LA == LB) {
    pool_body<LA, ROT, PAGES, WIDE>(p, p.pool[cls], i / S, i % S, smem);
  } else {
    if (cls == 0) pool_body<LA, ROT, PAGES, WIDE>(p, p.pool[0], i / S, i % S, smem);
    else pool_body<LB, ROT, PAGES, WIDE>(p, p.pool[1], i / S, i % S, smem);
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
  // Launched as a dependent of the pool kernel, it may run alongside it; it
  // finishes only after the pool kernel has, so the merge kernel that waits
  // for it sees both kernels' partials.  (Every thread gets here.)
  asm volatile("griddepcontrol.wait;" ::: "memory");
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
template <int L, bool PAGES, bool WIDE>
static int pool_smem_bytes(int G) {
  return Lay<L, PAGES, WIDE>::QOFF + Lay<L, PAGES, WIDE>::QFRAG + G * kD * 4;
}

// instances that exist: the pages' layout for its supported levels, unrotated;
// rotation only with G <= 4
template <int LA, int LB, bool ROT, bool PAGES, bool WIDE>
constexpr bool pools_instance() {
  return (!PAGES || (!ROT && pages_supported(LA) && pages_supported(LB))) && !(ROT && WIDE);
}

template <int LA, int LB, bool ROT, bool PAGES, bool WIDE>
static cudaError_t launch_pools(const DecParams &p, int grid, cudaStream_t st) {
  if constexpr (!pools_instance<LA, LB, ROT, PAGES, WIDE>()) {
    return cudaErrorInvalidValue;
  } else {
    const int sa = pool_smem_bytes<LA, PAGES, WIDE>(p.G), sb = pool_smem_bytes<LB, PAGES, WIDE>(p.G);
    const int ma = pool_smem_bytes<LA, PAGES, WIDE>(DEC_GMAX), mb = pool_smem_bytes<LB, PAGES, WIDE>(DEC_GMAX);
    const void *fn = reinterpret_cast<const void *>(decode_pool_kernel<LA, LB, ROT, PAGES, WIDE>);
    cudaError_t e = prepare_kernel(fn, ma > mb ? ma : mb);
    if (e != cudaSuccess) return e;
    if (grid > 0) decode_pool_kernel<LA, LB, ROT, PAGES, WIDE><<<grid, DEC_WARPS * 32, sa > sb ? sa : sb, st>>>(p);
    return cudaGetLastError();
  }
}

// resident CTAs per SM of the kernel instance <LA, LB, ROT, PAGES, WIDE> (queried once per device)
template <int LA, int LB, bool ROT, bool PAGES, bool WIDE>
static int pools_occupancy(int G) {
  if constexpr (!pools_instance<LA, LB, ROT, PAGES, WIDE>()) {
    return 1;
  } else {
    const int sa = pool_smem_bytes<LA, PAGES, WIDE>(G), sb = pool_smem_bytes<LB, PAGES, WIDE>(G);
    const int ma = pool_smem_bytes<LA, PAGES, WIDE>(DEC_GMAX), mb = pool_smem_bytes<LB, PAGES, WIDE>(DEC_GMAX);
    const void *fn = reinterpret_cast<const void *>(decode_pool_kernel<LA, LB, ROT, PAGES, WIDE>);
    int nb = 1;
    if (prepare_kernel(fn, ma > mb ? ma : mb) != cudaSuccess ||
        kernel_occupancy(fn, DEC_WARPS * 32, sa > sb ? sa : sb, &nb) != cudaSuccess)
      return 1;
    return nb;
  }
}

// F is called as f.template run<LA, LB>() for the instance of the levels
template <typename F>
static auto dispatch_one(int L, F &f) {
  switch (L) {
    case 2: return f.template run<2, 2>();
    case 3: return f.template run<3, 3>();
    case 4: return f.template run<4, 4>();
    case 5: return f.template run<5, 5>();
    case 6: return f.template run<6, 6>();
    case 7: return f.template run<7, 7>();
    case 8: return f.template run<8, 8>();
    case 9: return f.template run<9, 9>();
    case 10: return f.template run<10, 10>();
    case 11: return f.template run<11, 11>();
    case 12: return f.template run<12, 12>();
    case 13: return f.template run<13, 13>();
    case 14: return f.template run<14, 14>();
    case 15: return f.template run<15, 15>();
    default: return f.template run<16, 16>();
  }
}
// both classes in one launch: every uniform pair, and the adjacent pairs the
// pages use (6/5) or sweep (5/4, 8/6, 16/8); other pairs take two launches
static bool has_merged(int Lh, int Ll) {
  return Lh == Ll || (Lh == 6 && Ll == 5) || (Lh == 5 && Ll == 4) || (Lh == 8 && Ll == 6) || (Lh == 16 && Ll == 8);
}
template <typename F>
static auto dispatch_merged(int Lh, int Ll, F &f) {
  if (Lh == Ll) return dispatch_one(Lh, f);
  if (Lh == 6 && Ll == 5) return f.template run<6, 5>();
  if (Lh == 5 && Ll == 4) return f.template run<5, 4>();
  if (Lh == 8 && Ll == 6) return f.template run<8, 6>();
  return f.template run<16, 8>();
}

template <bool ROT, bool PAGES, bool WIDE>
struct LaunchF {
  const DecParams &p;
  int grid;
  cudaStream_t st;
  template <int LA, int LB>
  cudaError_t run() { return launch_pools<LA, LB, ROT, PAGES, WIDE>(p, grid, st); }
};
template <bool ROT, bool PAGES, bool WIDE>
struct OccF {
  int G;
  template <int LA, int LB>
  int run() { return pools_occupancy<LA, LB, ROT, PAGES, WIDE>(G); }
};

// F<ROT, PAGES, WIDE> for the cache's layout, rotation and group size, built
// from `args` and dispatched over the levels
template <template <bool, bool, bool> class F, typename... A>
static auto dispatch_cache(bool merged, int Lh, int Ll, const semkv_cache &c, A... args) {
  const bool wide = c.H_q / c.H > 4;
  auto go = [&](auto f) { return merged ? dispatch_merged(Lh, Ll, f) : dispatch_one(Lh, f); };
  if (c.layout == SEMKV_LAYOUT_PAGES)
    return wide ? go(F<false, true, true>{args...}) : go(F<false, true, false>{args...});
  if (c.rotate) return go(F<true, false, false>{args...});       // rotation needs G <= 4
  return wide ? go(F<false, false, true>{args...}) : go(F<false, false, false>{args...});
}

static cudaError_t launch_classes(bool merged, int Lh, int Ll, const semkv_cache &c, const DecParams &p, int grid,
                                  cudaStream_t st) {
  return dispatch_cache<LaunchF>(merged, Lh, Ll, c, std::cref(p), grid, st);
}

static int class_occupancy(bool merged, int Lh, int Ll, const semkv_cache &c) {
  return dispatch_cache<OccF>(merged, Lh, Ll, c, c.H_q / c.H);
}

// code words of one slab of a class
static int64_t slab_words(const semkv_cache &c, int L, int cap) {
  if (c.layout == SEMKV_LAYOUT_PAGES) return ((int64_t)cap * pages_row_bits(L) + 127) / 128 * 4;
  return (int64_t)cap * words_per_row(L);
}

// Splits per slab of each class (the host knows only capacities).  CTAs of
// one launch run in rounds of R = resident CTAs per SM x SMs; the model is
//   time ~ rounds * (tiles of the longest CTA + a per-CTA overhead of 2 tiles)
// with the splits of the two classes in proportion to their capacities, and
// the smallest split count within 0.5% of the best is taken.  On the 32-layer
// prefill cache (256 slabs, 1032 16-token tiles per pool, 4 CTAs per SM) this
// gives 8 splits per pool, 4096 CTAs in 7 rounds of 592.
static void pool_splits(const semkv_cache &c, int n_layers, int *Sh, int *Sl) {
  const bool merged = has_merged(c.L_high, c.L_low);
  int occ;
  if (merged) {
    occ = class_occupancy(true, c.L_high, c.L_low, c);
  } else {
    const int oh = class_occupancy(false, c.L_high, c.L_high, c);
    const int ol = class_occupancy(false, c.L_low, c.L_low, c);
    occ = oh < ol ? oh : ol;
  }
  const int64_t R = (int64_t)device_sm_count() * occ;
  const int64_t slabs = (int64_t)c.B * n_layers * c.H;
  const int64_t th = (c.cap_high + 15) / 16, tl = (c.cap_low + 15) / 16;
  const int64_t tmax = th > tl ? th : tl, tmin = th > tl ? tl : th;
  double best = 1e300;
  *Sh = *Sl = 1;
  for (int S = 1; S <= 64; ++S) {
    if (S > 1 && tmax / S < 16) break;                   // keep >= 16 tiles (4 per warp) per CTA
    int s_small = tmax > 0 ? (int)((S * tmin + tmax / 2) / tmax) : 1;
    if (s_small < 1) s_small = 1;
    const int sh = th >= tl ? S : s_small, sl = th >= tl ? s_small : S;
    const double wh = (double)th / sh + 2.0, wl = (double)tl / sl + 2.0;
    double est;
    if (merged) {
      const int64_t rounds = (slabs * (sh + sl) + R - 1) / R;
      est = rounds * (wh > wl ? wh : wl);
    } else {
      est = ((slabs * sh + R - 1) / R) * wh + ((slabs * sl + R - 1) / R) * wl;
    }
    if (est < best * 0.995) {
      best = est;
      *Sh = sh;
      *Sl = sl;
    }
  }
}

size_t decode_ws_bytes(const semkv_cache &c, int n_layers) {
  int Sh, Sl;
  pool_splits(c, n_layers, &Sh, &Sl);
  const int64_t slabs = (int64_t)c.B * n_layers * c.H;
  const int G = c.H_q / c.H;
  const size_t parts = (size_t)(slabs * (Sh + Sl + 1) * G * PART_STRIDE * sizeof(float));
  return parts + 2 * (size_t)c.B * c.H_q * c.block * sizeof(float);
}

cudaError_t launch_decode(const semkv_cache &c, int layer0, int n_layers, int score_layer, const uint16_t *q,
                          uint16_t *out, float sm_scale, void *ws, uint32_t *status, cudaStream_t st) {
  int Sh, Sl;
  pool_splits(c, n_layers, &Sh, &Sl);
  const int NU = Sh + Sl + 1;
  const int slabs = c.B * n_layers * c.H;
  const int G = c.H_q / c.H;
  DecParams p;
  p.slabs = slabs;
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
  p.rot = c.rotate;
  p.wait0 = first_wait_polls(kWaitLimit);
  const PoolArgs high = {c.k_high, c.v_high, reinterpret_cast<const float2 *>(c.k_high_meta),
                         reinterpret_cast<const float2 *>(c.v_high_meta), c.n_high, c.cap_high, Sh, 0,
                         slab_words(c, c.L_high, c.cap_high)};
  const PoolArgs low = {c.k_low, c.v_low, reinterpret_cast<const float2 *>(c.k_low_meta),
                        reinterpret_cast<const float2 *>(c.v_low_meta), c.n_low, c.cap_low, Sl, Sh,
                        slab_words(c, c.L_low, c.cap_low)};
  cudaError_t e;
  bool pool_launched = false;          // the last launch so far is a pool kernel
  if (has_merged(c.L_high, c.L_low)) {
    p.pool[0] = high;
    p.pool[1] = low;
    e = launch_classes(true, c.L_high, c.L_low, c, p, slabs * (Sh + Sl), st);
    if (e != cudaSuccess) return e;
    pool_launched = slabs * (Sh + Sl) > 0;
  } else {
    for (int cls = 0; cls < 2; ++cls) {
      p.pool[0] = cls ? low : high;
      p.pool[1] = p.pool[0];
      p.pool[1].S = 0;
      const int L = cls ? c.L_low : c.L_high;
      e = launch_classes(false, L, L, c, p, slabs * p.pool[0].S, st);
      if (e != cudaSuccess) return e;
      pool_launched = pool_launched || slabs * p.pool[0].S > 0;
    }
  }
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
  if (pool_launched) {
    // programmatic dependent launch right behind a pool kernel: the FP16-block
    // kernel reads only the block, q and its own outputs, so it may overlap the
    // pool kernel; it waits for that kernel before it exits.  (Behind any
    // other launch it must not start early: the block may still be written.)
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(slabs);
    cfg.blockDim = dim3(128);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = st;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, decode_buffer_kernel, bp);
  } else {
    decode_buffer_kernel<<<slabs, 128, 0, st>>>(bp);
    e = cudaGetLastError();
  }
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
