// common.cuh -- shared device helpers of libsemkv (sm_100a).
#pragma once

#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/semkv.h"

namespace semkv {

constexpr int kD = 128;          // head_dim
constexpr int kMaxL = 16;

// ---------------------------------------------------------------------------
// Layout sizes (compile-time twins of semkv_digits_per_word / words_per_row)
// ---------------------------------------------------------------------------
__host__ __device__ constexpr int digits_per_word(int L) {
  // largest n with L^n <= 2^32
  int n = 0;
  unsigned long long p = 1;
  while (p * (unsigned long long)L <= (1ull << 32)) {
    p *= (unsigned long long)L;
    ++n;
  }
  return n;
}
__host__ __device__ constexpr int words_per_row(int L) {
  return (kD + digits_per_word(L) - 1) / digits_per_word(L);
}
__host__ __device__ constexpr unsigned long long ipow(int L, int k) {
  unsigned long long p = 1;
  for (int i = 0; i < k; ++i) p *= (unsigned long long)L;
  return p;
}

// ---------------------------------------------------------------------------
// The pages' layout (SEMKV_LAYOUT_PAGES): groups of g <= 5 digits in b bits
// ---------------------------------------------------------------------------
// fewest bits that hold n values
__host__ __device__ constexpr int bits_for(unsigned long long n) {
  int b = 0;
  while ((1ull << b) < n) ++b;
  return b;
}
// g: the group size with the fewest bits per digit, the largest among equals
__host__ __device__ constexpr int pages_g(int L) {
  int best_k = 1, best_b = bits_for(ipow(L, 1));
  for (int k = 2; k <= 5; ++k) {
    const int b = bits_for(ipow(L, k));
    if (b * best_k <= best_b * k) {        // b/k <= best_b/best_k
      best_k = k;
      best_b = b;
    }
  }
  return best_k;
}
__host__ __device__ constexpr int pages_b(int L) { return bits_for(ipow(L, pages_g(L))); }
__host__ __device__ constexpr int pages_tail(int L) { return kD % pages_g(L); }
__host__ __device__ constexpr int pages_groups(int L) { return (kD + pages_g(L) - 1) / pages_g(L); }
__host__ __device__ constexpr int pages_row_bits(int L) {
  return (kD / pages_g(L)) * pages_b(L) + (pages_tail(L) ? bits_for(ipow(L, pages_tail(L))) : 0);
}
// levels the decode reads in this layout: 2, 4 and 16 (their stream is the
// word layout's), 8 (bit fields), and the levels whose groups split into at
// most two parts that the f16 digit steps cover (3, 5, 6, 7, 10, 11, 13);
// 9, 12, 14 and 15 would need a third part or a part beyond those steps
__host__ __device__ constexpr bool pages_supported(int L) {
  return L >= 2 && L <= 16 && L != 9 && L != 12 && L != 14 && L != 15;
}

// ---------------------------------------------------------------------------
// Device status word
// ---------------------------------------------------------------------------
__device__ __forceinline__ void set_flag(uint32_t *status, uint32_t f) {
  if (status) atomicOr(status, f);
}

// ---------------------------------------------------------------------------
// Fast unsigned division by a runtime constant (Granlund-Montgomery style
// multiply-high + shift).  Valid for numerators < 2^31 and divisors >= 1.
// ---------------------------------------------------------------------------
struct FastDiv {
  uint32_t d, m, s;
  __host__ FastDiv() : d(1), m(0), s(0) {}
  __host__ explicit FastDiv(uint32_t div) : d(div) {
    // smallest s with 2^s >= d; m = floor(2^(32+s) / d) + 1 - 2^32 (the
    // classic round-up reciprocal for 31-bit numerators)
    s = 0;
    while ((1ull << s) < d) ++s;
    unsigned long long mm = ((1ull << (32 + s)) + d - 1) / d;   // ceil(2^(32+s)/d)
    m = (uint32_t)(mm - (1ull << 32));
  }
  __device__ __forceinline__ uint32_t div(uint32_t n) const {
    uint32_t t = __umulhi(n, m);
    return (t + n) >> s;    // n < 2^31 so t + n does not overflow
  }
};

// ---------------------------------------------------------------------------
// Small PTX wrappers (documented instructions only)
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void *p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void cp_async16(void *smem_dst, const void *gmem_src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(smem_u32(smem_dst)),
               "l"(gmem_src)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory");
}

__device__ __forceinline__ uint4 ld_stream_u4(const void *p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

// max that propagates NaN (PTX max.NaN, sm_80+)
__device__ __forceinline__ float fmax_nan(float a, float b) {
  float r;
  asm("max.NaN.f32 %0, %1, %2;" : "=f"(r) : "f"(a), "f"(b));
  return r;
}

// max of three with NaN propagation (sm_100 three-input form)
__device__ __forceinline__ float fmin3_nan(float a, float b, float c) {
  float r;
  asm("min.NaN.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}
__device__ __forceinline__ float fmax3_nan(float a, float b, float c) {
  float r;
  asm("max.NaN.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// packed fp32 pairs (sm_100 .f32x2 arithmetic), each lane one IEEE RN operation
__device__ __forceinline__ uint64_t f2pack(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void f2unpack(uint64_t v, float &lo, float &hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t fma2_rn(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ uint64_t mul2_rn(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ uint64_t add2_rn(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ uint64_t sub2_rn(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
// (x_lo + c, x_hi + c) in fp32 with one rounding each, x an f16 pair (the
// f16 operand converts to fp32 exactly inside the mixed-precision add)
__device__ __forceinline__ uint64_t add_h2f(uint32_t h2, float c) {
  float lo, hi;
  asm("{\n\t.reg .f16 l, h;\n\tmov.b32 {l, h}, %2;\n\t"
      "add.rn.f32.f16 %0, l, %3;\n\tadd.rn.f32.f16 %1, h, %3;\n\t}"
      : "=f"(lo), "=f"(hi) : "r"(h2), "f"(c));
  return f2pack(lo, hi);
}

// 32x32 -> 64-bit product as (lo, hi) words: one wide integer multiply-add
__device__ __forceinline__ void mul_wide(uint32_t a, uint32_t b, uint32_t &lo, uint32_t &hi) {
  asm("{\n\t.reg .u64 t;\n\tmul.wide.u32 t, %2, %3;\n\tmov.b64 {%0, %1}, t;\n\t}"
      : "=r"(lo), "=r"(hi) : "r"(a), "r"(b));
}

__device__ __forceinline__ float ex2_approx(float x) {
  float r;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
  return r;
}

// D = A(16x16, f16, row) * B(16x8, f16, col) + C, fp32 accumulate
__device__ __forceinline__ void mma_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                          uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// transpose of an 8x8 b16 matrix held one row-pair per lane
__device__ __forceinline__ uint32_t movmatrix_t(uint32_t x) {
  uint32_t r;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;\n" : "=r"(r) : "r"(x));
  return r;
}

__device__ __forceinline__ void ldmatrix_x4(uint32_t (&r)[4], const void *smem) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(smem_u32(smem)));
}

// ---- mbarrier + bulk async copies (TMA engine, non-tensor form)
__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;\n" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
}
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint64_t *bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;\n" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}
// tiled tensor load of the box at (x, y, z, w) of `map` into shared memory,
// completing on `bar` (no multicast); x * 2 bytes must be a multiple of 16
__device__ __forceinline__ void tma_load_4d(void *dst, const CUtensorMap *map, int x, int y, int z, int w,
                                            uint64_t *bar) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4, %5}], "
      "[%6];\n" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(w), "r"(smem_u32(bar))
      : "memory");
}
// global -> shared bulk copy completing on `bar` (16-byte aligned, size % 16 == 0)
__device__ __forceinline__ void bulk_g2s(void *dst, const void *src, uint32_t bytes, uint64_t *bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];\n" ::"r"(
          smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}
// bounded wait for the phase with the given parity; false after `limit` polls
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity, int limit) {
  for (int i = 0; i < limit; ++i) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}\n"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    if (ok) return true;
  }
  return false;
}

__device__ __forceinline__ uint32_t pack_half2(float lo, float hi) {
  __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<uint32_t *>(&h);
}

}  // namespace semkv
