// api.cu -- the C ABI of libsemkv: argument checks, workspace carving, launches.
// Everything here runs on the host; every GPU step is one of the kernels in
// the other files of this directory.
#include <cuda_runtime.h>
#include <nvtx3/nvToolsExt.h>
#include <stdint.h>

#include "../../include/semkv.h"
#include "common.cuh"
#include "internal.h"

using namespace semkv;

namespace semkv {
static int g_first_wait_polls = -1;     // < 0: each kernel's own bound
int first_wait_polls(int dflt) { return g_first_wait_polls < 0 ? dflt : g_first_wait_polls; }
}  // namespace semkv

namespace {

// An NVTX range around each call that enqueues GPU work, named after the call,
// so a timeline tool shows which C-ABI call launched which kernels (a no-op
// when no tool is attached).
struct NvtxRange {
  explicit NvtxRange(const char *name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
};

inline bool al16(const void *p) { return p != nullptr && (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline size_t up256(size_t x) { return (x + 255) & ~size_t(255); }
inline cudaStream_t S(void *s) { return reinterpret_cast<cudaStream_t>(s); }
inline semkv_status cuda_status(cudaError_t e) { return e == cudaSuccess ? SEMKV_OK : SEMKV_ERR_CUDA; }

semkv_status check_cache(const semkv_cache *c) {
  if (!c) return SEMKV_ERR_INVALID_ARG;
  if (c->B <= 0 || c->n_layers <= 0 || c->H <= 0 || c->H_q <= 0) return SEMKV_ERR_INVALID_ARG;
  if (c->H_q % c->H != 0) return SEMKV_ERR_INVALID_ARG;
  if (c->D != kD || c->H_q / c->H > 8) return SEMKV_ERR_UNSUPPORTED;
  if (c->L_high < 2 || c->L_high > kMaxL || c->L_low < 2 || c->L_low > kMaxL) return SEMKV_ERR_UNSUPPORTED;
  if (c->r_ppm < 0 || c->r_ppm > 1000000) return SEMKV_ERR_INVALID_ARG;
  if (c->cap_high < 0 || c->cap_low < 0 || (c->cap_high % 16) || (c->cap_low % 16)) return SEMKV_ERR_INVALID_ARG;
  if (c->cap_high >= (1 << 30) || c->cap_low >= (1 << 30)) return SEMKV_ERR_INVALID_ARG;   // pool positions fit 30 bits
  if (c->block < 1 || c->block > 128) return SEMKV_ERR_INVALID_ARG;
  if (c->rotate != 0 && c->rotate != 1) return SEMKV_ERR_INVALID_ARG;
  if (c->rotate && c->H_q / c->H > 4) return SEMKV_ERR_UNSUPPORTED;
  if (c->layout != SEMKV_LAYOUT_WORDS && c->layout != SEMKV_LAYOUT_PAGES) return SEMKV_ERR_INVALID_ARG;
  if (c->layout == SEMKV_LAYOUT_PAGES &&
      (c->rotate || !pages_supported(c->L_high) || !pages_supported(c->L_low)))
    return SEMKV_ERR_UNSUPPORTED;
  if (c->buf_len < 0 || c->buf_len >= c->block) return SEMKV_ERR_INVALID_ARG;
  const void *ptrs[] = {c->k_high, c->v_high, c->k_low, c->v_low, c->k_high_meta, c->v_high_meta,
                        c->k_low_meta, c->v_low_meta, c->n_high, c->n_low, c->buf_k, c->buf_v,
                        c->buf_score};
  for (const void *p : ptrs)
    if (!al16(p)) return SEMKV_ERR_INVALID_ARG;
  // every slab, row and tile offset stays inside 31-bit element counts
  const int64_t slabs = (int64_t)c->B * c->n_layers * c->H;
  if (slabs * (int64_t)(c->cap_high > c->cap_low ? c->cap_high : c->cap_low) >= (1ll << 31))
    return SEMKV_ERR_INVALID_ARG;
  return SEMKV_OK;
}

size_t quant_ws(int B, int T) { return up256((size_t)B * T * 4) + up256((size_t)B * 4); }

// quantize rows of src [B][Lyr][H][T_stride][D] (tokens < len) onto the pools
semkv_status quantize_rows(semkv_cache *c, const uint16_t *k, const uint16_t *v, int T_stride,
                           const int32_t *seq_len, int len_const, const uint8_t *mask,
                           int64_t mask_bstride, void *ws, uint32_t *status, cudaStream_t st) {
  int32_t *slot = reinterpret_cast<int32_t *>(ws);
  int32_t *cnt = reinterpret_cast<int32_t *>(reinterpret_cast<char *>(ws) + up256((size_t)c->B * T_stride * 4));
  cudaError_t e = launch_slot_scan(mask, mask_bstride, seq_len, len_const, c->B, T_stride, c->n_high, c->n_low,
                                   c->cap_high, c->cap_low, slot, cnt, status, st);
  if (e != cudaSuccess) return SEMKV_ERR_CUDA;
  QuantLaunch q;
  q.k = k;
  q.v = v;
  q.B = c->B;
  q.Lyr = c->n_layers;
  q.H = c->H;
  q.T_stride = T_stride;
  q.seq_len = seq_len;
  q.len_const = len_const;
  q.mask = mask;
  q.mask_bstride = mask_bstride;
  q.slot = slot;
  q.n_high = c->n_high;
  q.n_low = c->n_low;
  q.k_high = c->k_high;
  q.v_high = c->v_high;
  q.k_low = c->k_low;
  q.v_low = c->v_low;
  q.k_high_meta = c->k_high_meta;
  q.v_high_meta = c->v_high_meta;
  q.k_low_meta = c->k_low_meta;
  q.v_low_meta = c->v_low_meta;
  q.cap_high = c->cap_high;
  q.cap_low = c->cap_low;
  q.L_high = c->L_high;
  q.rotate = c->rotate;
  q.layout = c->layout;
  q.L_low = c->L_low;
  q.status = status;
  return cuda_status(launch_quantize(q, st));
}

size_t append_ws(const semkv_cache *c) {
  return up256((size_t)c->B * c->block) + quant_ws(c->B, c->block);
}

// rank and quantize the buf_len tokens of the FP16 block, then empty it
semkv_status flush_block(semkv_cache *c, void *ws, uint32_t *status, cudaStream_t st) {
  const int n = c->buf_len;
  if (n == 0) return SEMKV_OK;
  uint8_t *mask = reinterpret_cast<uint8_t *>(ws);
  void *qws = reinterpret_cast<char *>(ws) + up256((size_t)c->B * c->block);
  cudaError_t e = launch_select(c->buf_score, c->block, nullptr, n, c->B, c->block, c->r_ppm, mask,
                                c->block, status, st);
  if (e != cudaSuccess) return SEMKV_ERR_CUDA;
  semkv_status s = quantize_rows(c, c->buf_k, c->buf_v, c->block, nullptr, n, mask, c->block, qws,
                                 status, st);
  if (s != SEMKV_OK) return s;
  c->buf_len = 0;
  return SEMKV_OK;
}

}  // namespace

extern "C" {

int64_t semkv_num_high(int64_t n, int32_t r_ppm) {
  if (n < 0 || r_ppm < 0 || r_ppm > 1000000) return -1;
  return ((int64_t)r_ppm * n + 999999) / 1000000;
}

int32_t semkv_digits_per_word(int32_t L) {
  if (L < 2 || L > kMaxL) return -1;
  return digits_per_word(L);
}

int32_t semkv_words_per_row(int32_t L, int32_t D) {
  if (L < 2 || L > kMaxL || D <= 0) return -1;
  const int n = digits_per_word(L);
  return (D + n - 1) / n;
}

int32_t semkv_row_bits(int32_t layout, int32_t L) {
  if (L < 2 || L > kMaxL) return -1;
  if (layout == SEMKV_LAYOUT_WORDS) return 32 * words_per_row(L);
  if (layout == SEMKV_LAYOUT_PAGES) return pages_supported(L) ? pages_row_bits(L) : -1;
  return -1;
}

int64_t semkv_pool_words(int32_t layout, int32_t L, int32_t cap) {
  const int32_t R = semkv_row_bits(layout, L);
  if (R < 0 || cap < 0) return -1;
  if (layout == SEMKV_LAYOUT_WORDS) return (int64_t)cap * words_per_row(L);
  return ((int64_t)cap * R + 127) / 128 * 4;
}

const char *semkv_version(void) { return "semkv-b200 0.3 (sm_100a)"; }

void semkv_set_first_copy_wait_polls(int32_t polls) { g_first_wait_polls = polls < 0 ? -1 : polls; }

semkv_status semkv_check_reciprocal(uint32_t exp_lo, uint32_t exp_hi, unsigned long long *mismatches, void *stream) {
  if (exp_lo < 1 || exp_hi > 254 || exp_lo > exp_hi || mismatches == nullptr) return SEMKV_ERR_INVALID_ARG;
  return cuda_status(launch_reciprocal_check(exp_lo, exp_hi, mismatches, S(stream)));
}

size_t semkv_score_workspace_size(int32_t kind, int32_t B, int32_t T_max, int32_t H, int32_t H_q,
                                  int32_t w) {
  if (kind != SEMKV_SCORE_ATTN_MASS) return 0;
  if (B <= 0 || T_max <= 0 || H <= 0 || H_q <= 0 || w <= 0) return 0;
  return attn_mass_ws_bytes(B, T_max, H, H_q, w);
}

semkv_status semkv_score(int32_t kind, const uint16_t *k, int64_t k_batch_stride,
                         const uint16_t *q_win, const int32_t *seq_len, int32_t B, int32_t T_max,
                         int32_t H, int32_t H_q, int32_t D, int32_t w, float *score, void *ws,
                         size_t ws_bytes, uint32_t *status, void *stream) {
  NvtxRange nvtx_range("semkv_score");
  if (kind != SEMKV_SCORE_ATTN_MASS && kind != SEMKV_SCORE_KEY_L2) return SEMKV_ERR_INVALID_ARG;
  if (B <= 0 || T_max <= 0 || H <= 0) return SEMKV_ERR_INVALID_ARG;
  if (D != kD) return SEMKV_ERR_UNSUPPORTED;
  if (!al16(k) || !al16(score) || !al16(seq_len)) return SEMKV_ERR_INVALID_ARG;
  if (k_batch_stride < (int64_t)H * T_max * D || (k_batch_stride % 8)) return SEMKV_ERR_INVALID_ARG;
  if ((int64_t)B * T_max >= (1ll << 31)) return SEMKV_ERR_INVALID_ARG;
  if (kind == SEMKV_SCORE_KEY_L2)
    return cuda_status(launch_score_key_l2(k, k_batch_stride, seq_len, B, T_max, H, score, status, S(stream)));
  if (H_q <= 0 || H_q % H || w <= 0 || !al16(q_win)) return SEMKV_ERR_INVALID_ARG;
  if (H_q / H > 8) return SEMKV_ERR_UNSUPPORTED;
  if (!al16(ws) || ws_bytes < attn_mass_ws_bytes(B, T_max, H, H_q, w)) return SEMKV_ERR_WORKSPACE;
  return cuda_status(launch_score_attn_mass(k, k_batch_stride, q_win, seq_len, B, T_max, H, H_q, w,
                                            score, ws, status, S(stream)));
}

size_t semkv_select_workspace_size(int32_t B, int32_t T_max) {
  (void)B;
  (void)T_max;
  return 0;
}

semkv_status semkv_select(const float *score, int64_t score_batch_stride, const int32_t *seq_len,
                          int32_t len_const, int32_t B, int32_t T_max, int32_t r_ppm, uint8_t *mask,
                          int64_t mask_batch_stride, void *ws, size_t ws_bytes, uint32_t *status,
                          void *stream) {
  NvtxRange nvtx_range("semkv_select");
  (void)ws;
  (void)ws_bytes;
  if (B <= 0 || T_max <= 0 || r_ppm < 0 || r_ppm > 1000000) return SEMKV_ERR_INVALID_ARG;
  if (!al16(score) || !al16(mask)) return SEMKV_ERR_INVALID_ARG;
  if (seq_len == nullptr && (len_const < 0 || len_const > T_max)) return SEMKV_ERR_INVALID_ARG;
  if (seq_len != nullptr && !al16(seq_len)) return SEMKV_ERR_INVALID_ARG;
  if (score_batch_stride < T_max || mask_batch_stride < T_max) return SEMKV_ERR_INVALID_ARG;
  return cuda_status(launch_select(score, score_batch_stride, seq_len, len_const, B, T_max, r_ppm, mask,
                                   mask_batch_stride, status, S(stream)));
}

size_t semkv_quantize_workspace_size(int32_t B, int32_t T_max) {
  if (B <= 0 || T_max <= 0) return 0;
  return quant_ws(B, T_max);
}

semkv_status semkv_quantize(semkv_cache *c, const uint16_t *k, const uint16_t *v, int32_t T_max,
                            const int32_t *seq_len, const uint8_t *mask, void *ws, size_t ws_bytes,
                            uint32_t *status, void *stream) {
  NvtxRange nvtx_range("semkv_quantize");
  semkv_status s = check_cache(c);
  if (s != SEMKV_OK) return s;
  if (T_max <= 0 || !al16(k) || !al16(v) || !al16(seq_len) || !al16(mask)) return SEMKV_ERR_INVALID_ARG;
  if ((int64_t)c->B * c->n_layers * c->H * T_max >= (1ll << 31)) return SEMKV_ERR_INVALID_ARG;
  if (!al16(ws) || ws_bytes < quant_ws(c->B, T_max)) return SEMKV_ERR_WORKSPACE;
  return quantize_rows(c, k, v, T_max, seq_len, 0, mask, T_max, ws, status, S(stream));
}

size_t semkv_append_workspace_size(const semkv_cache *c) {
  if (check_cache(c) != SEMKV_OK) return 0;
  return append_ws(c);
}

semkv_status semkv_append_block(semkv_cache *c, const uint16_t *k_new, const uint16_t *v_new,
                                const float *score_new, int32_t n, uint32_t flags, void *ws,
                                size_t ws_bytes, uint32_t *status, void *stream) {
  NvtxRange nvtx_range("semkv_append_block");
  semkv_status s = check_cache(c);
  if (s != SEMKV_OK) return s;
  if (n < 0 || (flags & ~SEMKV_FLUSH)) return SEMKV_ERR_INVALID_ARG;
  if (n > 0 && (!al16(k_new) || !al16(v_new) || score_new == nullptr ||
                (reinterpret_cast<uintptr_t>(score_new) & 3u)))
    return SEMKV_ERR_INVALID_ARG;
  if (!al16(ws) || ws_bytes < append_ws(c)) return SEMKV_ERR_WORKSPACE;
  cudaStream_t st = S(stream);
  int i0 = 0;
  while (i0 < n) {
    const int take = (n - i0) < (c->block - c->buf_len) ? (n - i0) : (c->block - c->buf_len);
    cudaError_t e = launch_buffer_append(*c, k_new, v_new, score_new, n, i0, take, st);
    if (e != cudaSuccess) return SEMKV_ERR_CUDA;
    c->buf_len += take;
    i0 += take;
    if (c->buf_len == c->block) {
      s = flush_block(c, ws, status, st);
      if (s != SEMKV_OK) return s;
    }
  }
  if ((flags & SEMKV_FLUSH) && c->buf_len > 0) return flush_block(c, ws, status, st);
  return SEMKV_OK;
}

size_t semkv_decode_workspace_size(const semkv_cache *c, int32_t n_layers) {
  if (check_cache(c) != SEMKV_OK || n_layers <= 0) return 0;
  return decode_ws_bytes(*c, n_layers);
}

static semkv_status decode_checked(const semkv_cache *c, int32_t layer0, int32_t n_layers, int32_t score_layer,
                                   const uint16_t *q, uint16_t *out, float sm_scale, void *ws,
                                   size_t ws_bytes, uint32_t *status, void *stream) {
  semkv_status s = check_cache(c);
  if (s != SEMKV_OK) return s;
  if (layer0 < 0 || n_layers <= 0 || layer0 + n_layers > c->n_layers) return SEMKV_ERR_INVALID_ARG;
  if (!al16(q) || !al16(out)) return SEMKV_ERR_INVALID_ARG;
  if (!(sm_scale > 0.0f) || sm_scale != sm_scale) return SEMKV_ERR_INVALID_ARG;
  if (!al16(ws) || ws_bytes < decode_ws_bytes(*c, n_layers)) return SEMKV_ERR_WORKSPACE;
  return cuda_status(launch_decode(*c, layer0, n_layers, score_layer, q, out, sm_scale, ws, status, S(stream)));
}

semkv_status semkv_decode_attn(const semkv_cache *c, int32_t layer0, int32_t n_layers,
                               const uint16_t *q, uint16_t *out, float sm_scale, void *ws,
                               size_t ws_bytes, uint32_t *status, void *stream) {
  NvtxRange nvtx_range("semkv_decode_attn");
  return decode_checked(c, layer0, n_layers, -1, q, out, sm_scale, ws, ws_bytes, status, stream);
}

semkv_status semkv_decode_attn_acc(const semkv_cache *c, int32_t layer0, int32_t n_layers,
                                   int32_t score_layer, const uint16_t *q, uint16_t *out, float sm_scale,
                                   void *ws, size_t ws_bytes, uint32_t *status, void *stream) {
  NvtxRange nvtx_range("semkv_decode_attn_acc");
  if (c && (score_layer < layer0 || score_layer >= layer0 + n_layers)) return SEMKV_ERR_INVALID_ARG;
  if (c && c->buf_score == nullptr) return SEMKV_ERR_INVALID_ARG;
  return decode_checked(c, layer0, n_layers, score_layer, q, out, sm_scale, ws, ws_bytes, status, stream);
}

}  // extern "C"
