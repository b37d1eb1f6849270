// internal.h -- host-side launchers shared by the C-ABI layer (not exported).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/semkv.h"

namespace semkv {

// Poll bound of the first wait of each warp's bulk-copy ring: `dflt` unless a
// test lowered it with semkv_set_first_copy_wait_polls.
int first_wait_polls(int dflt);

// Per-device host caches (devinfo.cu): SMs of the current device; set a
// kernel's dynamic shared-memory limit (and the max-shared carveout) once per
// device; its resident CTAs per SM for a launch shape, queried once.
int device_sm_count();
cudaError_t prepare_kernel(const void *fn, int smem_bytes);
cudaError_t kernel_occupancy(const void *fn, int threads, int smem_bytes, int *ctas_per_sm);
// A tiled TMA descriptor over an fp16 tensor: dims fastest first, strides in
// bytes of dims 1..rank-1, the box, and whether the box lands 128-byte
// swizzled (the tensor cores' K-major operand layout).  Out-of-range elements
// of a box read as zeros.
cudaError_t encode_tensor_map_f16(CUtensorMap *map, const void *base, int rank, const uint64_t *dims,
                                  const uint64_t *strides_bytes, const uint32_t *box, bool swizzle128);

// Slot of each token within its class and the high count per sequence, then
// the per-sequence counts advanced (clamped to the capacities).
//   slot int32 [B][T_max], cnt_high int32 [B].
cudaError_t launch_reciprocal_check(uint32_t e_lo, uint32_t e_hi, unsigned long long *mismatches, cudaStream_t st);
cudaError_t launch_slot_scan(const uint8_t *mask, int64_t mask_bstride, const int32_t *seq_len,
                             int len_const, int B, int T_max, int32_t *n_high, int32_t *n_low, int cap_high,
                             int cap_low, int32_t *slot, int32_t *cnt_high, uint32_t *status, cudaStream_t st);

struct QuantLaunch {
  const uint16_t *k, *v;            // [B][Lyr][H][T_stride][128]
  int B, Lyr, H, T_stride;
  const int32_t *seq_len;           // NULL -> len_const
  int len_const;
  const uint8_t *mask;
  int64_t mask_bstride;
  const int32_t *slot;              // [B][T_stride]
  int32_t *n_high, *n_low;          // device counts (bases before, advanced after)
  uint32_t *k_high, *v_high, *k_low, *v_low;
  float *k_high_meta, *v_high_meta, *k_low_meta, *v_low_meta;
  int cap_high, cap_low, L_high, L_low;
  int rotate;                       // 1: Hadamard-rotate each row before quantizing
  int layout;                       // SEMKV_LAYOUT_WORDS or SEMKV_LAYOUT_PAGES
  uint32_t *status;
};
cudaError_t launch_quantize(const QuantLaunch &q, cudaStream_t st);

cudaError_t launch_select(const float *score, int64_t score_bstride, const int32_t *seq_len,
                          int len_const, int B, int T_max, int r_ppm, uint8_t *mask,
                          int64_t mask_bstride, uint32_t *status, cudaStream_t st);

cudaError_t launch_score_key_l2(const uint16_t *k, int64_t k_bstride, const int32_t *seq_len,
                                int B, int T_max, int H, float *score, uint32_t *status,
                                cudaStream_t st);

size_t attn_mass_ws_bytes(int B, int T_max, int H, int H_q, int w);
cudaError_t launch_score_attn_mass(const uint16_t *k, int64_t k_bstride, const uint16_t *q_win,
                                   const int32_t *seq_len, int B, int T_max, int H, int H_q,
                                   int w, float *score, void *ws, uint32_t *status,
                                   cudaStream_t st);

cudaError_t launch_buffer_append(const semkv_cache &c, const uint16_t *k_new,
                                 const uint16_t *v_new, const float *score_new, int n_total,
                                 int i0, int take, cudaStream_t st);

size_t decode_ws_bytes(const semkv_cache &c, int n_layers);
cudaError_t launch_decode(const semkv_cache &c, int layer0, int n_layers, int score_layer, const uint16_t *q,
                          uint16_t *out, float sm_scale, void *ws, uint32_t *status, cudaStream_t st);

}  // namespace semkv
