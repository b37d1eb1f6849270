/*
 * semkv.h -- C ABI of the SemKV mixed-precision KV-cache hot path (libsemkv.so).
 *
 * The method: "SemKV: Semantic Mixed-Precision KV Cache Quantization Guided by
 * the Quality Cliff for Long-Context LLM Inference" (D. Lee, D.-H. Kim,
 * J.-H. Kim).  Every prompt token is scored by one model-internal indicator
 * (Fig. 2), tokens are ranked within the prompt and the top r get the high
 * level count, the rest the adjacent low one (Fig. 4); the per-token choice is
 * broadcast over every layer and KV head, for K and V alike (Fig. 5); each row
 * of head_dim values is affine-quantized (Table 2, Table 6: two scalars per
 * row); generated tokens wait in an FP16 block that is ranked and quantized as
 * a whole when it fills (Fig. 6); decoding attends over the mixed cache
 * (Fig. 5).
 *
 * Conventions for every call
 *   - Tensor pointers are DEVICE pointers owned by the caller.  The library
 *     never allocates, frees or synchronizes; every call only enqueues work on
 *     `stream` (a cudaStream_t passed as void*, NULL = legacy default stream).
 *   - fp16 tensors are IEEE binary16 bit patterns (uint16_t), fp32 is IEEE
 *     binary32.  KV tensors are laid out [B][n_layers][H][T][D] (row = D values).
 *   - Every tensor pointer must be 16-byte aligned.
 *   - Arguments are validated on the host before anything is launched; a bad
 *     argument returns an error and enqueues nothing.
 *   - Conditions only the GPU can see (a non-finite input, a pool that would
 *     overflow, a length beyond T_max) are OR-ed as SEMKV_FLAG_* bits into the
 *     caller's device word `status` (may be NULL for calls that take none);
 *     the caller reads it after synchronizing.  Kernels never trap, and every
 *     wait for an asynchronous copy or tensor-core result is bounded (a wait
 *     that gives up sets SEMKV_FLAG_TIMEOUT).
 *   - D (head_dim) must be 128; level counts L must be in [2, 16].
 */
#ifndef SEMKV_H
#define SEMKV_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum semkv_status {
  SEMKV_OK = 0,
  SEMKV_ERR_INVALID_ARG = 1,   /* null/misaligned pointer, bad size or shape    */
  SEMKV_ERR_UNSUPPORTED = 2,   /* D != 128, L outside [2,16], H_q/H > 8 (> 4 with rotate), a level the layout lacks */
  SEMKV_ERR_WORKSPACE = 3,     /* workspace smaller than the *_workspace_size    */
  SEMKV_ERR_CAPACITY = 4,      /* an append would overflow the FP16 block        */
  SEMKV_ERR_CUDA = 5           /* a launch failed (cudaGetLastError)             */
} semkv_status;

/* device status bits (OR-ed into *status) */
#define SEMKV_FLAG_NONFINITE 0x1u  /* a quantized row or a score held NaN/Inf; that row's output is unspecified */
#define SEMKV_FLAG_CAPACITY  0x2u  /* a row did not fit its pool; it was not written                           */
#define SEMKV_FLAG_SEQLEN    0x4u  /* seq_len[b] outside [0, T_max]; the sequence was skipped                  */
#define SEMKV_FLAG_TIMEOUT   0x8u  /* a bounded wait for an asynchronous copy gave up; that output is unspecified */

typedef enum semkv_score_kind {
  SEMKV_SCORE_ATTN_MASS = 0,   /* attention mass from the last w query rows (Table 1 "Attn."; Fig. 10) */
  SEMKV_SCORE_KEY_L2 = 1       /* key L2 norm over the scoring layer's KV heads (Table 3 "key-norm")   */
} semkv_score_kind;

#define SEMKV_FLUSH 0x1u       /* semkv_append_block: quantize the partial FP16 block (end of turn, Fig. 6) */

/* Pool storage layouts (semkv_cache.layout) */
#define SEMKV_LAYOUT_WORDS 0   /* floor(32/log2 L) base-L digits per 32-bit word, fp32 (min, scale) */
#define SEMKV_LAYOUT_PAGES 1   /* groups of <= 5 digits in whole bits, rows back to back in a bit
                                  stream, fp16 (min, scale): the layout of Table 3/5/6, Fig. 11 */

/*
 * The mixed cache.  A host-side struct of sizes and device pointers; the pools
 * are caller-allocated device memory of the sizes given below.  Pool layout
 * per class c in {high, low}, with W_c = semkv_words_per_row(L_c, 128):
 *   codes  k_c, v_c : uint32 [B][n_layers][H][cap_c][W_c]   mixed-radix words
 *   meta   k_c_meta, v_c_meta : float [B][n_layers][H][cap_c][2] = (min, scale)
 * Within a (sequence, layer, head) a class keeps its tokens in token order:
 * slot = number of same-class tokens quantized before it.  n_high[b] and
 * n_low[b] (device int32) count the slots in use; they are the same for every
 * layer and head because the token-wise choice is broadcast (Fig. 5).
 * The FP16 block (Fig. 6): buf_k, buf_v fp16 [B][n_layers][H][block][128],
 * buf_score fp32 [B][block]; buf_len (HOST field) tokens of it are in use,
 * the same number for every sequence.
 * rotate = 1 (SemKV, Table 2: the quantizer applies a Hadamard rotation):
 * every K and V row x (fp16) is widened to fp32 and replaced by x' = H x, H
 * the unnormalised 128-point Hadamard matrix computed by the fast transform
 * with stages h = 1, 2, ..., 64 (one fp32 rounding per butterfly); x' is what
 * is quantized and stored, (min, scale) are x''s.  Decode rotates q the same
 * way and returns H o' / 128, so outputs are in the tokens' own basis.  The
 * FP16 block is stored unrotated.  Needs H_q/H <= 4 (UNSUPPORTED otherwise).
 *
 * layout = SEMKV_LAYOUT_PAGES (SemKV, Table 3, Table 5, Table 6, Fig. 11: the
 * printed effective bits "include packing and per-row metadata" -- groups of
 * at most five base-L digits in whole bits and two 16-bit scalars per row):
 *   - a row's D codes form groups of g digits (the last group holds D mod g),
 *     g and the group's bit width b chosen as semkv_row_bits documents; group
 *     value = sum_j code[j] L^j (digit 0 least significant), least significant
 *     bit first; a row is R = semkv_row_bits(1, L) bits;
 *   - codes k_c, v_c: per (sequence, layer, head) slab one little-endian bit
 *     stream of semkv_pool_words(1, L_c, cap_c) uint32 words, row s at bits
 *     [s R, (s+1) R): rows sit back to back with no padding, so the stored
 *     bytes are the printed effective bits;
 *   - meta k_c_meta, v_c_meta: per row one 4-byte record of two IEEE fp16
 *     values (min, scale), [B][n_layers][H][cap_c], the fp32 min and scale
 *     rounded to nearest-even (the codes are those of the fp32 scalars);
 *   - levels 9, 12, 14 and 15 are UNSUPPORTED, and so is rotate = 1.
 * Quantize writes a row's boundary words with atomic bit operations, so rows
 * of one slab may be written concurrently and no zero-filling is needed.
 */
typedef struct semkv_cache {
  int32_t B, n_layers, H, H_q, D;
  int32_t L_high, L_low;
  int32_t r_ppm;                 /* high fraction r in parts per million, [0, 1e6]   */
  int32_t cap_high, cap_low;     /* slots per (sequence, layer, head); multiples of 16 */
  int32_t block;                 /* FP16 block length (128)                          */
  int32_t buf_len;               /* host: tokens in the FP16 block, 0 <= buf_len < block */
  int32_t rotate;                /* 0, or 1: Hadamard-rotated rows (Table 2), see below */
  int32_t layout;                /* SEMKV_LAYOUT_WORDS (0) or SEMKV_LAYOUT_PAGES (1), see below */
  uint32_t *k_high, *v_high, *k_low, *v_low;
  float *k_high_meta, *v_high_meta, *k_low_meta, *v_low_meta;
  int32_t *n_high, *n_low;       /* device [B] */
  uint16_t *buf_k, *buf_v;       /* device fp16 [B][n_layers][H][block][D] */
  float *buf_score;              /* device [B][block] */
} semkv_cache;

/* ---- host helpers (no GPU work) ------------------------------------------ */

/* ceil(r * n) with r = r_ppm / 1e6, exact in integers (Fig. 4: exactly the top r).
 * Returns -1 if n < 0 or r_ppm is outside [0, 1e6]. */
int64_t semkv_num_high(int64_t n, int32_t r_ppm);

/* Base-L digits per 32-bit word: the largest n with L^n <= 2^32, i.e.
 * floor(32 / log2 L) (Fig. 1: L levels carry log2 L bits).  -1 if L not in [2,16]. */
int32_t semkv_digits_per_word(int32_t L);

/* 32-bit words per row of D codes: ceil(D / digits_per_word(L)); -1 if invalid. */
int32_t semkv_words_per_row(int32_t L, int32_t D);

/* Code bits of one 128-value row in a layout: 32 * semkv_words_per_row(L, 128)
 * for SEMKV_LAYOUT_WORDS; for SEMKV_LAYOUT_PAGES, g <= 5 digits per group in b
 * bits, b the fewest bits holding L^g values and g the choice with the fewest
 * bits per digit (the largest g among equals), plus the last group's
 * 128 mod g digits in the fewest bits holding them (6 levels: 5 digits in 13
 * bits, 333 bits a row; 5 levels: 3 digits in 7 bits, 299 bits a row).
 * -1 for an invalid or unsupported (layout, L). */
int32_t semkv_row_bits(int32_t layout, int32_t L);

/* uint32 words of codes that one (sequence, layer, head) slab of a pool class
 * of capacity cap occupies: cap * words_per_row for SEMKV_LAYOUT_WORDS,
 * ceil(cap * row_bits / 128) * 4 for SEMKV_LAYOUT_PAGES.  -1 if invalid. */
int64_t semkv_pool_words(int32_t layout, int32_t L, int32_t cap);

/* Library build identification string (static storage). */
const char *semkv_version(void);

/*
 * Testing aid for the bounded waits (no counterpart on the pages).  Sets how
 * many times the FIRST wait of every warp's bulk-copy ring polls its mbarrier
 * in semkv_quantize and semkv_decode_attn launches enqueued after this call
 * (process-wide, not thread-safe).  polls < 0 restores each kernel's own bound
 * (the default).  polls = 0 makes that wait give up at once, so the launch
 * takes its timeout path: SEMKV_FLAG_TIMEOUT is set, the outputs of the warps
 * concerned are unspecified, and every copy already issued is still waited
 * for, with the default bound, before the warp exits.  No other wait is
 * affected.  Not for production use.
 */
void semkv_set_first_copy_wait_polls(int32_t polls);

/*
 * Self-check of the reciprocal the quantizer uses (no counterpart on the
 * pages).  Quantize forms a row's r = RN(1/scale) from the hardware's
 * approximate reciprocal and one Newton-Raphson step in fused multiply-adds,
 * not from an IEEE divide.  This call compares that reciprocal bit for bit with
 * the IEEE round-to-nearest reciprocal for every positive float whose exponent
 * field lies in [exp_lo, exp_hi] (2^23 values per exponent), and adds the
 * number of differences to *mismatches (device, unsigned 64-bit, caller
 * zeroed), enqueued on `stream`.  Exponent fields 1 .. 252 (b in [2^-126,
 * 2^126)) cover every scale a row can have, and there the count must be 0.
 * INVALID_ARG for exp_lo < 1, exp_hi > 254, exp_lo > exp_hi or a null pointer.
 */
semkv_status semkv_check_reciprocal(uint32_t exp_lo, uint32_t exp_hi, unsigned long long *mismatches,
                                    void *stream);

/* ---- a1: importance score (Fig. 2) ---------------------------------------- */

/* Workspace bytes semkv_score needs for these sizes (0 for KEY_L2). */
size_t semkv_score_workspace_size(int32_t kind, int32_t B, int32_t T_max, int32_t H,
                                  int32_t H_q, int32_t w);

/*
 * Per-token importance score of one scoring layer.
 *   k       fp16, sequence b's keys at k + b*k_batch_stride, laid out [H][T_max][D]
 *           (so a [B][n_layers][H][T_max][D] cache passes its layer slice with
 *           k_batch_stride = n_layers*H*T_max*D).
 *   q_win   fp16 [B][H_q][w][D]: the last w query rows of the scoring layer
 *           (ATTN_MASS only; NULL for KEY_L2).  Row i sits at position
 *           seq_len[b] - w + i and sees keys j <= that position; rows whose
 *           position is negative are skipped.  Query head h reads KV head
 *           floor(h / (H_q/H)); logits are scaled by 1/sqrt(D).
 *   seq_len int32 [B], tokens of each sequence (<= T_max).
 *   score   fp32 [B][T_max]; entries j >= seq_len[b] are written 0.
 * ATTN_MASS: s_j = sum_h sum_i softmax_j(q_hi . k_j / sqrt(D)) (fp32 tensor-core
 *   products, fp32 softmax; within 1e-4 relative of the float64 definition).
 * KEY_L2: s_j = sqrt(sum over heads and dims of k^2), in one fixed fp32 order:
 *   per head, 32 lane partials (x0^2+x1^2)+(x2^2+x3^2) over dims 4l..4l+3,
 *   an xor butterfly over 16,8,4,2,1, then heads summed in order, IEEE sqrt.
 * Errors: INVALID_ARG (null/misaligned, B,T_max,H <= 0, H_q % H, w <= 0),
 * UNSUPPORTED (D != 128, H_q/H > 8), WORKSPACE.
 */
semkv_status semkv_score(int32_t kind, const uint16_t *k, int64_t k_batch_stride,
                         const uint16_t *q_win, const int32_t *seq_len, int32_t B,
                         int32_t T_max, int32_t H, int32_t H_q, int32_t D, int32_t w,
                         float *score, void *ws, size_t ws_bytes, uint32_t *status,
                         void *stream);

/* ---- a2: per-prompt top-r selection (Fig. 2, Fig. 4) ---------------------- */

size_t semkv_select_workspace_size(int32_t B, int32_t T_max);

/*
 * mask[b][j] = 1 for the first ceil(r*seq_len[b]) tokens of sequence b in the
 * order (score descending, token index ascending), else 0; -0.0 ranks as +0.0.
 * No threshold is estimated: exactly that many tokens are high (Fig. 4), and
 * every other token is low, none is dropped (Table 1).
 *   score fp32 [B][T_max]; mask uint8 [B][T_max] (entries >= seq_len[b] set 0).
 *   seq_len int32 [B] (device), or NULL to use len_const for every sequence.
 * A NaN score sets SEMKV_FLAG_NONFINITE (the mask is then unspecified).
 */
semkv_status semkv_select(const float *score, int64_t score_batch_stride,
                          const int32_t *seq_len, int32_t len_const, int32_t B,
                          int32_t T_max, int32_t r_ppm, uint8_t *mask,
                          int64_t mask_batch_stride, void *ws, size_t ws_bytes,
                          uint32_t *status, void *stream);

/* ---- a3+a4: quantize and pack into the pools (Fig. 5; Table 2; Table 6) ---- */

size_t semkv_quantize_workspace_size(int32_t B, int32_t T_max);

/*
 * Quantize every row of K and V [B][n_layers][H][T_max][D] (fp16) with tokens
 * j < seq_len[b], row class from mask[b][j] (1 = high), and append the rows to
 * the pools after the slots already in use (n_high[b], n_low[b]), which are
 * then advanced.  With c->rotate the row x below is the rotated row H x (fp32,
 * see the cache struct).  Per row, in IEEE fp32 round-to-nearest-even:
 *   mn = min(x)+0, mx = max(x)+0, scale = (mx-mn)/(L-1),
 *   code = scale == 0 ? 0 : clamp(rint((x-mn)/scale), 0, L-1)      (exact division)
 *   word w = sum_j code[w*n+j] * L^j, n = semkv_digits_per_word(L)  (little-endian digits)
 *   meta = (mn, scale).
 * Bit-identical to the definition for all finite inputs.  Rows beyond a pool's
 * capacity are not written (SEMKV_FLAG_CAPACITY); non-finite rows set
 * SEMKV_FLAG_NONFINITE.
 */
semkv_status semkv_quantize(semkv_cache *c, const uint16_t *k, const uint16_t *v,
                            int32_t T_max, const int32_t *seq_len, const uint8_t *mask,
                            void *ws, size_t ws_bytes, uint32_t *status, void *stream);

/*
 * semkv_quantize without a caller workspace.  (The paper has no counterpart:
 * this is a library convenience.)  For callers that cannot allocate device
 * memory when they call in -- for example an inference engine that has handed
 * all device memory to its own pool allocator, or a plugin host that forbids
 * cudaMalloc on its hot path -- and so have no workspace to pass.  It computes
 * exactly what semkv_quantize computes, with the workspace taken from a fixed
 * array that the library keeps in device memory:
 *   - the array holds SEMKV_NOALLOC_SCRATCH_BYTES on every GPU that loads the
 *     library, until the process exits;
 *   - sizes needing more (semkv_quantize_workspace_size(c->B, T_max) larger
 *     than that, i.e. B*T_max above about one million tokens) are rejected
 *     with SEMKV_ERR_WORKSPACE before anything is enqueued;
 *   - the first call on a device looks up the array's device address on the
 *     host (once per device, with that device current); make that first call
 *     before any stream capture;
 *   - every call on a device uses the same array, which keeps the last call's
 *     contents: calls whose work overlaps on the GPU (other streams, other
 *     threads) race, so serialize them;
 *   - it calls no allocator: no cudaMalloc, cudaFree or allocating library;
 *   - the looked-up address is kept for the life of the process: after
 *     cudaDeviceReset (or anything else that tears down the device's primary
 *     context) it is stale, so do not call this entry point on that device
 *     again in the same process.
 * Arguments, results, flags and errors are otherwise those of semkv_quantize.
 */
#define SEMKV_NOALLOC_SCRATCH_BYTES (4u << 20)
semkv_status semkv_quantize_noalloc(semkv_cache *c, const uint16_t *k, const uint16_t *v,
                                    int32_t T_max, const int32_t *seq_len, const uint8_t *mask,
                                    uint32_t *status, void *stream);

/* ---- a5: generation-time block-exact path (Fig. 6) ------------------------- */

size_t semkv_append_workspace_size(const semkv_cache *c);

/*
 * Append n new tokens per sequence: k_new, v_new fp16 [B][n_layers][H][n][D],
 * score_new fp32 [B][n] (any indicator; only its ranking within a block is used).
 * Tokens go to the FP16 block; each time it holds `block` tokens, its own
 * scores are ranked, the top ceil(r*block) get L_high, the block is quantized
 * onto the pools exactly as semkv_quantize does, and emptied.  A full block is
 * never left in FP16.  flags & SEMKV_FLUSH (end of a generation turn): after
 * appending, a partial block of m > 0 tokens is quantized the same way with
 * ceil(r*m) high tokens.  Updates c->buf_len on the host.  n may be 0.
 */
semkv_status semkv_append_block(semkv_cache *c, const uint16_t *k_new, const uint16_t *v_new,
                                const float *score_new, int32_t n, uint32_t flags, void *ws,
                                size_t ws_bytes, uint32_t *status, void *stream);

/* ---- a6: decode attention over the mixed cache (Fig. 5) -------------------- */

size_t semkv_decode_workspace_size(const semkv_cache *c, int32_t n_layers);

/*
 * One decode query per query head for layers [layer0, layer0+n_layers):
 *   q   fp16 [B][n_layers][H_q][D];  out fp16 [B][n_layers][H_q][D].
 * out_h = sum_j softmax_j(sm_scale * q_h . k_j) v_j over every cached token of
 * KV head floor(h/(H_q/H)): the high pool, the low pool (dequantized as
 * mn + code*scale) and the buf_len FP16 tokens.  A sequence with no cached
 * token gets out = 0.  fp32 softmax, fp16 tensor-core products: within 1e-3
 * relative L2 of the float64 definition.
 */
semkv_status semkv_decode_attn(const semkv_cache *c, int32_t layer0, int32_t n_layers,
                               const uint16_t *q, uint16_t *out, float sm_scale, void *ws,
                               size_t ws_bytes, uint32_t *status, void *stream);

/*
 * semkv_decode_attn plus the attention-mass indicator for generated tokens
 * (SemKV, Fig. 6: the scores of generated tokens are accumulated until their
 * block is ranked; Fig. 12: attention-based indicators).  At the scoring layer
 * score_layer (layer0 <= score_layer < layer0 + n_layers), every FP16-block
 * token t < buf_len receives, in buf_score[b][t], the sum over the H_q query
 * heads of its softmax probability in this step, normalised over every cached
 * token exactly as the output is.  Heads are added in index order, so the
 * result is deterministic.  The block's ranking in semkv_append_block then
 * uses these accumulated scores (plus whatever score_new the caller gave).
 * Same workspace as semkv_decode_attn.  Errors: as semkv_decode_attn, plus
 * INVALID_ARG for score_layer outside the decoded layers or a null buf_score.
 */
semkv_status semkv_decode_attn_acc(const semkv_cache *c, int32_t layer0, int32_t n_layers,
                                   int32_t score_layer, const uint16_t *q, uint16_t *out, float sm_scale,
                                   void *ws, size_t ws_bytes, uint32_t *status, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* SEMKV_H */
