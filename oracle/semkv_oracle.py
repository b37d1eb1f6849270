"""Plain CPU oracle for the SemKV token-wise mixed-precision KV-cache hot path.

TEST INFRASTRUCTURE, NOT PRODUCT CODE.  Only ``tests/``,
``__graft_entry__.smoke()`` and the ``cpu_baseline`` / reference legs of
``bench.py`` may import or run anything in this directory.  The product path
(``kv_cache_mixed_b200``) never calls it and shares no code with it.

Source of the method: the web page "SemKV: Semantic Mixed-Precision KV Cache
Quantization Guided by the Quality Cliff for Long-Context LLM Inference"
(D. Lee, D.-H. Kim, J.-H. Kim), of which only the figure captions and tables are
available.  Citations below read "SemKV, Fig. n" or "SemKV, Table n".

Everything is written for clarity, not speed: numpy float32 where the method's
arithmetic is fixed to IEEE single precision (the bit-exact steps), numpy float64
for the attention-based steps, Python integers for counts and packing.  Steps the
pages leave open follow the plainest reading; each such reading is named where it
is used.

Pins (tests/test_oracle_*.py) tie every function here to something other than
itself: closed forms, brute force on tiny inputs, textbook/library special
cases, and the compression figures the pages print (tests/golden/).
"""
from __future__ import annotations

import math
from fractions import Fraction
from dataclasses import dataclass, field

import numpy as np

HEAD_DIM = 128          # every backbone on the pages has head_dim 128 (SemKV, Table 2)
BLOCK = 128             # generation-time block length (block-exact path, SemKV, Fig. 6)
RPPM_ONE = 1_000_000    # the high-precision fraction r is carried as parts per million


# ---------------------------------------------------------------------------
# a0: how many tokens get the high level (SemKV, Fig. 4: top-r, no threshold)
# ---------------------------------------------------------------------------
def num_high(n: int, r_ppm: int) -> int:
    """ceil(r * n) for r = r_ppm / 1e6, in exact integer arithmetic.

    SemKV, Fig. 4: the top-r tokens receive b_high, and the allocation is made by
    the ranking alone.  "Exactly ceil(r*n)" is the plainest integer reading of a
    fraction r of n tokens; integer parts-per-million avoid any rounding of r*n.
    """
    if n < 0 or not (0 <= r_ppm <= RPPM_ONE):
        raise ValueError("n must be >= 0 and 0 <= r_ppm <= 1e6")
    return (r_ppm * n + RPPM_ONE - 1) // RPPM_ONE


# ---------------------------------------------------------------------------
# storage layout of one quantized row (fractional-level codes, SemKV, Fig. 1)
# ---------------------------------------------------------------------------
def digits_per_word(L: int) -> int:
    """Largest n with L**n <= 2**32: base-L digits that fit one 32-bit word.

    A level count L carries log2(L) bits per value (SemKV, Fig. 1 and Table 2:
    6 levels = 2.585 bits, 5 levels = 2.322 bits); n digits of base L fit a
    32-bit word exactly when L**n <= 2**32, i.e. n = floor(32 / log2 L).
    """
    if not 2 <= L <= 16:
        raise ValueError("L must be in [2, 16]")
    n = 0
    while L ** (n + 1) <= 2 ** 32:
        n += 1
    return n


def words_per_row(L: int, D: int = HEAD_DIM) -> int:
    """32-bit words holding the D codes of one row (rows never share a word)."""
    n = digits_per_word(L)
    return (D + n - 1) // n


# ---------------------------------------------------------------------------
# a1': key-norm importance indicator (SemKV, Table 3, row "SemKV key-norm")
# ---------------------------------------------------------------------------
def score_key_l2(k: np.ndarray) -> np.ndarray:
    """Per-token key L2 norm over every KV head of the scoring layer.

    k: float16 [H][T][128] (one layer of one sequence) -> float32 [T].

    The pages name the indicator only ("key-norm", SemKV Table 3).  Reading: the
    L2 norm of the token's key concatenated over all KV heads of the scoring
    layer.  The float32 summation order is fixed so that the result is one
    definite IEEE value:
      * lane partial p_l = (x[4l]^2 + x[4l+1]^2) + (x[4l+2]^2 + x[4l+3]^2),
        l = 0..31 (each square of an fp16 value is exact in fp32);
      * butterfly for s = 16, 8, 4, 2, 1: p_l <- p_l + p_(l xor s);
      * acc = 0; for g = 0..H-1: acc = acc + p_0(g);  score = sqrt(acc).
    """
    if k.dtype != np.float16 or k.ndim != 3 or k.shape[2] != HEAD_DIM:
        raise ValueError("k must be float16 [H][T][128]")
    x = k.astype(np.float32)
    sq = x * x
    p = (sq[..., 0::4] + sq[..., 1::4]) + (sq[..., 2::4] + sq[..., 3::4])  # [H][T][32]
    lanes = np.arange(32)
    for s in (16, 8, 4, 2, 1):
        p = p + p[..., lanes ^ s]
    acc = np.zeros(k.shape[1], dtype=np.float32)
    for g in range(k.shape[0]):
        acc = acc + p[g, :, 0]
    return np.sqrt(acc)


# ---------------------------------------------------------------------------
# a1: attention-based indicator (SemKV, Table 1 "Attn."; Fig. 10; Fig. 12)
# ---------------------------------------------------------------------------
def score_attn_mass(k: np.ndarray, q_win: np.ndarray, T: int) -> np.ndarray:
    """Attention mass each key receives from the last w query rows, float64.

    k: float16 [H][T_max][128]; q_win: float16 [H_q][w][128]; T = tokens of the
    sequence.  Returns float64 [T].

    s_j = sum over query heads h and window rows i of softmax_j(q_hi . k_gj / sqrt(D)),
    with g = floor(h / (H_q / H)) (consecutive query heads share a KV head).
    Readings (the pages give only the indicator's name): row i sits at position
    T - w + i and sees keys j <= T - w + i (causal); rows whose position would be
    negative (T < w) are skipped.  Scores are only ranked, never normalised
    (SemKV, Fig. 2).
    """
    H, _, D = k.shape
    H_q, w, _ = q_win.shape
    G = H_q // H
    kk = k[:, :T, :].astype(np.float64)
    s = np.zeros(T, dtype=np.float64)
    pos = T - w + np.arange(w)                      # position of each window row
    visible = np.arange(T)[None, :] <= pos[:, None]  # [w][T] causal mask
    live = pos >= 0
    for h in range(H_q):
        g = h // G
        logits = (q_win[h].astype(np.float64) @ kk[g].T) / math.sqrt(D)   # [w][T]
        logits = np.where(visible, logits, -np.inf)
        for i in range(w):
            if not live[i]:
                continue
            row = logits[i]
            e = np.exp(row - row.max())
            s += e / e.sum()
    return s


# ---------------------------------------------------------------------------
# a2: per-prompt ranking and top-r selection (SemKV, Fig. 2 and Fig. 4)
# ---------------------------------------------------------------------------
def select_mask(score: np.ndarray, n_high: int) -> np.ndarray:
    """mask[j] = 1 for the first n_high tokens in (score descending, j ascending) order.

    SemKV, Fig. 2: tokens are ranked within each prompt; Fig. 4: the top-ranked
    ones get the high precision, with no score threshold.  Ties go to the lower
    token index (reading); -0.0 is treated as +0.0.  All tokens are kept: the
    others get the low level (SemKV, Table 1, "Deletes tokens: No").
    """
    s = np.asarray(score, dtype=np.float32)
    if not np.all(np.isfinite(s)):
        raise ValueError("scores must be finite")
    T = s.shape[0]
    if not 0 <= n_high <= T:
        raise ValueError("0 <= n_high <= T required")
    s = s + np.float32(0.0)                          # -0 -> +0
    order = np.lexsort((np.arange(T), -s))           # primary: -s, then index
    mask = np.zeros(T, dtype=np.uint8)
    mask[order[:n_high]] = 1
    return mask


# ---------------------------------------------------------------------------
# a3 + a4: per-token, per-head affine quantization over head_dim
#          (SemKV, Table 2 "integer-level scalar quantization"; Table 6: affine
#          quantization stores two scalars per row)
# ---------------------------------------------------------------------------
def fwht128(x: np.ndarray) -> np.ndarray:
    """Unnormalised fast Walsh-Hadamard transform of each row of 128 values.

    SemKV, Table 2: the quantizer rotates each row with a Hadamard transform
    before its min/max.  Stages h = 1, 2, 4, ..., 64 in that order; each
    butterfly maps (a, b) at positions (j, j + h) to (a + b, a - b), one
    rounding each in the dtype of x (float32 for the quantizer, float64 for
    the reference decode).  H is symmetric and H H = 128 I, so the inverse is
    the same transform divided by 128.
    """
    y = np.array(x, copy=True)
    n = y.shape[-1]
    if n != 128:
        raise ValueError("rows must hold 128 values")
    h = 1
    while h < n:
        v = y.reshape(y.shape[:-1] + (n // (2 * h), 2, h))
        a = v[..., 0, :].copy()
        b = v[..., 1, :].copy()
        v[..., 0, :] = a + b
        v[..., 1, :] = a - b
        h *= 2
    return y


def quantize_rows(xh: np.ndarray, L: int):
    """Affine quantization of each row of D values to L levels.

    xh: float16 [..., D] (or float32 rows, e.g. rotated by fwht128) ->
    (codes uint8 [..., D], mn float32 [...], scale float32 [...], bad bool [...]).

    Per row, in IEEE float32 with round-to-nearest-even:
      mn = min(x) + 0, mx = max(x) + 0   (adding +0 turns -0 into +0)
      scale = (mx - mn) / (L - 1)
      code  = 0 if scale == 0, else clamp(rint((x - mn) / scale), 0, L - 1)
    The two stored scalars are (mn, scale).  ``bad`` marks rows holding a
    non-finite value; their codes are unspecified.
    """
    if xh.dtype not in (np.float16, np.float32):
        raise ValueError("rows must be float16 or float32")
    if xh.shape[0] == 0:
        shp = xh.shape[:-1]
        return (np.zeros(xh.shape, np.uint8), np.zeros(shp, np.float32), np.zeros(shp, np.float32),
                np.zeros(shp, bool))
    x = xh.astype(np.float32)
    bad = ~np.all(np.isfinite(x), axis=-1)
    with np.errstate(invalid="ignore", divide="ignore", over="ignore"):
        mn = x.min(axis=-1) + np.float32(0.0)
        mx = x.max(axis=-1) + np.float32(0.0)
        scale = (mx - mn) / np.float32(L - 1)
        d = x - mn[..., None]
        safe = np.where(scale == 0, np.float32(1.0), scale)
        t = d / safe[..., None]
        c = np.clip(np.rint(t), 0, L - 1)
    c = np.where((scale == 0)[..., None] | bad[..., None], 0, c)
    return c.astype(np.uint8), mn.astype(np.float32), scale.astype(np.float32), bad


def pack_rows(codes: np.ndarray, L: int) -> np.ndarray:
    """Mixed-radix packing: word w = sum_j codes[w*n + j] * L**j  (uint32).

    n = digits_per_word(L) codes per word, little-endian digits (digit 0 is the
    least significant), zero-padded past D, rows never share a word (reading).
    Each word is formed by Horner's rule from its highest digit.
    """
    n = digits_per_word(L)
    D = codes.shape[-1]
    W = words_per_row(L, D)
    c = np.zeros(codes.shape[:-1] + (W * n,), dtype=np.uint64)
    c[..., :D] = codes
    c = c.reshape(codes.shape[:-1] + (W, n))
    word = np.zeros(codes.shape[:-1] + (W,), dtype=np.uint64)
    for j in reversed(range(n)):
        word = word * np.uint64(L) + c[..., j]
    assert np.all(word < (1 << 32))
    return word.astype(np.uint32)


def unpack_rows(words: np.ndarray, L: int, D: int = HEAD_DIM) -> np.ndarray:
    """Inverse of pack_rows by repeated division: returns uint8 codes [..., D]."""
    n = digits_per_word(L)
    w = words.astype(np.uint64)
    digits = []
    for _ in range(n):
        digits.append((w % np.uint64(L)).astype(np.uint8))
        w = w // np.uint64(L)
    c = np.stack(digits, axis=-1).reshape(words.shape[:-1] + (words.shape[-1] * n,))
    return c[..., :D]


def dequantize(codes: np.ndarray, mn: np.ndarray, scale: np.ndarray) -> np.ndarray:
    """x_hat = mn + code * scale, in float64 (exact for these operand sizes)."""
    return mn[..., None].astype(np.float64) + codes.astype(np.float64) * scale[..., None].astype(np.float64)


# ---------------------------------------------------------------------------
# a4 pool write: one mask per sequence broadcast to every layer and KV head,
# K and V alike (SemKV, Fig. 5); pools keep ascending token order.
# ---------------------------------------------------------------------------
@dataclass
class Pool:
    """Quantized rows of one class (high or low) for one (sequence, layer, head)."""
    words: np.ndarray   # uint32 [n][W]
    mn: np.ndarray      # float32 [n]
    scale: np.ndarray   # float32 [n]


def quantize_slab(x: np.ndarray, mask: np.ndarray, L_high: int, L_low: int, rotate: bool = False):
    """Quantize the rows x [T][D] of one (sequence, layer, head) under one mask.

    Returns (high Pool, low Pool, bad rows).  Row j goes to the high pool when
    mask[j] == 1, else to the low pool; within a pool rows keep token order,
    so a token's slot is the number of same-class tokens before it.  With
    rotate, each fp16 row is first widened to float32 and rotated (fwht128),
    and the rotated row is what is quantized and stored.
    """
    if rotate:
        x = fwht128(x.astype(np.float32))
    out = []
    bad_any = np.zeros(x.shape[0], dtype=bool)
    for cls, L in ((1, L_high), (0, L_low)):
        idx = np.nonzero(mask == cls)[0]
        codes, mn, scale, bad = quantize_rows(x[idx], L)
        bad_any[idx] |= bad
        out.append(Pool(pack_rows(codes, L), mn, scale))
    return out[0], out[1], bad_any


# ---------------------------------------------------------------------------
# a5: generation-time block-exact deferred quantization (SemKV, Fig. 6)
# ---------------------------------------------------------------------------
@dataclass
class SlabCache:
    """Mixed cache of one (sequence, layer, head): K and V pools plus the FP16 block."""
    kh: list = field(default_factory=list)
    kl: list = field(default_factory=list)
    vh: list = field(default_factory=list)
    vl: list = field(default_factory=list)


class MixedCache:
    """The whole mixed-precision cache of B sequences, Lyr layers, H KV heads.

    prefill(): one mask per sequence from the prompt ranking, applied to every
    layer and head (SemKV, Fig. 5).  append(): new tokens go to an FP16 block;
    each time the block holds BLOCK tokens its own scores are ranked, the top
    ceil(r * BLOCK) get L_high, the block is quantized onto the pools and
    emptied (SemKV, Fig. 6: deferred, block-exact, no threshold).  flush():
    the end-of-turn residual block is quantized by the same rule with
    ceil(r * n_residual).  Reading: the block is quantized as soon as it is
    full, so a full block never stays in FP16.
    """

    def __init__(self, B, Lyr, H, L_high, L_low, r_ppm, block=BLOCK, D=HEAD_DIM, rotate=False):
        self.B, self.Lyr, self.H, self.D = B, Lyr, H, D
        self.rotate = rotate
        self.L_high, self.L_low, self.r_ppm, self.block = L_high, L_low, r_ppm, block
        self.slabs = [[[SlabCache() for _ in range(H)] for _ in range(Lyr)] for _ in range(B)]
        self.buf_k = np.zeros((B, Lyr, H, 0, D), dtype=np.float16)
        self.buf_v = np.zeros((B, Lyr, H, 0, D), dtype=np.float16)
        self.buf_score = np.zeros((B, 0), dtype=np.float32)
        self.n_high = np.zeros(B, dtype=np.int64)
        self.n_low = np.zeros(B, dtype=np.int64)
        self.bad = False

    def _quantize_tokens(self, b, k, v, mask):
        """k, v: fp16 [Lyr][H][n][D] of sequence b; appends to its pools."""
        for l in range(self.Lyr):
            for h in range(self.H):
                slab = self.slabs[b][l][h]
                for x, hi_list, lo_list in ((k, slab.kh, slab.kl), (v, slab.vh, slab.vl)):
                    ph, pl, bad = quantize_slab(x[l, h], mask, self.L_high, self.L_low, self.rotate)
                    hi_list.append(ph)
                    lo_list.append(pl)
                    self.bad |= bool(bad.any())
        nh = int(mask.sum())
        self.n_high[b] += nh
        self.n_low[b] += mask.shape[0] - nh

    def prefill(self, k, v, seq_len, masks):
        """k, v: fp16 [B][Lyr][H][T_max][D]; masks[b]: uint8 [seq_len[b]]."""
        for b in range(self.B):
            T = int(seq_len[b])
            self._quantize_tokens(b, k[b, :, :, :T], v[b, :, :, :T], masks[b][:T])

    def _quantize_block(self):
        n = self.buf_k.shape[3]
        if n == 0:
            return
        nh = num_high(n, self.r_ppm)
        for b in range(self.B):
            mask = select_mask(self.buf_score[b], nh)
            self._quantize_tokens(b, self.buf_k[b], self.buf_v[b], mask)
        D = self.D
        self.buf_k = np.zeros((self.B, self.Lyr, self.H, 0, D), dtype=np.float16)
        self.buf_v = np.zeros((self.B, self.Lyr, self.H, 0, D), dtype=np.float16)
        self.buf_score = np.zeros((self.B, 0), dtype=np.float32)

    def append(self, k_new, v_new, score_new):
        """k_new, v_new: fp16 [B][Lyr][H][n][D]; score_new: fp32 [B][n]."""
        n = k_new.shape[3]
        i = 0
        while i < n:
            take = min(n - i, self.block - self.buf_k.shape[3])
            self.buf_k = np.concatenate([self.buf_k, k_new[:, :, :, i:i + take]], axis=3)
            self.buf_v = np.concatenate([self.buf_v, v_new[:, :, :, i:i + take]], axis=3)
            self.buf_score = np.concatenate([self.buf_score, score_new[:, i:i + take]], axis=1)
            i += take
            if self.buf_k.shape[3] == self.block:
                self._quantize_block()

    def flush(self):
        self._quantize_block()

    def pools(self, b, l, h, which):
        """Concatenated Pool of (sequence b, layer l, head h); which in kh/kl/vh/vl."""
        parts = getattr(self.slabs[b][l][h], which)
        if not parts:
            return Pool(np.zeros((0, 0), np.uint32), np.zeros(0, np.float32), np.zeros(0, np.float32))
        return Pool(np.concatenate([p.words for p in parts]),
                    np.concatenate([p.mn for p in parts]),
                    np.concatenate([p.scale for p in parts]))

    def decode(self, q, sm_scale=None, layer0=0, score_layer=None):
        """GQA decode attention over the mixed cache, float64 (see decode_attn).

        With score_layer set, the FP16 block's tokens also accumulate the
        attention they receive at that layer (see buffer_attention_mass)."""
        B, nL, H_q, D = q.shape
        out = np.zeros((B, nL, H_q, D), dtype=np.float64)
        for b in range(B):
            for li in range(nL):
                l = layer0 + li
                keys, vals = [], []
                for h in range(self.H):
                    kk, vv = [], []
                    for dst, pair in ((kk, (("kh", self.L_high), ("kl", self.L_low))),
                                      (vv, (("vh", self.L_high), ("vl", self.L_low)))):
                        for which, L in pair:
                            p = self.pools(b, l, h, which)
                            if p.words.shape[0]:
                                x = dequantize(unpack_rows(p.words, L, D), p.mn, p.scale)
                                # stored rows are rotated: back to the token's own basis
                                dst.append(fwht128(x) / 128.0 if self.rotate else x)
                    kk.append(self.buf_k[b, l, h].astype(np.float64))
                    vv.append(self.buf_v[b, l, h].astype(np.float64))
                    keys.append(np.concatenate(kk))
                    vals.append(np.concatenate(vv))
                out[b, li] = decode_attn(q[b, li], keys, vals, sm_scale)
                nb = self.buf_k.shape[3]
                if score_layer is not None and l == score_layer and nb > 0:
                    mass = buffer_attention_mass(q[b, li], keys, nb, sm_scale)
                    self.buf_score[b] = (self.buf_score[b].astype(np.float64) + mass).astype(np.float32)
        return out


# ---------------------------------------------------------------------------
# a6: decoding over the mixed cache (SemKV, Fig. 5: "used for decoding")
# ---------------------------------------------------------------------------
def decode_attn(q: np.ndarray, keys: list, vals: list, sm_scale=None) -> np.ndarray:
    """Textbook softmax attention of one decode query per head, float64.

    q: [H_q][D]; keys[g], vals[g]: [n_g][D] (already dequantized) for KV head g.
    Query head h attends over KV head floor(h / (H_q / H)).
    """
    H_q, D = q.shape
    H = len(keys)
    G = H_q // H
    if sm_scale is None:
        sm_scale = 1.0 / math.sqrt(D)
    out = np.zeros((H_q, D), dtype=np.float64)
    for h in range(H_q):
        g = h // G
        k = keys[g]
        if k.shape[0] == 0:
            continue
        logits = (k @ q[h].astype(np.float64)) * sm_scale
        e = np.exp(logits - logits.max())
        p = e / e.sum()
        out[h] = p @ vals[g]
    return out


def buffer_attention_mass(q: np.ndarray, keys: list, n_buf: int, sm_scale=None) -> np.ndarray:
    """Attention mass of the FP16-block tokens in one decode step, float64.

    SemKV, Fig. 6: generated tokens wait in the FP16 block and their scores
    are accumulated until the block is ranked; Fig. 12: attention-based
    indicators.  Reading: at the scoring layer, token t of the block receives
    sum over the H_q query heads of its softmax probability, normalised over
    every cached token of the head's KV head (pools and block), i.e. the same
    probabilities decode_attn uses.  keys[g] ends with the n_buf block tokens.
    """
    H_q, D = q.shape
    H = len(keys)
    G = H_q // H
    if sm_scale is None:
        sm_scale = 1.0 / math.sqrt(D)
    mass = np.zeros(n_buf, dtype=np.float64)
    for h in range(H_q):
        k = keys[h // G]
        logits = (k @ q[h].astype(np.float64)) * sm_scale
        e = np.exp(logits - logits.max())
        mass += (e / e.sum())[k.shape[0] - n_buf:]
    return mass


# ---------------------------------------------------------------------------
# Storage accounting (SemKV, Table 3, Table 5, Table 6, Table 7, Fig. 11, Fig. 18)
# ---------------------------------------------------------------------------
def pages_code_bits(L: int, max_group: int = 5) -> float:
    """Bits per value when groups of k <= 5 base-L digits are stored in ceil(k log2 L) bits.

    Reading of the pages' "effective bits include packing" (SemKV, Table 6):
    the densest such grouping reproduces the printed code-bit column
    (2.333 for 5 levels, 2.600 for 6 levels).
    """
    return min(math.ceil(k * math.log2(L) - 1e-12) / k for k in range(1, max_group + 1))


def pages_effective_bits(levels_and_fracs, meta_scalars: int, D: int = HEAD_DIM) -> float:
    """Average code bits over the token mix plus per-row metadata of 16-bit scalars.

    levels_and_fracs: [(L, fraction of tokens), ...]; meta_scalars = 2 for the
    affine quantizer, 1 for TurboQuant-MSE (SemKV, Table 6 caption).
    """
    code = sum(f * pages_code_bits(L) for L, f in levels_and_fracs)
    return code + meta_scalars * 16 / D


def layout_bytes_per_row(L: int, D: int = HEAD_DIM) -> int:
    """Bytes of one row in the library's layout: 32-bit mixed-radix words + fp32 (mn, scale)."""
    return 4 * words_per_row(L, D) + 8


# ---------------------------------------------------------------------------
# f1: the pages' own storage layout (SemKV, Table 3, Table 5, Table 6, Fig. 11:
# "effective bits include packing and per-row metadata", two 16-bit scalars)
# ---------------------------------------------------------------------------
def pages_group(L: int, max_group: int = 5):
    """(g, b) of the pages' packing: g <= 5 base-L digits held in b whole bits,
    b the fewest bits that hold L**g values, with the g of fewest bits per digit
    (of equal ones, the largest g).  Reading of the printed code bits
    (pages_code_bits): 5 levels -> 3 digits in 7 bits, 6 levels -> 5 in 13."""
    best = None
    for k in range(1, max_group + 1):
        b = (L ** k - 1).bit_length()
        key = (Fraction(b, k), -k)
        if best is None or key < best[0]:
            best = (key, k, b)
    return best[1], best[2]


def pages_row_bits(L: int, D: int = HEAD_DIM) -> int:
    """Code bits of one row: D // g full groups of b bits, then a tail group of
    the D % g remaining digits in the fewest bits that hold L**(D % g) values."""
    g, b = pages_group(L)
    t = D % g
    return (D // g) * b + ((L ** t - 1).bit_length() if t else 0)


def pages_groups(L: int, D: int = HEAD_DIM):
    """[(first digit, digits, bits, bit offset in the row)] of every group of a row."""
    g, b = pages_group(L)
    out, off, d0 = [], 0, 0
    while d0 < D:
        k = min(g, D - d0)
        bits = (L ** k - 1).bit_length()
        out.append((d0, k, bits, off))
        off += bits
        d0 += k
    return out


def pack_rows_pages(codes: np.ndarray, L: int) -> np.ndarray:
    """Rows of codes uint8 [n][D] -> the pages' bit stream, uint8 bytes.

    Row s occupies stream bits [s*R, (s+1)*R), R = pages_row_bits(L): rows sit
    back to back at bit granularity (reading: no padding, so that the stored
    bytes are the printed effective bits).  Stream bit k is bit k % 8 of byte
    k // 8.  Group (d0, k, bits, off) of a row holds the value
    sum_j codes[d0 + j] * L**j (digit 0 least significant) in row bits
    [off, off + bits), least significant bit first.  The stream is zero-padded
    to whole bytes.
    """
    n, D = codes.shape
    R = pages_row_bits(L, D)
    stream = np.zeros(n * R, dtype=np.uint8)
    rows = np.arange(n, dtype=np.int64) * R
    for d0, k, bits, off in pages_groups(L, D):
        val = np.zeros(n, dtype=np.int64)
        for j in reversed(range(k)):
            val = val * L + codes[:, d0 + j].astype(np.int64)
        for i in range(bits):
            stream[rows + off + i] = (val >> i) & 1
    return np.packbits(stream, bitorder="little")


def unpack_rows_pages(stream: np.ndarray, n: int, L: int, D: int = HEAD_DIM) -> np.ndarray:
    """Inverse of pack_rows_pages: uint8 codes [n][D], by repeated division of each group."""
    bits = np.unpackbits(np.asarray(stream, dtype=np.uint8), bitorder="little")
    R = pages_row_bits(L, D)
    rows = np.arange(n, dtype=np.int64) * R
    codes = np.zeros((n, D), dtype=np.uint8)
    for d0, k, nb, off in pages_groups(L, D):
        val = np.zeros(n, dtype=np.int64)
        for i in range(nb):
            val |= bits[rows + off + i].astype(np.int64) << i
        for j in range(k):
            codes[:, d0 + j] = val % L
            val //= L
    return codes


def pages_meta(mn: np.ndarray, scale: np.ndarray):
    """The two 16-bit scalars of a row: (min, scale) rounded to float16, nearest-even.
    A scale that does not fit float16 (possible only for L = 2) becomes inf."""
    with np.errstate(over="ignore"):
        return mn.astype(np.float16), scale.astype(np.float16)


def pages_layout_bytes(n_rows: int, L: int, D: int = HEAD_DIM) -> int:
    """Bytes of n_rows rows in the pages' layout: the bit stream plus 4 bytes of scalars per row."""
    return (n_rows * pages_row_bits(L, D) + 7) // 8 + 4 * n_rows
