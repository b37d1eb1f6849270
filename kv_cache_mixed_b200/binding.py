"""Thin ctypes binding of libsemkv (include/semkv.h), same names as the C ABI.

Argument marshalling only: torch tensors become device pointers, the current
torch CUDA stream becomes the cudaStream_t.  Every step of the path runs in the
library's kernels.  Importing this module fails loudly when libsemkv.so is
missing: there is no fallback of any kind.
"""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libsemkv.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"libsemkv.so not built at {LIB_PATH}; run `python kv_cache_mixed_b200/build.py`")
_lib = ctypes.CDLL(LIB_PATH)

SEMKV_OK = 0
STATUS_NAMES = {0: "OK", 1: "ERR_INVALID_ARG", 2: "ERR_UNSUPPORTED", 3: "ERR_WORKSPACE",
                4: "ERR_CAPACITY", 5: "ERR_CUDA"}
FLAG_NONFINITE, FLAG_CAPACITY, FLAG_SEQLEN, FLAG_TIMEOUT = 0x1, 0x2, 0x4, 0x8
SCORE_ATTN_MASS, SCORE_KEY_L2 = 0, 1
FLUSH = 0x1
LAYOUT_WORDS, LAYOUT_PAGES = 0, 1

_p = ctypes.c_void_p
_i32, _i64, _u32, _sz, _f32 = ctypes.c_int32, ctypes.c_int64, ctypes.c_uint32, ctypes.c_size_t, ctypes.c_float


class SemkvCache(ctypes.Structure):
    """Mirror of struct semkv_cache."""
    _fields_ = [(n, _i32) for n in ("B", "n_layers", "H", "H_q", "D", "L_high", "L_low", "r_ppm",
                                     "cap_high", "cap_low", "block", "buf_len", "rotate", "layout")] + \
               [(n, _p) for n in ("k_high", "v_high", "k_low", "v_low", "k_high_meta", "v_high_meta",
                                  "k_low_meta", "v_low_meta", "n_high", "n_low", "buf_k", "buf_v",
                                  "buf_score")]


def _sig(name, res, args):
    f = getattr(_lib, name)
    f.restype = res
    f.argtypes = args
    return f


_lib_num_high = _sig("semkv_num_high", _i64, [_i64, _i32])
_lib_digits = _sig("semkv_digits_per_word", _i32, [_i32])
_lib_words = _sig("semkv_words_per_row", _i32, [_i32, _i32])
_lib_row_bits = _sig("semkv_row_bits", _i32, [_i32, _i32])
_lib_pool_words = _sig("semkv_pool_words", _i64, [_i32, _i32, _i32])
_lib_version = _sig("semkv_version", ctypes.c_char_p, [])
_lib_set_wait0 = _sig("semkv_set_first_copy_wait_polls", None, [_i32])
_lib_rcp_check = _sig("semkv_check_reciprocal", _i32, [_u32, _u32, _p, _p])
_lib_score_ws = _sig("semkv_score_workspace_size", _sz, [_i32, _i32, _i32, _i32, _i32, _i32])
_lib_score = _sig("semkv_score", _i32, [_i32, _p, _i64, _p, _p, _i32, _i32, _i32, _i32, _i32, _i32,
                                        _p, _p, _sz, _p, _p])
_lib_select_ws = _sig("semkv_select_workspace_size", _sz, [_i32, _i32])
_lib_select = _sig("semkv_select", _i32, [_p, _i64, _p, _i32, _i32, _i32, _i32, _p, _i64, _p, _sz, _p, _p])
_lib_quant_ws = _sig("semkv_quantize_workspace_size", _sz, [_i32, _i32])
_lib_quant = _sig("semkv_quantize", _i32, [ctypes.POINTER(SemkvCache), _p, _p, _i32, _p, _p, _p, _sz, _p, _p])
_lib_quant_noalloc = _sig("semkv_quantize_noalloc", _i32, [ctypes.POINTER(SemkvCache), _p, _p, _i32, _p, _p, _p,
                                                            _p])
_lib_append_ws = _sig("semkv_append_workspace_size", _sz, [ctypes.POINTER(SemkvCache)])
_lib_append = _sig("semkv_append_block", _i32, [ctypes.POINTER(SemkvCache), _p, _p, _p, _i32, _u32, _p, _sz,
                                                _p, _p])
_lib_decode_ws = _sig("semkv_decode_workspace_size", _sz, [ctypes.POINTER(SemkvCache), _i32])
_lib_decode = _sig("semkv_decode_attn", _i32, [ctypes.POINTER(SemkvCache), _i32, _i32, _p, _p, _f32, _p, _sz, _p,
                                                _p])
_lib_decode_acc = _sig("semkv_decode_attn_acc", _i32, [ctypes.POINTER(SemkvCache), _i32, _i32, _i32, _p, _p, _f32,
                                                      _p, _sz, _p, _p])

EXPORTED = ["semkv_num_high", "semkv_digits_per_word", "semkv_words_per_row", "semkv_row_bits",
            "semkv_pool_words", "semkv_version",
            "semkv_set_first_copy_wait_polls", "semkv_check_reciprocal",
            "semkv_score_workspace_size", "semkv_score", "semkv_select_workspace_size", "semkv_select",
            "semkv_quantize_workspace_size", "semkv_quantize", "semkv_quantize_noalloc",
            "semkv_append_workspace_size",
            "semkv_append_block", "semkv_decode_workspace_size", "semkv_decode_attn", "semkv_decode_attn_acc"]


class SemkvError(RuntimeError):
    pass


def _check(code, what):
    if code != SEMKV_OK:
        raise SemkvError(f"{what}: {STATUS_NAMES.get(code, code)}")


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _ws(nbytes, device):
    return torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device=device)


# ------------------------------------------------------------------ host helpers
def semkv_num_high(n: int, r_ppm: int) -> int:
    return int(_lib_num_high(n, r_ppm))


def semkv_digits_per_word(L: int) -> int:
    return int(_lib_digits(L))


def semkv_words_per_row(L: int, D: int = 128) -> int:
    return int(_lib_words(L, D))


def semkv_row_bits(layout: int, L: int) -> int:
    return int(_lib_row_bits(layout, L))


def semkv_pool_words(layout: int, L: int, cap: int) -> int:
    return int(_lib_pool_words(layout, L, cap))


def semkv_version() -> str:
    return _lib_version().decode()


def semkv_set_first_copy_wait_polls(polls: int) -> None:
    """Testing aid: poll bound of the first copy wait of later quantize/decode launches (< 0: default)."""
    _lib_set_wait0(int(polls))


def semkv_check_reciprocal(exp_lo: int, exp_hi: int, stream=None) -> int:
    """Differences between the quantizer's reciprocal and the IEEE one over exponent fields [exp_lo, exp_hi]."""
    out = torch.zeros(1, dtype=torch.int64, device="cuda")
    _check(_lib_rcp_check(exp_lo, exp_hi, _ptr(out), _stream(stream)), "semkv_check_reciprocal")
    return int(out.item())


# ------------------------------------------------------------------ a1 score
def semkv_score(kind: int, k: torch.Tensor, k_batch_stride: int, q_win, seq_len: torch.Tensor,
                B: int, T_max: int, H: int, H_q: int, w: int, score: torch.Tensor, ws=None,
                status=None, stream=None):
    """k: fp16 view whose sequence b starts at k.data_ptr() + 2*b*k_batch_stride ([H][T_max][128])."""
    nbytes = int(_lib_score_ws(kind, B, T_max, H, H_q, w))
    if ws is None and nbytes:
        ws = _ws(nbytes, k.device)
    _check(_lib_score(kind, _ptr(k), k_batch_stride, _ptr(q_win), _ptr(seq_len), B, T_max, H, H_q, 128, w,
                      _ptr(score), _ptr(ws), 0 if ws is None else ws.numel(), _ptr(status),
                      _stream(stream)), "semkv_score")
    return score


def semkv_select(score: torch.Tensor, seq_len, r_ppm: int, mask: torch.Tensor, len_const: int = 0,
                 status=None, stream=None):
    """score fp32 [B][T_max] (contiguous rows), mask uint8 [B][T_max]."""
    B, T_max = score.shape
    _check(_lib_select(_ptr(score), score.stride(0), _ptr(seq_len), len_const, B, T_max, r_ppm, _ptr(mask),
                       mask.stride(0), None, 0, _ptr(status), _stream(stream)), "semkv_select")
    return mask


# ------------------------------------------------------------------ the mixed cache
class MixedCache:
    """Device memory of one mixed cache (pools, counts, FP16 block) and its C struct.

    Pools are torch tensors on `device`, laid out as include/semkv.h describes:
    with layout=LAYOUT_WORDS the codes are int32 [B][n_layers][H][cap][W] and the
    meta float32 [B][n_layers][H][cap][2]; with layout=LAYOUT_PAGES the codes are
    one int32 bit stream [B][n_layers][H][semkv_pool_words(...)] per slab and the
    meta float16 [B][n_layers][H][cap][2].
    """

    def __init__(self, B, n_layers, H, H_q, L_high, L_low, r_ppm, cap_high, cap_low, block=128,
                 device="cuda", rotate=False, layout=LAYOUT_WORDS):
        self.device = torch.device(device)
        cap_high = (int(cap_high) + 15) // 16 * 16
        cap_low = (int(cap_low) + 15) // 16 * 16
        self.layout = layout
        self.W_high = semkv_words_per_row(L_high)
        self.W_low = semkv_words_per_row(L_low)
        self.row_bits_high = semkv_row_bits(layout, L_high)
        self.row_bits_low = semkv_row_bits(layout, L_low)
        if self.row_bits_high < 0 or self.row_bits_low < 0:
            raise SemkvError("semkv_row_bits: ERR_UNSUPPORTED (level not available in this layout)")
        d = self.device
        if layout == LAYOUT_PAGES:
            def codes(L, cap):
                return torch.zeros((B, n_layers, H, semkv_pool_words(layout, L, cap)), dtype=torch.int32, device=d)
            mdt = torch.float16
        else:
            def codes(L, cap):
                return torch.zeros((B, n_layers, H, cap, semkv_words_per_row(L)), dtype=torch.int32, device=d)
            mdt = torch.float32
        self.k_high = codes(L_high, cap_high)
        self.v_high = torch.zeros_like(self.k_high)
        self.k_low = codes(L_low, cap_low)
        self.v_low = torch.zeros_like(self.k_low)
        self.k_high_meta = torch.zeros((B, n_layers, H, cap_high, 2), dtype=mdt, device=d)
        self.v_high_meta = torch.zeros_like(self.k_high_meta)
        self.k_low_meta = torch.zeros((B, n_layers, H, cap_low, 2), dtype=mdt, device=d)
        self.v_low_meta = torch.zeros_like(self.k_low_meta)
        self.n_high = torch.zeros(B, dtype=torch.int32, device=d)
        self.n_low = torch.zeros(B, dtype=torch.int32, device=d)
        self.buf_k = torch.zeros((B, n_layers, H, block, 128), dtype=torch.float16, device=d)
        self.buf_v = torch.zeros_like(self.buf_k)
        self.buf_score = torch.zeros((B, block), dtype=torch.float32, device=d)
        self.status = torch.zeros(1, dtype=torch.int32, device=d)
        self.c = SemkvCache(B, n_layers, H, H_q, 128, L_high, L_low, r_ppm, cap_high, cap_low, block, 0,
                            1 if rotate else 0, int(layout),
                            *[t.data_ptr() for t in (self.k_high, self.v_high, self.k_low, self.v_low,
                                                     self.k_high_meta, self.v_high_meta, self.k_low_meta,
                                                     self.v_low_meta, self.n_high, self.n_low, self.buf_k,
                                                     self.buf_v, self.buf_score)])
        self._ws = {}

    # plain attributes
    B = property(lambda s: s.c.B)
    n_layers = property(lambda s: s.c.n_layers)
    H = property(lambda s: s.c.H)
    H_q = property(lambda s: s.c.H_q)
    buf_len = property(lambda s: s.c.buf_len)

    def workspace(self, key, nbytes):
        t = self._ws.get(key)
        if t is None or t.numel() < nbytes:
            t = _ws(nbytes, self.device)
            self._ws[key] = t
        return t

    def status_flags(self) -> int:
        return int(self.status.item()) & 0xFFFFFFFF

    def pool_bytes(self) -> int:
        """Bytes of the pools (codes + meta) currently in use, summed over sequences."""
        nh = self.n_high.sum().item()
        nl = self.n_low.sum().item()
        rows = self.c.n_layers * self.c.H * 2
        if self.layout == LAYOUT_PAGES:
            return int(rows * ((nh * self.row_bits_high + 7) // 8 + (nl * self.row_bits_low + 7) // 8 + 4 * (nh + nl)))
        return int(rows * (nh * (4 * self.W_high + 8) + nl * (4 * self.W_low + 8)))


def semkv_quantize(cache: MixedCache, k: torch.Tensor, v: torch.Tensor, seq_len: torch.Tensor,
                   mask: torch.Tensor, stream=None):
    """k, v fp16 [B][n_layers][H][T_max][128]; mask uint8 [B][T_max]."""
    T_max = k.shape[3]
    ws = cache.workspace("quant", int(_lib_quant_ws(cache.c.B, T_max)))
    _check(_lib_quant(ctypes.byref(cache.c), _ptr(k), _ptr(v), T_max, _ptr(seq_len), _ptr(mask), _ptr(ws),
                      ws.numel(), _ptr(cache.status), _stream(stream)), "semkv_quantize")


def semkv_quantize_noalloc(cache: MixedCache, k: torch.Tensor, v: torch.Tensor, seq_len: torch.Tensor,
                           mask: torch.Tensor, stream=None):
    """semkv_quantize with the library's fixed scratch array instead of a workspace."""
    _check(_lib_quant_noalloc(ctypes.byref(cache.c), _ptr(k), _ptr(v), k.shape[3], _ptr(seq_len), _ptr(mask),
                              _ptr(cache.status), _stream(stream)), "semkv_quantize_noalloc")


def semkv_append_block(cache: MixedCache, k_new, v_new, score_new, n: int, flags: int = 0, stream=None):
    """k_new, v_new fp16 [B][n_layers][H][n][128]; score_new fp32 [B][n]."""
    ws = cache.workspace("append", int(_lib_append_ws(ctypes.byref(cache.c))))
    _check(_lib_append(ctypes.byref(cache.c), _ptr(k_new), _ptr(v_new), _ptr(score_new), n, flags, _ptr(ws),
                       ws.numel(), _ptr(cache.status), _stream(stream)), "semkv_append_block")


def semkv_decode_attn(cache: MixedCache, layer0: int, n_layers: int, q: torch.Tensor, out: torch.Tensor,
                      sm_scale: float = 128 ** -0.5, stream=None):
    """q, out fp16 [B][n_layers][H_q][128]."""
    ws = cache.workspace(("decode", n_layers), int(_lib_decode_ws(ctypes.byref(cache.c), n_layers)))
    _check(_lib_decode(ctypes.byref(cache.c), layer0, n_layers, _ptr(q), _ptr(out), sm_scale, _ptr(ws),
                       ws.numel(), _ptr(cache.status), _stream(stream)), "semkv_decode_attn")
    return out


def semkv_decode_attn_acc(cache: MixedCache, layer0: int, n_layers: int, score_layer: int, q: torch.Tensor,
                          out: torch.Tensor, sm_scale: float = 128 ** -0.5, stream=None):
    """semkv_decode_attn, and the FP16 block's attention mass at score_layer added into cache.buf_score."""
    ws = cache.workspace(("decode", n_layers), int(_lib_decode_ws(ctypes.byref(cache.c), n_layers)))
    _check(_lib_decode_acc(ctypes.byref(cache.c), layer0, n_layers, score_layer, _ptr(q), _ptr(out), sm_scale,
                           _ptr(ws), ws.numel(), _ptr(cache.status), _stream(stream)), "semkv_decode_attn_acc")
    return out
