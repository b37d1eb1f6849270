"""SemKV token-wise mixed-precision KV-cache hot path for B200 (sm_100a).

The kernels live in libsemkv.so (C ABI: include/semkv.h); this package is a
thin binding with the same names.  Importing it fails loudly if the library
has not been built (`python kv_cache_mixed_b200/build.py`).
"""
from .binding import (FLAG_CAPACITY, FLAG_NONFINITE, FLAG_SEQLEN, FLAG_TIMEOUT, FLUSH, LAYOUT_PAGES,  # noqa: F401
                      LAYOUT_WORDS, SCORE_ATTN_MASS, semkv_pool_words, semkv_row_bits,
                      SCORE_KEY_L2, EXPORTED, LIB_PATH, MixedCache, SemkvError, semkv_append_block,
                      semkv_decode_attn, semkv_decode_attn_acc, semkv_digits_per_word, semkv_num_high, semkv_quantize,
                      semkv_quantize_noalloc, semkv_score, semkv_select, semkv_set_first_copy_wait_polls,
                      semkv_check_reciprocal, semkv_version,
                      semkv_words_per_row)
