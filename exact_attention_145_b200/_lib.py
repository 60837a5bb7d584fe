"""ctypes mirror of include/attn.h. Loading fails loudly when libattn.so is
missing: there is no fallback path of any kind."""
from __future__ import annotations

import ctypes
import os
import threading

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libattn.so")
TRACE_LIB_PATH = os.path.join(HERE, "libattn_trace.so")


def lib_path() -> str:
    """libattn.so, or with ATTN_LIBRARY_VARIANT=trace (set before the first
    call) the cycle-trace build libattn_trace.so: the same kernels plus trace
    records at the pipeline hand-offs (see trace.py). ATTN_LIBRARY=<path>
    loads another build of the same C ABI instead."""
    if os.environ.get("ATTN_LIBRARY"):
        return os.path.abspath(os.environ["ATTN_LIBRARY"])
    return TRACE_LIB_PATH if os.environ.get("ATTN_LIBRARY_VARIANT") == "trace" else LIB_PATH

ATTN_OK, ATTN_ERR_INVALID_ARG, ATTN_ERR_UNSUPPORTED, ATTN_ERR_CUDA, ATTN_ERR_WORKSPACE = range(5)
ATTN_DEV_TIMEOUT, ATTN_DEV_BAD_PAGE, ATTN_DEV_BAD_LEN, ATTN_DEV_BAD_MASK = 1, 2, 4, 8
MASK_NONE, MASK_CAUSAL, MASK_WINDOW, MASK_DOCUMENT = range(4)
MOD_NONE, MOD_SOFTCAP, MOD_ALIBI, MOD_RELU = range(4)

EXPORTS = ("attn_block_mask_bytes", "attn_block_mask_layout", "attn_build_block_mask", "attn_fwd",
           "attn_decode_num_splits", "attn_decode_workspace_bytes", "attn_decode", "attn_lse_combine",
           "attn_status_str", "attn_decode_noalloc", "attn_selftest_wait_timeout", "attn_bwd_workspace_bytes",
           "attn_bwd", "attn_kvcache_update")
ATTN_DECODE_NOALLOC_MAX_BYTES = 32 * 1024 * 1024

c_i64x3 = ctypes.c_int64 * 3
c_i64x2 = ctypes.c_int64 * 2


class MaskSpec(ctypes.Structure):
    _fields_ = [("kind", ctypes.c_int), ("window_left", ctypes.c_int), ("window_right", ctypes.c_int),
                ("q_offset", ctypes.c_int), ("doc_id", ctypes.c_void_p), ("doc_batch_stride", ctypes.c_int64)]


class BlockMaskC(ctypes.Structure):
    _fields_ = [("Bm", ctypes.c_int), ("Hm", ctypes.c_int),
                ("Sq", ctypes.c_int), ("Skv", ctypes.c_int), ("blk_q", ctypes.c_int), ("blk_kv", ctypes.c_int),
                ("n_q_tiles", ctypes.c_int), ("n_kv_tiles", ctypes.c_int),
                ("cls", ctypes.c_void_p), ("part_cnt", ctypes.c_void_p), ("part_idx", ctypes.c_void_p),
                ("full_cnt", ctypes.c_void_p), ("full_idx", ctypes.c_void_p),
                ("row_order", ctypes.c_void_p), ("doc_start", ctypes.c_void_p), ("doc_sorted", ctypes.c_void_p)]


class FwdParams(ctypes.Structure):
    _fields_ = [("q", ctypes.c_void_p), ("k", ctypes.c_void_p), ("v", ctypes.c_void_p), ("o", ctypes.c_void_p),
                ("lse", ctypes.c_void_p),
                ("q_stride", c_i64x3), ("k_stride", c_i64x3), ("v_stride", c_i64x3), ("o_stride", c_i64x3),
                ("B", ctypes.c_int), ("Hq", ctypes.c_int), ("Hkv", ctypes.c_int), ("Sq", ctypes.c_int),
                ("Skv", ctypes.c_int), ("D", ctypes.c_int), ("scale", ctypes.c_float),
                ("mask", MaskSpec), ("block_mask", ctypes.POINTER(BlockMaskC)),
                ("mod", ctypes.c_int), ("softcap", ctypes.c_float), ("alibi_slopes", ctypes.c_void_p),
                ("alibi_batch_stride", ctypes.c_int), ("status", ctypes.c_void_p)]


class BwdParams(ctypes.Structure):
    _fields_ = [("q", ctypes.c_void_p), ("k", ctypes.c_void_p), ("v", ctypes.c_void_p), ("o", ctypes.c_void_p),
                ("dout", ctypes.c_void_p), ("lse", ctypes.c_void_p),
                ("dq", ctypes.c_void_p), ("dk", ctypes.c_void_p), ("dv", ctypes.c_void_p),
                ("q_stride", c_i64x3), ("k_stride", c_i64x3), ("v_stride", c_i64x3), ("o_stride", c_i64x3),
                ("do_stride", c_i64x3), ("dq_stride", c_i64x3), ("dk_stride", c_i64x3), ("dv_stride", c_i64x3),
                ("B", ctypes.c_int), ("Hq", ctypes.c_int), ("Hkv", ctypes.c_int), ("Sq", ctypes.c_int),
                ("Skv", ctypes.c_int), ("D", ctypes.c_int), ("scale", ctypes.c_float),
                ("mask", MaskSpec), ("deterministic", ctypes.c_int), ("status", ctypes.c_void_p)]


class DecodeParams(ctypes.Structure):
    _fields_ = [("q", ctypes.c_void_p), ("q_stride", c_i64x2),
                ("k_cache", ctypes.c_void_p), ("v_cache", ctypes.c_void_p), ("cache_stride", c_i64x3),
                ("block_table", ctypes.c_void_p), ("block_table_stride", ctypes.c_int),
                ("cache_seqlens", ctypes.c_void_p),
                ("B", ctypes.c_int), ("Hq", ctypes.c_int), ("Hkv", ctypes.c_int), ("D", ctypes.c_int),
                ("page_size", ctypes.c_int), ("num_pages", ctypes.c_int), ("max_seqlen", ctypes.c_int),
                ("scale", ctypes.c_float), ("mod", ctypes.c_int), ("softcap", ctypes.c_float),
                ("alibi_slopes", ctypes.c_void_p), ("alibi_batch_stride", ctypes.c_int),
                ("num_splits", ctypes.c_int),
                ("o", ctypes.c_void_p), ("o_stride", c_i64x2), ("lse", ctypes.c_void_p),
                ("status", ctypes.c_void_p),
                ("q_len", ctypes.c_int), ("q_token_stride", ctypes.c_int64), ("o_token_stride", ctypes.c_int64),
                ("causal", ctypes.c_int), ("cache_batch_idx", ctypes.c_void_p)]


class KvUpdateParams(ctypes.Structure):
    _fields_ = [("q", ctypes.c_void_p), ("q_stride", c_i64x3), ("q_out", ctypes.c_void_p), ("q_out_stride", c_i64x3),
                ("k_new", ctypes.c_void_p), ("v_new", ctypes.c_void_p), ("k_new_stride", c_i64x3),
                ("v_new_stride", c_i64x3), ("k_cache", ctypes.c_void_p), ("v_cache", ctypes.c_void_p),
                ("cache_stride", c_i64x3), ("block_table", ctypes.c_void_p), ("block_table_stride", ctypes.c_int),
                ("cache_batch_idx", ctypes.c_void_p), ("cache_seqlens", ctypes.c_void_p),
                ("seqlens_out", ctypes.c_void_p),
                ("B", ctypes.c_int), ("Snew", ctypes.c_int), ("Hq", ctypes.c_int), ("Hkv", ctypes.c_int),
                ("D", ctypes.c_int), ("page_size", ctypes.c_int), ("num_pages", ctypes.c_int),
                ("rotary_cos", ctypes.c_void_p), ("rotary_sin", ctypes.c_void_p), ("rotary_dim", ctypes.c_int),
                ("rotary_positions", ctypes.c_int), ("rotary_interleaved", ctypes.c_int),
                ("status", ctypes.c_void_p)]


_lock = threading.Lock()
_lib = None


def load() -> ctypes.CDLL:
    """Load libattn.so (built by exact_attention_145_b200.build). Raises if absent."""
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        path = lib_path()
        if not os.path.exists(path):
            raise RuntimeError(
                "%s is not built (expected at %s); run `python -m exact_attention_145_b200.build`"
                % (os.path.basename(path), path))
        lib = ctypes.CDLL(path)
        lib.attn_block_mask_bytes.argtypes = [ctypes.c_int] * 6
        lib.attn_block_mask_bytes.restype = ctypes.c_size_t
        lib.attn_block_mask_layout.argtypes = [ctypes.c_void_p, ctypes.c_size_t] + [ctypes.c_int] * 6 + [
            ctypes.POINTER(BlockMaskC)]
        lib.attn_block_mask_layout.restype = ctypes.c_int
        lib.attn_build_block_mask.argtypes = [ctypes.POINTER(MaskSpec), ctypes.POINTER(BlockMaskC), ctypes.c_void_p]
        lib.attn_build_block_mask.restype = ctypes.c_int
        lib.attn_fwd.argtypes = [ctypes.POINTER(FwdParams), ctypes.c_void_p]
        lib.attn_fwd.restype = ctypes.c_int
        lib.attn_decode_num_splits.argtypes = [ctypes.c_int] * 5
        lib.attn_decode_num_splits.restype = ctypes.c_int
        lib.attn_decode_workspace_bytes.argtypes = [ctypes.c_int] * 4
        lib.attn_decode_workspace_bytes.restype = ctypes.c_size_t
        lib.attn_decode.argtypes = [ctypes.POINTER(DecodeParams), ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p]
        lib.attn_decode.restype = ctypes.c_int
        lib.attn_decode_noalloc.argtypes = [ctypes.POINTER(DecodeParams), ctypes.c_void_p]
        lib.attn_decode_noalloc.restype = ctypes.c_int
        lib.attn_bwd_workspace_bytes.argtypes = [ctypes.POINTER(BwdParams)]
        lib.attn_bwd_workspace_bytes.restype = ctypes.c_size_t
        lib.attn_bwd.argtypes = [ctypes.POINTER(BwdParams), ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p]
        lib.attn_bwd.restype = ctypes.c_int
        lib.attn_kvcache_update.argtypes = [ctypes.POINTER(KvUpdateParams), ctypes.c_void_p]
        lib.attn_kvcache_update.restype = ctypes.c_int
        lib.attn_lse_combine.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                         ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p, ctypes.c_void_p]
        lib.attn_lse_combine.restype = ctypes.c_int
        lib.attn_selftest_wait_timeout.argtypes = [ctypes.c_void_p, ctypes.c_void_p]
        lib.attn_selftest_wait_timeout.restype = ctypes.c_int
        if hasattr(lib, "attn_trace_configure"):
            lib.attn_trace_configure.argtypes = [ctypes.c_void_p, ctypes.c_int]
            lib.attn_trace_configure.restype = ctypes.c_int
        lib.attn_status_str.argtypes = [ctypes.c_int]
        lib.attn_status_str.restype = ctypes.c_char_p
        _lib = lib
        return lib


class AttnError(RuntimeError):
    def __init__(self, code: int, what: str):
        self.code = code
        super().__init__("%s failed: %s (status %d)" % (what, load().attn_status_str(code).decode(), code))


def check(code: int, what: str) -> None:
    if code != ATTN_OK:
        raise AttnError(code, what)
