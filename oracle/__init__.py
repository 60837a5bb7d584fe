"""fp64 CPU oracle for exact attention forward (test infrastructure).

TEST INFRASTRUCTURE ONLY: the test suite, the package smoke check and the
benchmark's CPU-baseline leg are the only code allowed to import this package.
The CUDA product path never imports, links or calls it, and shares no code
with it. The arithmetic lives in ``oracle.c`` (plain C, double precision, one
materialised score row at a time); this module compiles it with gcc and
marshals numpy arrays into it.

Pins (tests/test_oracle.py): closed forms (one key, two keys, uniform scores
-> mean of V and LSE = ln(count)), constant V, causal row 0, GQA equal to the
repeat_kv-expanded MHA, mask counts and analytic tile classes, split
invariance of the LSE combine, paging invariance, the ALiBi slope sequence for
8 heads, and torch's fp64 CPU scaled_dot_product_attention on small cases.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading
from typing import Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

MASK_NONE, MASK_CAUSAL, MASK_WINDOW, MASK_DOCUMENT = 0, 1, 2, 3
MOD_NONE, MOD_SOFTCAP, MOD_ALIBI, MOD_RELU = 0, 1, 2, 3


def build(force: bool = False) -> str:
    """Compile oracle.c into liboracle.so (plain gcc, no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp.%d" % os.getpid()
        subprocess.check_call(["gcc", "-O2", "-fPIC", "-shared", "-std=c11", "-fno-fast-math", "-pthread",
                               "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


class _AttnArgs(ctypes.Structure):
    _fields_ = [
        ("q", ctypes.c_void_p), ("k", ctypes.c_void_p), ("v", ctypes.c_void_p),
        ("q_sb", ctypes.c_int64), ("q_ss", ctypes.c_int64), ("q_sh", ctypes.c_int64),
        ("k_sb", ctypes.c_int64), ("k_ss", ctypes.c_int64), ("k_sh", ctypes.c_int64),
        ("v_sb", ctypes.c_int64), ("v_ss", ctypes.c_int64), ("v_sh", ctypes.c_int64),
        ("B", ctypes.c_int), ("Hq", ctypes.c_int), ("Hkv", ctypes.c_int),
        ("Sq", ctypes.c_int), ("Skv", ctypes.c_int), ("D", ctypes.c_int),
        ("scale", ctypes.c_double),
        ("mask", ctypes.c_int), ("window_left", ctypes.c_int), ("window_right", ctypes.c_int),
        ("q_offset", ctypes.c_int),
        ("doc_id", ctypes.c_void_p), ("doc_bstride", ctypes.c_int64),
        ("mod", ctypes.c_int), ("softcap", ctypes.c_double),
        ("alibi", ctypes.c_void_p), ("alibi_bstride", ctypes.c_int64),
        ("kv_begin", ctypes.c_int), ("kv_end", ctypes.c_int),
    ]


class _DecodeArgs(ctypes.Structure):
    _fields_ = [
        ("q", ctypes.c_void_p), ("q_sb", ctypes.c_int64), ("q_sh", ctypes.c_int64),
        ("k_cache", ctypes.c_void_p), ("v_cache", ctypes.c_void_p),
        ("c_sp", ctypes.c_int64), ("c_ss", ctypes.c_int64), ("c_sh", ctypes.c_int64),
        ("block_table", ctypes.c_void_p), ("bt_stride", ctypes.c_int64), ("seqlens", ctypes.c_void_p),
        ("B", ctypes.c_int), ("Hq", ctypes.c_int), ("Hkv", ctypes.c_int), ("D", ctypes.c_int),
        ("page_size", ctypes.c_int), ("num_pages", ctypes.c_int),
        ("scale", ctypes.c_double), ("mod", ctypes.c_int), ("softcap", ctypes.c_double),
        ("alibi", ctypes.c_void_p), ("alibi_bstride", ctypes.c_int64),
    ]


class _F64Args(ctypes.Structure):
    _fields_ = [
        ("q", ctypes.c_void_p), ("k", ctypes.c_void_p), ("v", ctypes.c_void_p), ("dout", ctypes.c_void_p),
        ("q_sb", ctypes.c_int64), ("q_ss", ctypes.c_int64), ("q_sh", ctypes.c_int64),
        ("k_sb", ctypes.c_int64), ("k_ss", ctypes.c_int64), ("k_sh", ctypes.c_int64),
        ("v_sb", ctypes.c_int64), ("v_ss", ctypes.c_int64), ("v_sh", ctypes.c_int64),
        ("B", ctypes.c_int), ("Hq", ctypes.c_int), ("Hkv", ctypes.c_int),
        ("Sq", ctypes.c_int), ("Skv", ctypes.c_int), ("D", ctypes.c_int),
        ("scale", ctypes.c_double),
        ("mask", ctypes.c_int), ("window_left", ctypes.c_int), ("window_right", ctypes.c_int),
        ("q_offset", ctypes.c_int),
        ("doc_id", ctypes.c_void_p), ("doc_bstride", ctypes.c_int64),
        ("mod", ctypes.c_int), ("softcap", ctypes.c_double),
        ("alibi", ctypes.c_void_p), ("alibi_bstride", ctypes.c_int64),
    ]


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            lib.oracle_attn.argtypes = [ctypes.POINTER(_AttnArgs), ctypes.c_void_p, ctypes.c_int64,
                                        ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int]
            lib.oracle_attn.restype = ctypes.c_int
            lib.oracle_decode.argtypes = [ctypes.POINTER(_DecodeArgs), ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int]
            lib.oracle_decode.restype = ctypes.c_int
            lib.oracle_lse_combine.argtypes = [ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int,
                                               ctypes.c_void_p, ctypes.c_void_p]
            lib.oracle_lse_combine.restype = None
            lib.oracle_block_mask.argtypes = [ctypes.c_int] * 4 + [ctypes.c_void_p] + [ctypes.c_int] * 4 + \
                [ctypes.c_void_p] * 5
            lib.oracle_block_mask.restype = ctypes.c_int
            lib.oracle_count_pairs.argtypes = [ctypes.c_int] * 4 + [ctypes.c_void_p] + [ctypes.c_int] * 2
            lib.oracle_count_pairs.restype = ctypes.c_int64
            lib.oracle_attn_f64.argtypes = [ctypes.POINTER(_F64Args), ctypes.c_void_p, ctypes.c_void_p]
            lib.oracle_attn_f64.restype = ctypes.c_int
            lib.oracle_attn_bwd_f64.argtypes = [ctypes.POINTER(_F64Args), ctypes.c_void_p, ctypes.c_void_p,
                                                ctypes.c_void_p, ctypes.c_int]
            lib.oracle_attn_bwd_f64.restype = ctypes.c_int
            _lib = lib
    return _lib


def _ptr(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data


def default_threads() -> int:
    return os.cpu_count() or 1


def attn(q, k, v, *, scale: Optional[float] = None, mask: int = MASK_NONE, window=(-1, -1), q_offset: int = 0,
         doc_id=None, mod: int = MOD_NONE, softcap: float = 0.0, alibi=None, rows=None, kv_range=None,
         nthreads: Optional[int] = None):
    """Exact attention forward in fp64.

    q: uint16 bf16 bits [B, Sq, Hq, D]; k, v: [B, Skv, Hkv, D] (any strides,
    last dim contiguous). doc_id: [S] (shared by every batch) or [B, S].
    rows: optional int array [n, 3] of (b, h, i).
    Returns (O, LSE): O float64 [B, Sq, Hq, D] and LSE [B, Hq, Sq] for all rows,
    or O [n, D] and LSE [n] for the given rows.
    """
    lib = _load()
    for t in (q, k, v):
        assert t.dtype == np.uint16 and t.ndim == 4 and t.strides[3] == 2
    B, Sq, Hq, D = q.shape
    Skv, Hkv = k.shape[1], k.shape[2]
    a = _AttnArgs()
    a.q, a.k, a.v = q.ctypes.data, k.ctypes.data, v.ctypes.data
    a.q_sb, a.q_ss, a.q_sh = (s // 2 for s in q.strides[:3])
    a.k_sb, a.k_ss, a.k_sh = (s // 2 for s in k.strides[:3])
    a.v_sb, a.v_ss, a.v_sh = (s // 2 for s in v.strides[:3])
    a.B, a.Hq, a.Hkv, a.Sq, a.Skv, a.D = B, Hq, Hkv, Sq, Skv, D
    a.scale = (1.0 / np.sqrt(D)) if scale is None else float(scale)
    a.mask, a.window_left, a.window_right, a.q_offset = mask, int(window[0]), int(window[1]), q_offset
    doc = None if doc_id is None else np.ascontiguousarray(doc_id, dtype=np.int32)
    a.doc_id = _ptr(doc)
    # doc_id [S]: one layout for every batch; [B, S]: row b for batch b
    a.doc_bstride = doc.shape[1] if doc is not None and doc.ndim == 2 else 0
    a.mod, a.softcap = mod, float(softcap)
    al = None
    if alibi is not None:
        al = np.ascontiguousarray(alibi, dtype=np.float32)
        a.alibi_bstride = Hq if al.ndim == 2 else 0
    a.alibi = _ptr(al)
    a.kv_begin, a.kv_end = (0, Skv) if kv_range is None else (int(kv_range[0]), int(kv_range[1]))
    nt = default_threads() if nthreads is None else nthreads
    if rows is None:
        n = B * Hq * Sq
        o = np.empty((n, D), dtype=np.float64)
        lse = np.empty(n, dtype=np.float64)
        rc = lib.oracle_attn(ctypes.byref(a), None, n, o.ctypes.data, lse.ctypes.data, nt)
        if rc != 0:
            raise ValueError("oracle_attn: bad arguments")
        return o.reshape(B, Hq, Sq, D).transpose(0, 2, 1, 3).copy(), lse.reshape(B, Hq, Sq)
    r = np.ascontiguousarray(rows, dtype=np.int32).reshape(-1, 3)
    n = r.shape[0]
    o = np.empty((n, D), dtype=np.float64)
    lse = np.empty(n, dtype=np.float64)
    rc = lib.oracle_attn(ctypes.byref(a), r.ctypes.data, n, o.ctypes.data, lse.ctypes.data, nt)
    if rc != 0:
        raise ValueError("oracle_attn: bad arguments")
    return o, lse


def decode(q, k_cache, v_cache, block_table, cache_seqlens, *, scale: Optional[float] = None, mod: int = MOD_NONE,
           softcap: float = 0.0, alibi=None, nthreads: Optional[int] = None):
    """Single-query attention over a paged KV cache, fp64.

    q: [B, 1, Hq, D] or [B, Hq, D] bf16 bits; k_cache/v_cache: [num_pages,
    page_size, Hkv, D]; block_table int32 [B, max_pages]; cache_seqlens int32 [B].
    Returns O float64 [B, Hq, D], LSE [B, Hq].
    """
    lib = _load()
    if q.ndim == 4:
        q = q[:, 0]
    B, Hq, D = q.shape
    P, page, Hkv, _ = k_cache.shape
    bt = np.ascontiguousarray(block_table, dtype=np.int32)
    sl = np.ascontiguousarray(cache_seqlens, dtype=np.int32)
    a = _DecodeArgs()
    a.q = q.ctypes.data
    a.q_sb, a.q_sh = q.strides[0] // 2, q.strides[1] // 2
    assert k_cache.strides == v_cache.strides
    a.k_cache, a.v_cache = k_cache.ctypes.data, v_cache.ctypes.data
    a.c_sp, a.c_ss, a.c_sh = (s // 2 for s in k_cache.strides[:3])
    a.block_table, a.bt_stride, a.seqlens = bt.ctypes.data, bt.shape[1], sl.ctypes.data
    a.B, a.Hq, a.Hkv, a.D, a.page_size, a.num_pages = B, Hq, Hkv, D, page, P
    a.scale = (1.0 / np.sqrt(D)) if scale is None else float(scale)
    a.mod, a.softcap = mod, float(softcap)
    al = None
    if alibi is not None:
        al = np.ascontiguousarray(alibi, dtype=np.float32)
        a.alibi_bstride = Hq if al.ndim == 2 else 0
    a.alibi = _ptr(al)
    o = np.empty((B, Hq, D), dtype=np.float64)
    lse = np.empty((B, Hq), dtype=np.float64)
    rc = lib.oracle_decode(ctypes.byref(a), o.ctypes.data, lse.ctypes.data,
                           default_threads() if nthreads is None else nthreads)
    if rc != 0:
        raise ValueError("oracle_decode: bad arguments or page id out of range")
    return o, lse


def lse_combine(lse_parts, o_parts):
    """Combine partial (LSE_i, O_i) over disjoint key sets. lse_parts [n], o_parts [n, D]."""
    lib = _load()
    lp = np.ascontiguousarray(lse_parts, dtype=np.float64)
    op = np.ascontiguousarray(o_parts, dtype=np.float64)
    D = op.shape[1]
    o = np.empty(D, dtype=np.float64)
    lse = np.empty(1, dtype=np.float64)
    lib.oracle_lse_combine(lp.shape[0], lp.ctypes.data, op.ctypes.data, D, o.ctypes.data, lse.ctypes.data)
    return o, float(lse[0])


def block_mask(mask: int, Sq: int, Skv: int, blk_q: int = 128, blk_kv: int = 128, window=(-1, -1),
               q_offset: int = 0, doc_id=None) -> dict:
    """Brute-force tile classification: dict(cls, part_cnt, part_idx, full_cnt, full_idx).

    The *_idx arrays are [nQ, nK] with entries past the count set to -1.
    """
    lib = _load()
    nQ, nK = -(-Sq // blk_q), -(-Skv // blk_kv)
    cls = np.zeros((nQ, nK), dtype=np.uint8)
    pc = np.zeros(nQ, dtype=np.int32)
    fc = np.zeros(nQ, dtype=np.int32)
    pi = np.full((nQ, nK), -1, dtype=np.int32)
    fi = np.full((nQ, nK), -1, dtype=np.int32)
    doc = None if doc_id is None else np.ascontiguousarray(doc_id, dtype=np.int32)
    rc = lib.oracle_block_mask(mask, int(window[0]), int(window[1]), q_offset, _ptr(doc), Sq, Skv, blk_q, blk_kv,
                               cls.ctypes.data, pc.ctypes.data, pi.ctypes.data, fc.ctypes.data, fi.ctypes.data)
    if rc != 0:
        raise ValueError("oracle_block_mask: bad arguments")
    return dict(cls=cls, part_cnt=pc, part_idx=pi, full_cnt=fc, full_idx=fi)


def count_pairs(mask: int, Sq: int, Skv: int, window=(-1, -1), q_offset: int = 0, doc_id=None) -> int:
    """Allowed (q, kv) pairs of one (batch, head) under the mask."""
    lib = _load()
    doc = None if doc_id is None else np.ascontiguousarray(doc_id, dtype=np.int32)
    return int(lib.oracle_count_pairs(mask, int(window[0]), int(window[1]), q_offset, _ptr(doc), Sq, Skv))


def _f64_args(q, k, v, dout, scale, mask, window, q_offset, doc_id, mod, softcap, alibi, keep):
    for t in (q, k, v) + (() if dout is None else (dout,)):
        assert t.dtype == np.float64 and t.ndim == 4 and t.strides[3] == 8
    B, Sq, Hq, D = q.shape
    Skv, Hkv = k.shape[1], k.shape[2]
    a = _F64Args()
    a.q, a.k, a.v = q.ctypes.data, k.ctypes.data, v.ctypes.data
    a.dout = None if dout is None else dout.ctypes.data
    if dout is not None:
        assert dout.shape == q.shape and dout.strides == q.strides
    a.q_sb, a.q_ss, a.q_sh = (x // 8 for x in q.strides[:3])
    a.k_sb, a.k_ss, a.k_sh = (x // 8 for x in k.strides[:3])
    a.v_sb, a.v_ss, a.v_sh = (x // 8 for x in v.strides[:3])
    a.B, a.Hq, a.Hkv, a.Sq, a.Skv, a.D = B, Hq, Hkv, Sq, Skv, D
    a.scale = (1.0 / np.sqrt(D)) if scale is None else float(scale)
    a.mask, a.window_left, a.window_right, a.q_offset = mask, int(window[0]), int(window[1]), q_offset
    doc = None if doc_id is None else np.ascontiguousarray(doc_id, dtype=np.int32)
    a.doc_id = _ptr(doc)
    a.doc_bstride = doc.shape[1] if doc is not None and doc.ndim == 2 else 0
    a.mod, a.softcap = mod, float(softcap)
    al = None
    if alibi is not None:
        al = np.ascontiguousarray(alibi, dtype=np.float32)
        a.alibi_bstride = Hq if al.ndim == 2 else 0
    a.alibi = _ptr(al)
    keep.extend([doc, al])
    return a


def attn_f64(q, k, v, *, scale: Optional[float] = None, mask: int = MASK_NONE, window=(-1, -1),
             q_offset: int = 0, doc_id=None, mod: int = MOD_NONE, softcap: float = 0.0, alibi=None):
    """The forward on float64 inputs [B, S, H, D] (no bf16 rounding): for
    finite-difference checks of the backward, and as the reference where the
    inputs are computed values (a rotated q, gathered cache rows).
    Returns (O [B, Sq, Hq, D], LSE [B, Hq, Sq])."""
    lib = _load()
    keep = []
    a = _f64_args(q, k, v, None, scale, mask, window, q_offset, doc_id, mod, softcap, alibi, keep)
    B, Sq, Hq, D = q.shape
    o = np.empty((B, Sq, Hq, D), dtype=np.float64)
    lse = np.empty((B, Hq, Sq), dtype=np.float64)
    if lib.oracle_attn_f64(ctypes.byref(a), o.ctypes.data, lse.ctypes.data) != 0:
        raise ValueError("oracle_attn_f64: bad arguments")
    return o, lse


def attn_bwd(q, k, v, dout, *, scale: Optional[float] = None, mask: int = MASK_NONE, window=(-1, -1),
             q_offset: int = 0, doc_id=None, mod: int = MOD_NONE, softcap: float = 0.0, alibi=None,
             nthreads: Optional[int] = None):
    """Gradients of the attention forward with respect to q, k, v for the
    upstream gradient dout = dL/dO, by the chain rule in fp64. Inputs are
    float64 [B, S, H, D] (widen bf16 bits with workloads.bf16_bits_to_f64).
    Returns (dq [B, Sq, Hq, D], dk [B, Skv, Hkv, D], dv [B, Skv, Hkv, D])."""
    lib = _load()
    keep = []
    a = _f64_args(q, k, v, dout, scale, mask, window, q_offset, doc_id, mod, softcap, alibi, keep)
    B, Sq, Hq, D = q.shape
    Skv, Hkv = k.shape[1], k.shape[2]
    dq = np.empty((B, Sq, Hq, D), dtype=np.float64)
    dk = np.empty((B, Skv, Hkv, D), dtype=np.float64)
    dv = np.empty((B, Skv, Hkv, D), dtype=np.float64)
    nt = default_threads() if nthreads is None else nthreads
    if lib.oracle_attn_bwd_f64(ctypes.byref(a), dq.ctypes.data, dk.ctypes.data, dv.ctypes.data, nt) != 0:
        raise ValueError("oracle_attn_bwd_f64: bad arguments")
    return dq, dk, dv


# ---------------------------------------------------------------- kv-cache update
# FlashAttention overview ("Examples", flash_attn_with_kvcache): new keys and
# values are written into the cache in place, and rotary embeddings
# (rotary_cos, rotary_sin, rotary_interleaved) are applied on the fly. The
# pages give only the argument list; the readings used here:
#  - the new tokens of sequence b take cache positions cache_seqlens[b] + i,
#    i = 0 .. Snew - 1, and their rotary position is that same cache position,
#    for q and for the new k alike; v is not rotated;
#  - the rotary tables hold cos / sin of angle j at each position, shape
#    [positions, rotary_dim / 2]; pair j of a head vector is (x[2j], x[2j+1])
#    when interleaved, else (x[j], x[j + rotary_dim / 2]); dims past
#    rotary_dim are left unchanged;
#  - a paged cache maps position p of sequence b to page
#    block_table[b][p // page_size], row p % page_size; a contiguous cache
#    [B_cache][S][Hkv][D] maps it to batch row cache_batch_idx[b] (or b).


def rotary(x, cos, sin, positions, interleaved: bool):
    """Rotates the first 2 * cos.shape[1] dims of x[..., t, h, :] by the angles at
    positions[..., t]: x float64 [B, T, H, D]; cos, sin float64 [P, R/2];
    positions int [B, T]. Returns a new float64 array."""
    x = np.array(x, dtype=np.float64, copy=True)
    half = cos.shape[1]
    c = cos[positions][:, :, None, :]  # [B, T, 1, R/2]
    s = sin[positions][:, :, None, :]
    if interleaved:
        a, b = x[..., 0:2 * half:2].copy(), x[..., 1:2 * half:2].copy()
        x[..., 0:2 * half:2] = a * c - b * s
        x[..., 1:2 * half:2] = a * s + b * c
    else:
        a, b = x[..., :half].copy(), x[..., half:2 * half].copy()
        x[..., :half] = a * c - b * s
        x[..., half:2 * half] = a * s + b * c
    return x


def cache_rows(B: int, Snew: int, cache_seqlens, block_table=None, page_size: int = 0, cache_batch_idx=None):
    """(page or batch row, slot) of every new token: arrays [B, Snew] each."""
    pos = np.asarray(cache_seqlens, dtype=np.int64)[:, None] + np.arange(Snew, dtype=np.int64)[None, :]
    if block_table is not None:
        bt = np.asarray(block_table, dtype=np.int64)
        return bt[np.arange(B)[:, None], pos // page_size], pos % page_size
    idx = np.arange(B) if cache_batch_idx is None else np.asarray(cache_batch_idx, dtype=np.int64)
    return np.broadcast_to(idx[:, None], pos.shape).copy(), pos


def kvcache_append(k_cache, v_cache, k_new, v_new, cache_seqlens, *, block_table=None, page_size: int = 0,
                   cache_batch_idx=None, rotary_cos=None, rotary_sin=None, interleaved: bool = True,
                   round_bf16=None):
    """Returns updated copies of k_cache / v_cache (float64, same shapes) with the
    new tokens written at their cache positions, k rotated when tables are
    given. round_bf16, when given, rounds the rotated k to the cache's storage
    type before it is stored (the update writes bf16)."""
    kc, vc = np.array(k_cache, dtype=np.float64, copy=True), np.array(v_cache, dtype=np.float64, copy=True)
    B, Snew = k_new.shape[0], k_new.shape[1]
    pos = np.asarray(cache_seqlens, dtype=np.int64)[:, None] + np.arange(Snew, dtype=np.int64)[None, :]
    k = np.asarray(k_new, dtype=np.float64)
    if rotary_cos is not None:
        k = rotary(k, rotary_cos, rotary_sin, pos, interleaved)
    if round_bf16 is not None:
        k = round_bf16(k)
    row, slot = cache_rows(B, Snew, cache_seqlens, block_table, page_size, cache_batch_idx)
    for b in range(B):
        for i in range(Snew):
            kc[row[b, i], slot[b, i]] = k[b, i]
            vc[row[b, i], slot[b, i]] = v_new[b, i]
    return kc, vc
