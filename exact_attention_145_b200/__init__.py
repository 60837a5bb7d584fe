"""Exact attention forward on B200 (sm_100a): Python binding of libattn.

Every function here only marshals arguments into the C ABI of
include/attn.h (pointers, sizes, strides, the current CUDA stream). All of
the computation runs in the library's CUDA kernels; PyTorch supplies device
memory and streams. There is no CPU or PyTorch fallback: if libattn.so is
missing or a call fails, an exception is raised.

Entry points (same names as the C ABI):
  attn_fwd(q, k, v, ...)            prefill / full-sequence forward -> (O, LSE)
  attn_decode(q, k_cache, ...)      split-KV paged decode          -> (O, LSE)
  attn_build_block_mask(...)        FlexAttention-style block mask -> BlockMask
  attn_lse_combine(o_parts, ...)    merge split partial results    -> (O, LSE)
  attn_decode_noalloc(q, ...)       attn_decode for callers that cannot allocate
                                    device memory (scratch inside the library)
  attn_bwd(q, k, v, o, lse, dout)   backward of attn_fwd            -> (dQ, dK, dV)
"""
from __future__ import annotations

import ctypes
from typing import Optional, Tuple

from . import _lib
from ._lib import (ATTN_DEV_BAD_LEN, ATTN_DEV_BAD_MASK, ATTN_DEV_BAD_PAGE, ATTN_DEV_TIMEOUT, MASK_CAUSAL,
                   MASK_DOCUMENT, MASK_NONE, MASK_WINDOW,
                   MOD_ALIBI, MOD_NONE, MOD_RELU, MOD_SOFTCAP, AttnError)

__all__ = ["attn_fwd", "attn_fwd_qkvpacked", "attn_bwd", "attn_bwd_workspace_bytes", "attn_kvcache_update", "attn_with_kvcache", "attn_decode", "attn_decode_noalloc", "attn_build_block_mask", "attn_lse_combine",
           "BlockMask", "AttnError",
           "load_library", "ATTN_DEV_TIMEOUT", "ATTN_DEV_BAD_PAGE", "ATTN_DEV_BAD_LEN",
           "ATTN_DEV_BAD_MASK"]


def load_library():
    return _lib.load()


def _torch():
    import torch
    return torch


def _stream_handle(device) -> int:
    torch = _torch()
    return torch.cuda.current_stream(device).cuda_stream


def _ptr(t) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _check_bf16(name, t, ndim):
    torch = _torch()
    if t.dtype != torch.bfloat16:
        raise TypeError("%s must be bfloat16, got %s" % (name, t.dtype))
    if t.dim() != ndim:
        raise ValueError("%s must have %d dims, got %d" % (name, ndim, t.dim()))
    if not t.is_cuda:
        raise ValueError("%s must be a CUDA tensor" % name)
    if t.stride(-1) != 1:
        raise ValueError("%s: the head dimension must be contiguous" % name)


class BlockMask:
    """Tile-level mask (FlexAttention BlockMask equivalent) in one device buffer.

    cls[b, h, q_tile, kv_tile] is 0 (empty), 1 (partial) or 2 (full); part_idx /
    full_idx list the partial / full kv tiles of each (b, h, q tile) in
    ascending order, the first part_cnt / full_cnt entries of each row being
    valid. Bm / Hm of 1 mean one slice shared by every batch / head.
    """

    def __init__(self, Sq: int, Skv: int, blk_q: int, blk_kv: int, device, Bm: int = 1, Hm: int = 1):
        torch = _torch()
        lib = _lib.load()
        nbytes = lib.attn_block_mask_bytes(Bm, Hm, Sq, Skv, blk_q, blk_kv)
        if nbytes == 0:
            raise ValueError("invalid block mask sizes")
        self.buffer = torch.empty(nbytes, dtype=torch.uint8, device=device)
        self.c = _lib.BlockMaskC()
        _lib.check(lib.attn_block_mask_layout(self.buffer.data_ptr(), nbytes, Bm, Hm, Sq, Skv, blk_q, blk_kv,
                                              ctypes.byref(self.c)), "attn_block_mask_layout")
        self.Bm, self.Hm, self.Sq, self.Skv, self.blk_q, self.blk_kv = Bm, Hm, Sq, Skv, blk_q, blk_kv
        self.shape = (Bm, Hm, self.c.n_q_tiles, self.c.n_kv_tiles)

    def _view(self, addr, dtype, shape):
        torch = _torch()
        off = addr - self.buffer.data_ptr()
        n = 1
        for s in shape:
            n *= s
        esz = torch.empty((), dtype=dtype).element_size()
        return self.buffer[off:off + n * esz].view(dtype).view(*shape)

    @property
    def cls(self):
        return self._view(self.c.cls, _torch().uint8, self.shape)

    @property
    def part_cnt(self):
        return self._view(self.c.part_cnt, _torch().int32, self.shape[:3])

    @property
    def full_cnt(self):
        return self._view(self.c.full_cnt, _torch().int32, self.shape[:3])

    @property
    def part_idx(self):
        return self._view(self.c.part_idx, _torch().int32, self.shape)

    @property
    def full_idx(self):
        return self._view(self.c.full_idx, _torch().int32, self.shape)

    @property
    def row_order(self):
        """[Bm, n_q_tiles]: q-tiles by decreasing visited kv tiles (work order)."""
        return self._view(self.c.row_order, _torch().int32, (self.Bm, self.shape[2]))

    @property
    def doc_start(self):
        """[Bm, Sq]: first position of each position's run of equal document ids."""
        return self._view(self.c.doc_start, _torch().int32, (self.Bm, self.Sq))

    @property
    def doc_sorted(self):
        """[Bm]: 1 where the document ids never decrease."""
        return self._view(self.c.doc_sorted, _torch().int32, (self.Bm,))


def _doc_rows(doc_id):
    """(pointer, batch stride in elements) of a doc_id tensor [S] or [B, S]."""
    torch = _torch()
    if doc_id is None:
        return None, 0
    if doc_id.dtype != torch.int32 or not doc_id.is_cuda or doc_id.stride(-1) != 1 or doc_id.dim() not in (1, 2):
        raise ValueError("doc_id must be an int32 CUDA tensor [S] or [B, S] with contiguous rows")
    return doc_id.data_ptr(), (doc_id.stride(0) if doc_id.dim() == 2 else 0)


def _mask_spec(causal: bool, window, q_offset: int, doc_id) -> Tuple[_lib.MaskSpec, int]:
    spec = _lib.MaskSpec()
    wl, wr = (-1, -1) if window is None else (int(window[0]), int(window[1]))
    if doc_id is not None:
        kind = MASK_DOCUMENT
    elif causal:
        kind = MASK_CAUSAL
    elif (wl, wr) != (-1, -1):
        kind = MASK_WINDOW
    else:
        kind = MASK_NONE
    spec.kind, spec.window_left, spec.window_right, spec.q_offset = kind, wl, wr, int(q_offset)
    spec.doc_id, spec.doc_batch_stride = _doc_rows(doc_id)
    return spec, kind


def attn_build_block_mask(Sq: int, Skv: int, *, causal: bool = False, window=None, q_offset: int = 0,
                          doc_id=None, B: Optional[int] = None, H: int = 1, blk_q: int = 128, blk_kv: int = 128,
                          device=None, stream=None) -> BlockMask:
    """Classify every (batch, head, q-tile, kv-tile) of the mask on the device
    (FlexAttention create_block_mask(mask_mod, B, H, Q_LEN, KV_LEN, BLOCK_SIZE)).
    doc_id [S] gives one slice shared by every batch, [B, S] one slice per
    batch; B defaults to the rows of doc_id (1 otherwise) and H to 1 (shared by
    every head)."""
    torch = _torch()
    if doc_id is not None:
        _doc_rows(doc_id)
        device = doc_id.device
        if B is None:
            B = doc_id.shape[0] if doc_id.dim() == 2 else 1
        if doc_id.dim() == 2 and doc_id.shape[0] != B:
            raise ValueError("doc_id has %d rows but B = %d" % (doc_id.shape[0], B))
    B = 1 if B is None else int(B)
    device = device if device is not None else torch.device("cuda")
    bm = BlockMask(Sq, Skv, blk_q, blk_kv, device, Bm=B, Hm=int(H))
    spec, _ = _mask_spec(causal, window, q_offset, doc_id)
    h = _stream_handle(device) if stream is None else stream
    _lib.check(_lib.load().attn_build_block_mask(ctypes.byref(spec), ctypes.byref(bm.c), h),
               "attn_build_block_mask")
    bm._doc_id = doc_id
    return bm


def _mod_args(softcap, alibi_slopes, Hq, activation=None):
    torch = _torch()
    if sum(x is not None for x in (softcap, alibi_slopes, activation)) > 1:
        raise ValueError("choose one score mod: softcap, alibi_slopes or activation")
    if activation is not None:
        if activation != "relu":
            raise ValueError("activation must be 'relu'")
        return MOD_RELU, 0.0, None, 0
    if softcap is not None:
        return MOD_SOFTCAP, float(softcap), None, 0
    if alibi_slopes is not None:
        if alibi_slopes.dtype != torch.float32 or not alibi_slopes.is_cuda or not alibi_slopes.is_contiguous():
            raise ValueError("alibi_slopes must be a contiguous fp32 CUDA tensor")
        stride = 0 if alibi_slopes.dim() == 1 else Hq
        return MOD_ALIBI, 0.0, alibi_slopes.data_ptr(), stride
    return MOD_NONE, 0.0, None, 0


def attn_fwd(q, k, v, *, scale: Optional[float] = None, causal: bool = False, window=None, q_offset: int = 0,
             doc_id=None, block_mask: Optional[BlockMask] = None, softcap: Optional[float] = None,
             alibi_slopes=None, activation: Optional[str] = None, out=None, lse=None, status=None,
             with_lse: bool = True, stream=None):
    """Exact attention forward. q [B, Sq, Hq, D], k/v [B, Skv, Hkv, D] bf16 (any
    strides with a contiguous last dim, e.g. BHSD views). Returns (O, LSE):
    O bf16 [B, Sq, Hq, D] and LSE fp32 [B, Hq, Sq] (natural log).
    activation="relu" replaces the softmax by the activation wrapper:
    O = sum_j max(scale q.k_j, 0) v_j over allowed keys, LSE = ln of the weights' sum."""
    torch = _torch()
    _check_bf16("q", q, 4)
    _check_bf16("k", k, 4)
    _check_bf16("v", v, 4)
    B, Sq, Hq, D = q.shape
    Skv, Hkv = k.shape[1], k.shape[2]
    if out is None:
        out = torch.empty((B, Sq, Hq, D), dtype=torch.bfloat16, device=q.device)
    if lse is None and with_lse:
        lse = torch.empty((B, Hq, Sq), dtype=torch.float32, device=q.device)
    p = _lib.FwdParams()
    p.q, p.k, p.v, p.o = q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr()
    p.lse = _ptr(lse)
    p.q_stride = _lib.c_i64x3(*q.stride()[:3])
    p.k_stride = _lib.c_i64x3(*k.stride()[:3])
    p.v_stride = _lib.c_i64x3(*v.stride()[:3])
    p.o_stride = _lib.c_i64x3(*out.stride()[:3])
    p.B, p.Hq, p.Hkv, p.Sq, p.Skv, p.D = B, Hq, Hkv, Sq, Skv, D
    p.scale = 0.0 if scale is None else float(scale)
    spec, kind = _mask_spec(causal, window, q_offset, doc_id)
    p.mask = spec
    if kind == MASK_DOCUMENT and block_mask is None:
        block_mask = attn_build_block_mask(Sq, Skv, doc_id=doc_id, stream=stream)
    p.block_mask = ctypes.pointer(block_mask.c) if block_mask is not None else None
    p.mod, p.softcap, p.alibi_slopes, p.alibi_batch_stride = _mod_args(softcap, alibi_slopes, Hq, activation)
    p.status = _ptr(status)
    h = _stream_handle(q.device) if stream is None else stream
    _lib.check(_lib.load().attn_fwd(ctypes.byref(p), h), "attn_fwd")
    return out, lse


def attn_fwd_qkvpacked(qkv, *, num_heads_q: Optional[int] = None, **kw):
    """QKV-packed entry (flash_attn_qkvpacked_func, FlashAttention overview):
    qkv bf16 [B, S, 3, H, D] (Q, K, V of H heads each), or [B, S, Hq + 2 Hkv, D]
    with num_heads_q = Hq for packed GQA (the Q heads, then K, then V). The
    three operands are strided views of the one buffer, read in place by
    attn_fwd's tensor maps; keyword arguments are attn_fwd's."""
    if qkv.dim() == 5:
        if qkv.shape[2] != 3:
            raise ValueError("qkv [B, S, 3, H, D] expected")
        return attn_fwd(qkv[:, :, 0], qkv[:, :, 1], qkv[:, :, 2], **kw)
    if qkv.dim() != 4 or num_heads_q is None:
        raise ValueError("qkv [B, S, 3, H, D], or [B, S, Hq + 2 Hkv, D] with num_heads_q")
    Hq = int(num_heads_q)
    rest = qkv.shape[2] - Hq
    if rest <= 0 or rest % 2 != 0:
        raise ValueError("the packed head count must be num_heads_q + 2 Hkv")
    Hkv = rest // 2
    return attn_fwd(qkv[:, :, :Hq], qkv[:, :, Hq:Hq + Hkv], qkv[:, :, Hq + Hkv:], **kw)


def _bwd_params(q, k, v, out, lse, dout, dq, dk, dv, scale, causal, window, q_offset, deterministic, status):
    """Checks the backward inputs and fills the C parameter block."""
    torch = _torch()
    for name, t in (("q", q), ("k", k), ("v", v), ("out", out), ("dout", dout)):
        _check_bf16(name, t, 4)
    B, Sq, Hq, D = q.shape
    Skv, Hkv = k.shape[1], k.shape[2]
    if out.shape != q.shape or dout.shape != q.shape or v.shape != k.shape:
        raise ValueError("out and dout must be shaped like q, v like k")
    if lse is not None and (lse.dtype != torch.float32 or tuple(lse.shape) != (B, Hq, Sq) or not lse.is_contiguous()):
        raise ValueError("lse must be contiguous fp32 [B, Hq, Sq]")
    p = _lib.BwdParams()
    p.q, p.k, p.v, p.o, p.dout = q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), dout.data_ptr()
    p.lse = 0 if lse is None else lse.data_ptr()
    p.dq, p.dk, p.dv = (0 if t is None else t.data_ptr() for t in (dq, dk, dv))
    for name, t in (("q_stride", q), ("k_stride", k), ("v_stride", v), ("o_stride", out), ("do_stride", dout),
                    ("dq_stride", q if dq is None else dq), ("dk_stride", k if dk is None else dk),
                    ("dv_stride", v if dv is None else dv)):
        setattr(p, name, _lib.c_i64x3(*t.stride()[:3]))
    p.B, p.Hq, p.Hkv, p.Sq, p.Skv, p.D = B, Hq, Hkv, Sq, Skv, D
    p.scale = 0.0 if scale is None else float(scale)
    spec, _ = _mask_spec(causal, window, q_offset, None)
    p.mask = spec
    p.deterministic = 1 if deterministic else 0
    p.status = _ptr(status)
    return p


def attn_bwd_workspace_bytes(q, k, v, *, causal: bool = False, window=None, q_offset: int = 0) -> int:
    """Bytes of device workspace attn_bwd needs for these shapes and mask on
    the current device (the delta rows, the dK/dV plan and the fp32 partials
    of key tiles cut into pieces)."""
    p = _bwd_params(q, k, v, q, None, q, None, None, None, None, causal, window, q_offset, True, None)
    return int(_lib.load().attn_bwd_workspace_bytes(ctypes.byref(p)))


def attn_bwd(q, k, v, out, lse, dout, *, scale: Optional[float] = None, causal: bool = False, window=None,
             q_offset: int = 0, deterministic: bool = True, dq=None, dk=None, dv=None, workspace=None, status=None,
             stream=None):
    """Backward of attn_fwd: q [B, Sq, Hq, D], k/v [B, Skv, Hkv, D], the forward's
    out (O) and lse [B, Hq, Sq], and the upstream gradient dout (shaped like q),
    all bf16 except lse. Returns (dQ, dK, dV) shaped like q, k, v. Results are
    deterministic whatever `deterministic` says. `workspace` (uint8, device)
    needs attn_bwd_workspace_bytes(q, k, v, ...) bytes; allocated when None."""
    torch = _torch()
    if lse is None:
        raise ValueError("lse is required")
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    p = _bwd_params(q, k, v, out, lse, dout, dq, dk, dv, scale, causal, window, q_offset, deterministic, status)
    lib = _lib.load()
    if workspace is None:
        workspace = torch.empty(max(int(lib.attn_bwd_workspace_bytes(ctypes.byref(p))), 16), dtype=torch.uint8,
                                device=q.device)
    h = _stream_handle(q.device) if stream is None else stream
    _lib.check(lib.attn_bwd(ctypes.byref(p), workspace.data_ptr(), workspace.numel() * workspace.element_size(), h),
               "attn_bwd")
    return dq, dk, dv


def _decode_params(q, k_cache, v_cache, block_table, cache_seqlens, max_seqlen, scale, softcap, alibi_slopes,
                   num_splits, out, lse, status, causal=False, cache_batch_idx=None):
    """Checks the decode inputs and fills the C parameter block (shared by
    attn_decode and attn_decode_noalloc). q is [B, Hq, D] or [B, q_len, Hq, D];
    block_table None selects a contiguous cache [rows, positions, Hkv, D]."""
    torch = _torch()
    q_len = 1
    if q.dim() == 4:
        q_len = q.shape[1]
        if q_len == 1:
            q = q[:, 0]
    _check_bf16("q", q, 4 if q_len > 1 else 3)
    _check_bf16("k_cache", k_cache, 4)
    _check_bf16("v_cache", v_cache, 4)
    if k_cache.shape != v_cache.shape or k_cache.stride() != v_cache.stride():
        raise ValueError("k_cache and v_cache must share shape and strides")
    tables = [("cache_seqlens", cache_seqlens)]
    if block_table is not None:
        tables.append(("block_table", block_table))
    if cache_batch_idx is not None:
        tables.append(("cache_batch_idx", cache_batch_idx))
    for name, t in tables:
        if t.dtype != torch.int32 or not t.is_cuda or not t.is_contiguous():
            raise ValueError("%s must be a contiguous int32 CUDA tensor" % name)
    B, Hq, D = q.shape[0], q.shape[-2], q.shape[-1]
    P, page, Hkv, Dk = k_cache.shape
    if Dk != D or cache_seqlens.numel() != B or (block_table is not None and block_table.shape[0] != B):
        raise ValueError("q, caches, block_table and cache_seqlens disagree on B or D")
    if cache_batch_idx is not None and (block_table is not None or cache_batch_idx.numel() != B):
        raise ValueError("cache_batch_idx needs a contiguous cache (no block_table) and B entries")
    oshape = (B, Hq, D) if q_len == 1 else (B, q_len, Hq, D)
    if out is not None and (tuple(out.shape) != oshape or out.dtype != torch.bfloat16):
        raise ValueError("out must be bf16 %s" % (oshape,))
    lshape = (B, Hq) if q_len == 1 else (B, q_len, Hq)
    if lse is not None and (tuple(lse.shape) != lshape or lse.dtype != torch.float32 or not lse.is_contiguous()):
        raise ValueError("lse must be contiguous fp32 %s" % (lshape,))
    if max_seqlen is None:
        max_seqlen = block_table.shape[1] * page if block_table is not None else page
    p = _lib.DecodeParams()
    p.q = q.data_ptr()
    p.q_stride = _lib.c_i64x2(q.stride(0), q.stride(-2))
    p.q_len = q_len
    p.q_token_stride = q.stride(1) if q_len > 1 else 0
    p.causal = 1 if causal else 0
    p.k_cache, p.v_cache = k_cache.data_ptr(), v_cache.data_ptr()
    p.cache_stride = _lib.c_i64x3(*k_cache.stride()[:3])
    if block_table is not None:
        p.block_table, p.block_table_stride = block_table.data_ptr(), block_table.stride(0)
    p.cache_batch_idx = _ptr(cache_batch_idx)
    p.cache_seqlens = cache_seqlens.data_ptr()
    p.B, p.Hq, p.Hkv, p.D, p.page_size, p.num_pages = B, Hq, Hkv, D, page, P
    p.max_seqlen = int(max_seqlen)
    p.scale = 0.0 if scale is None else float(scale)
    p.mod, p.softcap, p.alibi_slopes, p.alibi_batch_stride = _mod_args(softcap, alibi_slopes, Hq)
    p.num_splits = int(num_splits)
    p.lse = _ptr(lse)
    p.status = _ptr(status)
    return p, q


def _set_out(p, out):
    p.o = out.data_ptr()
    p.o_stride = _lib.c_i64x2(out.stride(0), out.stride(-2))
    p.o_token_stride = out.stride(1) if p.q_len > 1 else 0


def attn_decode(q, k_cache, v_cache, block_table, cache_seqlens, *, max_seqlen: Optional[int] = None,
                scale: Optional[float] = None, softcap: Optional[float] = None, alibi_slopes=None,
                num_splits: int = 0, out=None, lse=None, workspace=None, status=None, with_lse: bool = True,
                causal: bool = False, cache_batch_idx=None, stream=None):
    """Split-KV decode over a KV cache. q [B, Hq, D], or [B, q_len, Hq, D] for
    several new tokens per sequence (they are the last q_len positions;
    `causal` masks each token's later keys); k_cache/v_cache
    [num_pages, page_size, Hkv, D] with block_table int32 [B, max_pages], or
    a contiguous cache [rows, positions, Hkv, D] with block_table None and
    optional cache_batch_idx int32 [B]; cache_seqlens int32 [B] counts every
    key, new tokens included. Returns O [B, Hq, D] for one token, else
    [B, q_len, Hq, D], and LSE [B, Hq] or [B, q_len, Hq]."""
    torch = _torch()
    B, Hq, D = (q.shape[0], q.shape[-2], q.shape[-1])
    q_len = q.shape[1] if q.dim() == 4 else 1
    if out is None:  # one token: [B, Hq, D] whether q came as [B, Hq, D] or [B, 1, Hq, D]
        out = torch.empty((B, Hq, D) if q_len == 1 else (B, q_len, Hq, D), dtype=torch.bfloat16, device=q.device)
    if lse is None and with_lse:
        lse = torch.empty((B, Hq) if q_len == 1 else (B, q_len, Hq), dtype=torch.float32, device=q.device)
    p, q = _decode_params(q, k_cache, v_cache, block_table, cache_seqlens, max_seqlen, scale, softcap,
                          alibi_slopes, num_splits, out, lse, status, causal, cache_batch_idx)
    lib = _lib.load()
    splits = lib.attn_decode_num_splits(p.B, p.Hq, p.Hkv, p.max_seqlen, p.num_splits)
    need = lib.attn_decode_workspace_bytes(p.B, p.Hq * p.q_len, p.D, splits)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    _set_out(p, out)
    h = _stream_handle(q.device) if stream is None else stream
    _lib.check(lib.attn_decode(ctypes.byref(p), workspace.data_ptr(), workspace.numel() * workspace.element_size(),
                               h), "attn_decode")
    return out, lse


def attn_decode_noalloc(q, k_cache, v_cache, block_table, cache_seqlens, out, lse, *, max_seqlen: int,
                        scale: Optional[float] = None, softcap: Optional[float] = None, alibi_slopes=None,
                        num_splits: int = 0, status=None, causal: bool = False, cache_batch_idx=None, stream=None):
    """attn_decode whose split partials live in a fixed 32 MiB array inside the
    library, for callers that may not allocate device memory (out and lse are
    the caller's). Calls that would need more scratch raise AttnError
    (workspace too small). The first call on a device should precede any
    stream capture; calls that overlap on the GPU share the array and race."""
    p, q = _decode_params(q, k_cache, v_cache, block_table, cache_seqlens, max_seqlen, scale, softcap,
                          alibi_slopes, num_splits, out, lse, status, causal, cache_batch_idx)
    _set_out(p, out)
    h = _stream_handle(q.device) if stream is None else stream
    _lib.check(_lib.load().attn_decode_noalloc(ctypes.byref(p), h), "attn_decode_noalloc")
    return out, lse


def attn_kvcache_update(k_cache, v_cache, cache_seqlens, *, q=None, q_out=None, k=None, v=None, block_table=None,
                        cache_batch_idx=None, rotary_cos=None, rotary_sin=None, rotary_interleaved: bool = True,
                        seqlens_out=None, status=None, stream=None):
    """In-place cache update of flash_attn_with_kvcache: k/v [B, Snew, Hkv, D]
    (k rotated) are written at positions cache_seqlens[b] + i of the paged
    (block_table) or contiguous (cache_batch_idx) cache, q [B, Snew, Hq, D]
    rotated at the same positions into q_out (allocated when None, may be q).
    rotary_cos / rotary_sin: fp32 [positions, rotary_dim / 2]. Returns q_out."""
    torch = _torch()
    _check_bf16("k_cache", k_cache, 4)
    _check_bf16("v_cache", v_cache, 4)
    if k_cache.shape != v_cache.shape or k_cache.stride() != v_cache.stride():
        raise ValueError("k_cache and v_cache must share shape and strides")
    P, page, Hkv, D = k_cache.shape
    ref = q if q is not None else k
    if ref is None:
        raise ValueError("nothing to update: give q and/or k, v")
    B, Snew = ref.shape[0], ref.shape[1]
    p = _lib.KvUpdateParams()
    if q is not None:
        _check_bf16("q", q, 4)
        if q_out is None:
            q_out = torch.empty_like(q)
        p.q, p.q_out = q.data_ptr(), q_out.data_ptr()
        p.q_stride, p.q_out_stride = _lib.c_i64x3(*q.stride()[:3]), _lib.c_i64x3(*q_out.stride()[:3])
        p.Hq = q.shape[2]
    else:
        p.q_stride = p.q_out_stride = _lib.c_i64x3(8, 8, 8)
    if (k is None) != (v is None):
        raise ValueError("give k and v together")
    if k is not None:
        _check_bf16("k", k, 4)
        _check_bf16("v", v, 4)
        p.k_new, p.v_new = k.data_ptr(), v.data_ptr()
        p.k_new_stride, p.v_new_stride = _lib.c_i64x3(*k.stride()[:3]), _lib.c_i64x3(*v.stride()[:3])
    else:
        p.k_new_stride = p.v_new_stride = _lib.c_i64x3(8, 8, 8)
    p.k_cache, p.v_cache = k_cache.data_ptr(), v_cache.data_ptr()
    p.cache_stride = _lib.c_i64x3(*k_cache.stride()[:3])
    if block_table is not None:
        p.block_table, p.block_table_stride = block_table.data_ptr(), block_table.stride(0)
    p.cache_batch_idx = _ptr(cache_batch_idx)
    p.cache_seqlens = cache_seqlens.data_ptr()
    p.seqlens_out = _ptr(seqlens_out)
    p.B, p.Snew, p.Hkv, p.D, p.page_size, p.num_pages = B, Snew, Hkv, D, page, P
    if rotary_cos is not None:
        if rotary_cos.dtype != torch.float32 or rotary_sin is None or rotary_sin.dtype != torch.float32:
            raise ValueError("rotary_cos / rotary_sin must be fp32 [positions, rotary_dim / 2]")
        if not (rotary_cos.is_contiguous() and rotary_sin.is_contiguous()) or rotary_cos.shape != rotary_sin.shape:
            raise ValueError("rotary tables must be contiguous and of one shape")
        p.rotary_cos, p.rotary_sin = rotary_cos.data_ptr(), rotary_sin.data_ptr()
        p.rotary_positions, p.rotary_dim = rotary_cos.shape[0], 2 * rotary_cos.shape[1]
    p.rotary_interleaved = 1 if rotary_interleaved else 0
    p.status = _ptr(status)
    h = _stream_handle(k_cache.device) if stream is None else stream
    _lib.check(_lib.load().attn_kvcache_update(ctypes.byref(p), h), "attn_kvcache_update")
    return q_out


def attn_with_kvcache(q, k_cache, v_cache, cache_seqlens, *, k=None, v=None, rotary_cos=None, rotary_sin=None,
                      cache_batch_idx=None, block_table=None, softmax_scale: Optional[float] = None,
                      causal: bool = False, rotary_interleaved: bool = True, alibi_slopes=None,
                      softcap: Optional[float] = None, num_splits: int = 0, max_seqlen: Optional[int] = None,
                      status=None, stream=None):
    """flash_attn_with_kvcache (FlashAttention overview, "Examples"): optional
    in-place append of k/v with rotary embedding (attn_kvcache_update), then
    attention of q [B, Sq, Hq, D] over each sequence's cache, the Sq new
    tokens at its last positions. Returns (O [B, Sq, Hq, D], LSE [B, Sq, Hq])."""
    torch = _torch()
    seqlens = cache_seqlens
    if k is not None or rotary_cos is not None:
        seqlens = torch.empty_like(cache_seqlens) if k is not None else cache_seqlens
        q = attn_kvcache_update(k_cache, v_cache, cache_seqlens, q=q, k=k, v=v, block_table=block_table,
                                cache_batch_idx=cache_batch_idx, rotary_cos=rotary_cos, rotary_sin=rotary_sin,
                                rotary_interleaved=rotary_interleaved,
                                seqlens_out=seqlens if k is not None else None, status=status, stream=stream)
    if max_seqlen is None:
        page = k_cache.shape[1]
        max_seqlen = block_table.shape[1] * page if block_table is not None else page
    return attn_decode(q, k_cache, v_cache, block_table, seqlens, max_seqlen=max_seqlen, scale=softmax_scale,
                       softcap=softcap, alibi_slopes=alibi_slopes, num_splits=num_splits, causal=causal,
                       cache_batch_idx=cache_batch_idx, status=status, stream=stream)


def attn_lse_combine(o_parts, lse_parts, *, out=None, lse=None, stream=None):
    """Merge split partials: o_parts fp32 [rows, n, D], lse_parts fp32 [rows, n]."""
    torch = _torch()
    rows, n, D = o_parts.shape
    if o_parts.dtype != torch.float32 or lse_parts.dtype != torch.float32:
        raise TypeError("partials must be fp32")
    if not (o_parts.is_contiguous() and lse_parts.is_contiguous()):
        raise ValueError("partials must be contiguous")
    if out is None:
        out = torch.empty((rows, D), dtype=torch.bfloat16, device=o_parts.device)
    if lse is None:
        lse = torch.empty((rows,), dtype=torch.float32, device=o_parts.device)
    h = _stream_handle(o_parts.device) if stream is None else stream
    _lib.check(_lib.load().attn_lse_combine(o_parts.data_ptr(), lse_parts.data_ptr(), rows, n, D, out.data_ptr(),
                                            out.stride(0), _ptr(lse), h), "attn_lse_combine")
    return out, lse
