"""CPU-only checks of the C ABI: the library loads, exports every function
include/attn.h declares, and its host-side logic (sizes, layouts, argument
checks that return before any CUDA call) behaves as documented."""
import ctypes
import os
import re

import pytest

from exact_attention_145_b200 import _lib
from exact_attention_145_b200.build import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "attn.h")


@pytest.fixture(scope="module")
def lib():
    build()
    return _lib.load()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(attn_[a-z_0-9]+)\s*\(", text)))


def test_header_declares_the_documented_entry_points():
    names = declared_functions()
    for n in ("attn_fwd", "attn_decode", "attn_build_block_mask", "attn_lse_combine"):
        assert n in names
    assert sorted(_lib.EXPORTS) == names


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name
        assert ctypes.cast(getattr(lib, name), ctypes.c_void_p).value


def test_selftest_rejects_a_null_status(lib):
    assert lib.attn_selftest_wait_timeout(None, None) == _lib.ATTN_ERR_INVALID_ARG


def test_status_strings(lib):
    assert lib.attn_status_str(0) == b"ok"
    assert lib.attn_status_str(4) == b"workspace too small"
    assert lib.attn_status_str(99) == b"unknown status"


def test_block_mask_sizes_and_layout(lib):
    n = lib.attn_block_mask_bytes(1, 1, 16384, 16384, 128, 128)
    assert n >= 128 * 128 * (1 + 4 + 4) + 2 * 128 * 4
    assert lib.attn_block_mask_bytes(1, 1, 0, 10, 128, 128) == 0
    assert lib.attn_block_mask_bytes(0, 1, 10, 10, 128, 128) == 0
    bm = _lib.BlockMaskC()
    base = 1 << 20  # host-side arithmetic only: the layout never dereferences
    assert lib.attn_block_mask_layout(base, n, 1, 1, 16384, 16384, 128, 128, ctypes.byref(bm)) == 0
    assert (bm.Bm, bm.Hm, bm.n_q_tiles, bm.n_kv_tiles) == (1, 1, 128, 128)
    ptrs = [bm.cls, bm.part_cnt, bm.full_cnt, bm.part_idx, bm.full_idx]
    assert all(p % 16 == 0 for p in ptrs) and ptrs == sorted(ptrs)
    assert bm.full_idx + 128 * 128 * 4 <= base + n
    assert lib.attn_block_mask_layout(base, n - 1, 1, 1, 16384, 16384, 128, 128, ctypes.byref(bm)) == \
        _lib.ATTN_ERR_WORKSPACE
    assert lib.attn_block_mask_layout(base + 4, n, 1, 1, 16384, 16384, 128, 128, ctypes.byref(bm)) == \
        _lib.ATTN_ERR_INVALID_ARG
    # per-batch and per-head slices: every table scales with Bm * Hm
    n6 = lib.attn_block_mask_bytes(2, 3, 1000, 700, 128, 128)
    assert lib.attn_block_mask_layout(base, n6, 2, 3, 1000, 700, 128, 128, ctypes.byref(bm)) == 0
    nq, nk = 8, 6
    assert bm.part_cnt - bm.cls >= 6 * nq * nk and bm.full_cnt - bm.part_cnt >= 6 * nq * 4
    assert bm.full_idx - bm.part_idx >= 6 * nq * nk * 4 and bm.full_idx + 6 * nq * nk * 4 <= base + n6


def test_decode_workspace_bytes(lib):
    n = lib.attn_decode_workspace_bytes(32, 128, 128, 16)
    rows = 32 * 128 * 16
    assert n >= rows * 128 * 4 + rows * 4
    assert lib.attn_decode_workspace_bytes(0, 128, 128, 16) == 0
    assert lib.attn_decode_num_splits(32, 128, 1, 32768, 5) == 5
    assert lib.attn_decode_num_splits(1, 8, 1, 100, 7) == 1  # never more splits than key tiles


def _bwd_params(B, Hq, Hkv, S, D, mask=_lib.MASK_CAUSAL):
    p = _lib.BwdParams()
    p.B, p.Hq, p.Hkv, p.Sq, p.Skv, p.D = B, Hq, Hkv, S, S, D
    p.mask.kind = mask
    p.mask.window_left = p.mask.window_right = -1
    return p


def test_bwd_workspace_plan_sizes(lib):
    # Without a GPU the library plans for 148 SMs. Causal B1 Hq32 Hkv8 S2048
    # D128: key tile t meets 16 - t query tiles x 4 heads = 4 (16 - t) steps,
    # 8 groups x 4 x 136 = 4352 steps, cap = ceil(4352 / (2 x 148)) = 15.
    # Pieces per tile ceil(4 (16 - t) / 15): 5, 4 x4, 3 x4, 2 x4, 1 x3 = 44,
    # of which 41 belong to split tiles (fp32 partial slots).
    delta = 32 * 2048 * 4
    pieces = 44 * 16 + 64            # 704 rounded up to 256
    tiles = 256                      # 16 x 8 rounded up to 256
    part = 8 * 41 * 2 * 128 * 128 * 4
    n = lib.attn_bwd_workspace_bytes(ctypes.byref(_bwd_params(1, 32, 8, 2048, 128)))
    assert n == delta + pieces + tiles + part
    # no mask, one key tile per group: 1 piece each, nothing split
    n = lib.attn_bwd_workspace_bytes(ctypes.byref(_bwd_params(2, 4, 4, 128, 64, _lib.MASK_NONE)))
    assert n == 2 * 4 * 128 * 4 + 256 + 256
    # unsupported: document mask, D = 96
    assert lib.attn_bwd_workspace_bytes(ctypes.byref(_bwd_params(1, 4, 4, 128, 64, _lib.MASK_DOCUMENT))) == 0
    assert lib.attn_bwd_workspace_bytes(ctypes.byref(_bwd_params(1, 4, 4, 128, 96))) == 0


def _fwd_params(**kw):
    p = _lib.FwdParams()
    p.q = p.k = p.v = p.o = 1 << 20
    p.B, p.Hq, p.Hkv, p.Sq, p.Skv, p.D = 1, 4, 2, 128, 128, 128
    for s in ("q_stride", "k_stride", "v_stride", "o_stride"):
        setattr(p, s, _lib.c_i64x3(128 * 4 * 128, 4 * 128, 128))
    for k, v in kw.items():
        setattr(p, k, v)
    return p


@pytest.mark.parametrize("kw,code", [
    (dict(D=96), _lib.ATTN_ERR_UNSUPPORTED),
    (dict(Hq=3), _lib.ATTN_ERR_INVALID_ARG),
    (dict(Hkv=0), _lib.ATTN_ERR_INVALID_ARG),
    (dict(q=0), _lib.ATTN_ERR_INVALID_ARG),
    (dict(q=(1 << 20) + 2), _lib.ATTN_ERR_UNSUPPORTED),
    (dict(mod=_lib.MOD_SOFTCAP, softcap=0.0), _lib.ATTN_ERR_INVALID_ARG),
    (dict(mod=_lib.MOD_ALIBI), _lib.ATTN_ERR_INVALID_ARG),
])
def test_fwd_argument_checks(lib, kw, code):
    assert lib.attn_fwd(ctypes.byref(_fwd_params(**kw)), None) == code


def test_fwd_bad_strides_and_document_mask(lib):
    p = _fwd_params()
    p.q_stride = _lib.c_i64x3(128 * 4 * 128, 4 * 128, 100)
    assert lib.attn_fwd(ctypes.byref(p), None) == _lib.ATTN_ERR_UNSUPPORTED
    # a zero stride is refused on a dimension longer than 1 (rows would alias) ...
    p = _fwd_params()
    p.o_stride = _lib.c_i64x3(128 * 4 * 128, 4 * 128, 0)  # 4 heads, head stride 0
    assert lib.attn_fwd(ctypes.byref(p), None) == _lib.ATTN_ERR_UNSUPPORTED
    p = _fwd_params()
    p.k_stride = _lib.c_i64x3(128 * 2 * 128, 0, 128)  # 128 keys, sequence stride 0
    assert lib.attn_fwd(ctypes.byref(p), None) == _lib.ATTN_ERR_UNSUPPORTED
    p = _fwd_params()
    p.mask.kind = _lib.MASK_DOCUMENT  # no doc ids, no block mask
    assert lib.attn_fwd(ctypes.byref(p), None) == _lib.ATTN_ERR_INVALID_ARG
    # a block mask whose batch / head slices match neither 1 nor the call's B / Hq
    bm = _lib.BlockMaskC()
    nb = lib.attn_block_mask_bytes(3, 1, 128, 128, 128, 128)
    assert lib.attn_block_mask_layout(1 << 20, nb, 3, 1, 128, 128, 128, 128, ctypes.byref(bm)) == 0
    p = _fwd_params()
    p.block_mask = ctypes.pointer(bm)
    assert lib.attn_fwd(ctypes.byref(p), None) == _lib.ATTN_ERR_INVALID_ARG
    # document rows must be 16-byte strided
    p = _fwd_params()
    p.mask.kind, p.mask.doc_id, p.mask.doc_batch_stride = _lib.MASK_DOCUMENT, 1 << 20, 130
    nb = lib.attn_block_mask_bytes(1, 1, 128, 128, 128, 128)
    assert lib.attn_block_mask_layout(1 << 20, nb, 1, 1, 128, 128, 128, 128, ctypes.byref(bm)) == 0
    p.block_mask = ctypes.pointer(bm)
    assert lib.attn_fwd(ctypes.byref(p), None) == _lib.ATTN_ERR_UNSUPPORTED
    assert lib.attn_fwd(None, None) == _lib.ATTN_ERR_INVALID_ARG
    assert lib.attn_fwd(ctypes.byref(_fwd_params(B=0)), None) == _lib.ATTN_OK  # empty batch: nothing to do


def test_decode_argument_checks(lib):
    p = _lib.DecodeParams()
    p.B, p.Hq, p.Hkv, p.D, p.page_size, p.num_pages = 2, 256, 1, 128, 256, 10
    assert lib.attn_decode(ctypes.byref(p), None, 0, None) == _lib.ATTN_ERR_UNSUPPORTED  # group of 256 heads
    p.Hq = 8
    p.page_size = 48
    p.block_table = 1 << 20  # the page-size rule binds paged caches only
    assert lib.attn_decode(ctypes.byref(p), None, 0, None) == _lib.ATTN_ERR_UNSUPPORTED
    p.q_len, p.Hq = 33, 32   # 33 tokens x a group of 4 heads > 128 MMA rows
    assert lib.attn_decode(ctypes.byref(p), None, 0, None) == _lib.ATTN_ERR_UNSUPPORTED
    p.q_len, p.Hq = 0, 8
    p.page_size = 256
    assert lib.attn_decode(ctypes.byref(p), None, 0, None) == _lib.ATTN_ERR_INVALID_ARG  # null pointers
    assert lib.attn_lse_combine(None, None, 4, 0, 128, None, 128, None, None) == _lib.ATTN_ERR_INVALID_ARG
    assert lib.attn_lse_combine(None, None, 4, 2, 96, None, 128, None, None) == _lib.ATTN_ERR_UNSUPPORTED


def test_product_path_has_no_fallback(monkeypatch, tmp_path):
    monkeypatch.setattr(_lib, "LIB_PATH", str(tmp_path / "missing.so"))
    monkeypatch.setattr(_lib, "_lib", None)
    with pytest.raises(RuntimeError):
        _lib.load()
