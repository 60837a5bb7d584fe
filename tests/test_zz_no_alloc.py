"""attn_decode_noalloc: the paged decode for callers that cannot allocate
device memory (its split partials live in a fixed array inside the library).
Called through the C ABI and checked against attn_decode, which takes a
caller-allocated workspace, and against the fp64 oracle, on two calls in a
row with different inputs, score mods and group sizes.
This file is collected last on purpose."""
import ctypes

import numpy as np
import pytest

import oracle
import workloads as W
from tests._gpu_util import O_MAX_ERR, O_MEAN_ERR, LSE_MAX_ERR, compare, dev_bf16, host_f64

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

import exact_attention_145_b200 as ea  # noqa: E402
from exact_attention_145_b200 import _lib  # noqa: E402


def decode_params(q, kc, vc, bt, sl, o, lse, max_seqlen, mod=0, softcap=0.0, alibi=None):
    p = _lib.DecodeParams()
    p.q = q.data_ptr()
    p.q_stride = _lib.c_i64x2(q.stride(0), q.stride(1))
    p.k_cache, p.v_cache = kc.data_ptr(), vc.data_ptr()
    p.cache_stride = _lib.c_i64x3(*kc.stride()[:3])
    p.block_table, p.block_table_stride = bt.data_ptr(), bt.stride(0)
    p.cache_seqlens = sl.data_ptr()
    p.B, p.Hq, p.D = q.shape
    p.num_pages, p.page_size, p.Hkv = kc.shape[0], kc.shape[1], kc.shape[2]
    p.max_seqlen = max_seqlen
    p.mod, p.softcap = mod, softcap
    p.alibi_slopes = None if alibi is None else alibi.data_ptr()
    p.o = o.data_ptr()
    p.o_stride = _lib.c_i64x2(o.stride(0), o.stride(1))
    p.lse = lse.data_ptr()
    return p


def inputs(B, Hq, Hkv, kv_len, page, seed, seqlens):
    w = W.Decode("noalloc", B=B, Hq=Hq, Hkv=Hkv, D=128, kv_len=kv_len, page_size=page, seed=seed)
    d = W.make_decode_inputs(w, seqlens=np.array(seqlens, np.int32))
    q = dev_bf16(d["q"])[:, 0]
    return d, (q, dev_bf16(d["k_cache"]), dev_bf16(d["v_cache"]), torch.from_numpy(d["block_table"]).cuda(),
               torch.from_numpy(d["cache_seqlens"]).cuda())


def test_noalloc_decode_matches_workspace_decode_and_oracle_on_two_calls():
    lib = _lib.load()
    stream = torch.cuda.current_stream().cuda_stream
    cases = [dict(B=4, Hq=128, Hkv=1, kv_len=3000, page=256, seed=501, seqlens=[3000, 1, 2047, 1500], mod="alibi"),
             dict(B=6, Hq=16, Hkv=2, kv_len=1200, page=64, seed=502, seqlens=[1200, 700, 5, 1200, 999, 64],
                  mod="softcap")]
    for c in cases:
        d, (q, kc, vc, bt, sl) = inputs(c["B"], c["Hq"], c["Hkv"], c["kv_len"], c["page"], c["seed"], c["seqlens"])
        if c["mod"] == "alibi":
            slopes = W.alibi_slopes(c["Hq"])
            kw, okw = dict(alibi_slopes=torch.from_numpy(slopes).cuda()), dict(mod=W.MOD_ALIBI, alibi=slopes)
            ckw = dict(mod=_lib.MOD_ALIBI, alibi=kw["alibi_slopes"])
        else:
            kw, okw = dict(softcap=7.0), dict(mod=W.MOD_SOFTCAP, softcap=7.0)
            ckw = dict(mod=_lib.MOD_SOFTCAP, softcap=7.0)
        o_ws, lse_ws = ea.attn_decode(q, kc, vc, bt, sl, max_seqlen=c["kv_len"], **kw)
        o = torch.full_like(o_ws, float("nan"))
        lse = torch.full_like(lse_ws, float("nan"))
        p = decode_params(q, kc, vc, bt, sl, o, lse, c["kv_len"], **ckw)
        assert lib.attn_decode_noalloc(ctypes.byref(p), stream) == _lib.ATTN_OK
        torch.cuda.synchronize()
        # against the entry point that takes a caller-allocated workspace
        err = (o.float() - o_ws.float()).abs()
        assert torch.isfinite(o.float()).all()
        assert err.max().item() <= O_MAX_ERR and err.mean().item() <= O_MEAN_ERR
        assert (lse - lse_ws).abs().max().item() <= LSE_MAX_ERR
        # and against the fp64 oracle
        o_ref, lse_ref = oracle.decode(d["q"], d["k_cache"], d["v_cache"], d["block_table"], d["cache_seqlens"],
                                       **okw)
        compare(host_f64(o), o_ref, lse.cpu().numpy().astype(np.float64), lse_ref, "noalloc %s" % c["mod"])


def test_noalloc_python_wrapper_passes_score_mods():
    d, (q, kc, vc, bt, sl) = inputs(2, 8, 2, 700, 64, 504, [700, 333])
    slopes = W.alibi_slopes(8)
    o = torch.empty((2, 8, 128), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((2, 8), dtype=torch.float32, device="cuda")
    ea.attn_decode_noalloc(q, kc, vc, bt, sl, o, lse, max_seqlen=700, alibi_slopes=torch.from_numpy(slopes).cuda())
    torch.cuda.synchronize()
    o_ref, lse_ref = oracle.decode(d["q"], d["k_cache"], d["v_cache"], d["block_table"], d["cache_seqlens"],
                                   mod=W.MOD_ALIBI, alibi=slopes)
    compare(host_f64(o), o_ref, lse.cpu().numpy().astype(np.float64), lse_ref, "noalloc wrapper alibi")


def test_noalloc_decode_refuses_calls_beyond_its_scratch():
    lib = _lib.load()
    B, Hq, D, splits = 64, 128, 128, 64
    assert lib.attn_decode_workspace_bytes(B, Hq, D, splits) > _lib.ATTN_DECODE_NOALLOC_MAX_BYTES
    _, (q, kc, vc, bt, sl) = inputs(2, 128, 1, 256, 256, 503, [256, 256])
    qb = q.repeat(32, 1, 1)  # B = 64
    btb = bt.repeat(32, 1)
    slb = sl.repeat(32)
    o = torch.empty((B, Hq, D), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((B, Hq), dtype=torch.float32, device="cuda")
    p = decode_params(qb, kc, vc, btb, slb, o, lse, 256 * splits)
    p.num_splits = splits
    p.block_table_stride = splits  # claims 64 pages per sequence; refused before any launch
    assert lib.attn_decode_noalloc(ctypes.byref(p), torch.cuda.current_stream().cuda_stream) == \
        _lib.ATTN_ERR_WORKSPACE
