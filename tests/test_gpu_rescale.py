"""Parity where the running row max keeps growing: some keys are scaled by
exact powers of two, so a tile's (or half tile's) max exceeds the row's
reference by far more than the rescale threshold. This drives the paths that
redo P against the new max and rescale O: within a tile (first-chunk guess
too low), across tiles, in the whole-tile schedule (no score mod, decode)
and in the half-tile schedule (softcap), and with ALiBi."""
import numpy as np
import pytest

import oracle
import workloads as W
from tests._gpu_util import compare, dev_bf16, host_f64

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

import exact_attention_145_b200 as ea  # noqa: E402


def scale_rows(bits: np.ndarray, axis: int, ranges) -> np.ndarray:
    """bf16 bit patterns with the rows [lo, hi) along `axis` multiplied by a
    power of two (exact in bf16)."""
    x = W.bf16_bits_to_f64(bits)
    for lo, hi, f in ranges:
        sl = [slice(None)] * x.ndim
        sl[axis] = slice(lo, hi)
        x[tuple(sl)] *= f
    return W.f32_to_bf16_bits(x.astype(np.float32))


def prefill_case(Sq, Skv, Hq, Hkv, D, seed, ranges, **kw):
    q = W.normal_bf16(seed, (1, Sq, Hq, D))
    k = scale_rows(W.normal_bf16(seed + 1, (1, Skv, Hkv, D)), 1, ranges)
    v = W.normal_bf16(seed + 2, (1, Skv, Hkv, D))
    okw = {}
    if kw.get("causal"):
        okw.update(mask=W.MASK_CAUSAL, window=(-1, 0))
    if kw.get("window") is not None:
        okw.update(mask=W.MASK_WINDOW, window=kw["window"])
    if kw.get("softcap") is not None:
        okw.update(mod=W.MOD_SOFTCAP, softcap=kw["softcap"])
    alibi = kw.pop("alibi_np", None)
    if alibi is not None:
        okw.update(mod=W.MOD_ALIBI, alibi=alibi)
        kw["alibi_slopes"] = torch.from_numpy(alibi).cuda()
    o_ref, lse_ref = oracle.attn(q, k, v, **okw)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    o, lse = ea.attn_fwd(dev_bf16(q), dev_bf16(k), dev_bf16(v), status=status, **kw)
    torch.cuda.synchronize()
    assert status.item() == 0
    compare(host_f64(o), o_ref, lse.cpu().numpy().astype(np.float64), lse_ref, "rescale %s" % (kw,))


GROWING = [(40, 64, 8.0), (300, 340, 16.0), (650, 700, 32.0)]


def test_growing_max_no_mask_cross_lengths():
    prefill_case(300, 700, 4, 2, 128, 201, GROWING)


def test_growing_max_causal():
    prefill_case(700, 700, 4, 2, 128, 211, GROWING, causal=True)


def test_growing_max_head_dim_64():
    prefill_case(400, 700, 2, 2, 64, 221, GROWING)


def test_growing_max_softcap_half_tiles():
    prefill_case(700, 700, 4, 2, 128, 231, GROWING, softcap=30.0, window=(1023, 0))


def test_growing_max_alibi():
    # ALiBi tiles are walked from the diagonal back; the max still grows here
    prefill_case(700, 700, 4, 2, 128, 235, GROWING, causal=True, alibi_np=W.alibi_slopes(4))
    prefill_case(500, 900, 4, 1, 64, 236, GROWING, alibi_np=W.alibi_slopes(4))


def test_growing_max_decode():
    w = W.Decode("g", B=3, Hq=16, Hkv=2, D=128, kv_len=1500, page_size=64, seed=241)
    d = W.make_decode_inputs(w)
    num_pages = d["k_cache"].shape[0]
    ranges = [(p, p + 1, 16.0) for p in range(0, num_pages, 3)]
    d["k_cache"] = scale_rows(d["k_cache"], 0, ranges)
    o_ref, lse_ref = oracle.decode(d["q"], d["k_cache"], d["v_cache"], d["block_table"], d["cache_seqlens"])
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    o, lse = ea.attn_decode(dev_bf16(d["q"]), dev_bf16(d["k_cache"]), dev_bf16(d["v_cache"]),
                            torch.from_numpy(d["block_table"]).cuda(), torch.from_numpy(d["cache_seqlens"]).cuda(),
                            status=status)
    torch.cuda.synchronize()
    assert status.item() == 0
    compare(host_f64(o), o_ref, lse.cpu().numpy().astype(np.float64), lse_ref, "rescale decode")
