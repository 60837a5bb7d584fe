"""GPU parity of the pointwise hook (the ReLU activation wrapper of the
FlexAttention + FlashAttention-4 talk) against the fp64 oracle, and of the
QKV-packed entry (flash_attn_qkvpacked_func, FlashAttention overview)
against attn_fwd on unpacked copies."""
import ctypes

import numpy as np
import pytest

import oracle
import workloads as W
from tests._gpu_util import LSE_MAX_ERR, dev_bf16, host_f64

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

import exact_attention_145_b200 as ea  # noqa: E402

# The activation output is an unnormalised sum of bf16-rounded weights times
# V, stored as bf16, so its error scales with the output's own size. Two
# roundings to bf16 (each weight, then O itself) each err by at most 2^-9 of
# the value: the mean error is bounded by 2 * 2^-9 of the mean magnitude, the
# max error by 1e-2 of the largest entry. The LSE slot is ln of the fp32 sum
# of the unrounded weights.
R_MAX_REL = 1e-2
R_MEAN_REL = 2 * 2.0 ** -9


def _relu_case(B, S, Hq, Hkv, D, seed, Skv=None, **mask):
    Skv = S if Skv is None else Skv
    q, k, v = (W.normal_bf16(seed, (B, S, Hq, D)), W.normal_bf16(seed + 1, (B, Skv, Hkv, D)),
               W.normal_bf16(seed + 2, (B, Skv, Hkv, D)))
    kw, okw = {}, {}
    if mask.get("causal"):
        kw["causal"] = True
        okw = dict(mask=oracle.MASK_CAUSAL, window=(-1, 0))
    elif mask.get("window"):
        kw["window"] = mask["window"]
        okw = dict(mask=oracle.MASK_WINDOW, window=mask["window"])
    elif mask.get("doc"):
        lens = mask["doc"]
        doc = W.doc_ids_from_lengths(lens)
        kw["doc_id"] = torch.from_numpy(doc).cuda()
        okw = dict(mask=oracle.MASK_DOCUMENT, doc_id=doc)
    o, lse = ea.attn_fwd(dev_bf16(q), dev_bf16(k), dev_bf16(v), activation="relu", **kw)
    torch.cuda.synchronize()
    ro, rl = oracle.attn(q, k, v, mod=oracle.MOD_RELU, **okw)
    og, lg = host_f64(o), lse.cpu().numpy().astype(np.float64)
    err = np.abs(og - ro)
    scale_max, scale_mean = max(np.abs(ro).max(), 1e-3), max(np.abs(ro).mean(), 1e-4)
    assert err.max() <= R_MAX_REL * scale_max, "relu O max err %.3e (ref max %.3e)" % (err.max(), scale_max)
    assert err.mean() <= R_MEAN_REL * scale_mean, "relu O mean err %.3e" % err.mean()
    fin = np.isfinite(rl)
    assert np.array_equal(np.isfinite(lg), fin)
    assert np.abs(lg[fin] - rl[fin]).max(initial=0.0) <= LSE_MAX_ERR


@pytest.mark.parametrize("D", [64, 128])
def test_relu_activation_no_mask_and_gqa(D):
    _relu_case(2, 300, 8, 2, D, seed=400 + D)


@pytest.mark.parametrize("S", [77, 128, 700])
def test_relu_activation_causal(S):
    _relu_case(1, S, 4, 4, 128, seed=410 + S, causal=True)


def test_relu_activation_window_and_documents():
    _relu_case(1, 900, 4, 2, 128, seed=420, window=(200, 0))
    _relu_case(1, 1000, 4, 1, 128, seed=421, doc=[300, 77, 500, 123])


def test_relu_activation_rejected_by_decode():
    q = torch.zeros((1, 8, 128), dtype=torch.bfloat16, device="cuda")
    kc = torch.zeros((2, 128, 1, 128), dtype=torch.bfloat16, device="cuda")
    bt = torch.zeros((1, 2), dtype=torch.int32, device="cuda")
    sl = torch.full((1,), 10, dtype=torch.int32, device="cuda")
    p, _ = ea._decode_params(q, kc, kc, bt, sl, 256, None, None, None, 0, None, None, None)
    p.mod = ea.MOD_RELU
    ea._set_out(p, q)
    assert ea.load_library().attn_decode(ctypes.byref(p), 0, 0, None) == ea._lib.ATTN_ERR_UNSUPPORTED


@pytest.mark.parametrize("causal", [False, True])
def test_qkv_packed_equals_unpacked(causal):
    B, S, H, D = 2, 333, 4, 128
    qkv = dev_bf16(W.normal_bf16(430, (B, S, 3, H, D)))
    o1, l1 = ea.attn_fwd_qkvpacked(qkv, causal=causal)
    o2, l2 = ea.attn_fwd(qkv[:, :, 0].contiguous(), qkv[:, :, 1].contiguous(), qkv[:, :, 2].contiguous(),
                         causal=causal)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_qkv_packed_gqa_layout():
    B, S, Hq, Hkv, D = 1, 500, 8, 2, 64
    qkv = dev_bf16(W.normal_bf16(431, (B, S, Hq + 2 * Hkv, D)))
    o1, l1 = ea.attn_fwd_qkvpacked(qkv, num_heads_q=Hq, causal=True)
    o2, l2 = ea.attn_fwd(qkv[:, :, :Hq].contiguous(), qkv[:, :, Hq:Hq + Hkv].contiguous(),
                         qkv[:, :, Hq + Hkv:].contiguous(), causal=True)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
