"""GPU parity of the backward (attn_bwd through the C ABI) against the fp64
oracle's chain-rule backward on the same seeded inputs: masks, GQA/MQA,
ragged and cross lengths, rows with no allowed key, the full-size causal GQA
shape, and bit-identical results from run to run (the deterministic option)."""
import numpy as np
import pytest

import oracle
import workloads as W
from tests._gpu_util import dev_bf16, host_f64

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

import exact_attention_145_b200 as ea  # noqa: E402

# Gradients are bf16 outputs of bf16 products (P and dS are rounded to bf16
# before their MMAs), so errors scale with the gradient's own size: the max
# error is bounded relative to the largest reference entry and the mean error
# relative to the mean reference magnitude.
G_MAX_REL = 2e-2
G_MEAN_REL = 1e-2


def compare_grad(got, ref, what):
    err = np.abs(got - ref)
    assert np.isfinite(got).all(), "%s: non-finite" % what
    scale_max = max(float(np.abs(ref).max(initial=0.0)), 1e-3)
    scale_mean = max(float(np.abs(ref).mean()) if ref.size else 0.0, 1e-4)
    mx, mean = float(err.max(initial=0.0)), float(err.mean()) if err.size else 0.0
    assert mx <= G_MAX_REL * scale_max, "%s: max err %.3e (ref max %.3e)" % (what, mx, scale_max)
    assert mean <= G_MEAN_REL * scale_mean, "%s: mean err %.3e (ref mean %.3e)" % (what, mean, scale_mean)
    return mx / scale_max, mean / scale_mean


def bwd_case(B, Sq, Hq, Hkv, D, Skv=None, seed=1, causal=False, window=None, q_offset=0, scale=None):
    Skv = Sq if Skv is None else Skv
    q = W.normal_bf16(seed, (B, Sq, Hq, D))
    k = W.normal_bf16(seed + 1, (B, Skv, Hkv, D))
    v = W.normal_bf16(seed + 2, (B, Skv, Hkv, D))
    do = W.normal_bf16(seed + 3, (B, Sq, Hq, D))
    tq, tk, tv, tdo = dev_bf16(q), dev_bf16(k), dev_bf16(v), dev_bf16(do)
    kw = dict(causal=causal, window=window, q_offset=q_offset, scale=scale)
    o, lse = ea.attn_fwd(tq, tk, tv, **kw)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    dq, dk, dv = ea.attn_bwd(tq, tk, tv, o, lse, tdo, status=status, **kw)
    torch.cuda.synchronize()
    assert status.item() == 0
    okw = {}
    if causal:
        okw = dict(mask=W.MASK_CAUSAL, window=(-1, 0))
    elif window is not None:
        okw = dict(mask=W.MASK_WINDOW, window=window)
    if q_offset:
        okw["q_offset"] = q_offset
    f = W.bf16_bits_to_f64
    rq, rk, rv = oracle.attn_bwd(f(q), f(k), f(v), f(do), scale=scale, **okw)
    tag = str((B, Sq, Hq, Hkv, D, Skv, causal, window, q_offset))
    return [compare_grad(host_f64(x), r, n + " " + tag) for x, r, n in ((dq, rq, "dq"), (dk, rk, "dk"), (dv, rv, "dv"))]


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("Hq,Hkv", [(4, 4), (8, 2), (6, 1)])
def test_bwd_no_mask(Hq, Hkv, D):
    bwd_case(2, 300, Hq, Hkv, D, seed=200 + Hq + D)


@pytest.mark.parametrize("S", [1, 77, 128, 129, 500])
def test_bwd_causal_lengths(S):
    bwd_case(1, S, 4, 2, 128, seed=210 + S, causal=True)


def test_bwd_windows_and_offsets():
    bwd_case(1, 700, 4, 2, 128, seed=220, window=(100, 0))
    bwd_case(1, 600, 2, 2, 64, seed=221, window=(50, 30))
    bwd_case(1, 200, 4, 4, 128, Skv=650, seed=222, causal=True, q_offset=450)
    # the first 64 rows see no key: their dQ is 0 and they add nothing to dK, dV
    bwd_case(1, 300, 2, 2, 128, seed=223, causal=True, q_offset=-64)


def test_bwd_tiles_without_any_allowed_pair():
    # causal with a large negative offset: the first query tiles see no key and
    # the last key tiles are seen by no query; their gradients are exactly 0
    bwd_case(1, 500, 2, 1, 128, Skv=500, seed=235, causal=True, q_offset=-300)
    bwd_case(1, 300, 2, 2, 64, Skv=700, seed=236, window=(20, 0), q_offset=10)


def test_bwd_explicit_scale():
    bwd_case(1, 256, 2, 2, 128, seed=230, causal=True, scale=0.3)


def test_bwd_split_key_tiles():
    # small causal problems get a piece cap of 4 steps, so most key tiles are
    # cut into several pieces whose fp32 partials the reduction sums
    bwd_case(1, 1024, 8, 2, 128, seed=250, causal=True)
    bwd_case(2, 700, 4, 1, 64, seed=251, causal=True)
    bwd_case(1, 900, 6, 2, 128, Skv=1300, seed=252, window=(300, 40), q_offset=200)


def test_bwd_full_size_causal_gqa():
    w = W.WORKLOADS["causal_gqa_llama8b_s2048"]
    bwd_case(w.B, w.S, w.Hq, w.Hkv, w.D, seed=w.seed, causal=True)


def test_bwd_is_bit_identical_across_runs():
    q, k, v, do = (dev_bf16(W.normal_bf16(240 + i, (1, 900, 8 if i in (0, 3) else 2, 128))) for i in range(4))
    o, lse = ea.attn_fwd(q, k, v, causal=True)
    r1 = ea.attn_bwd(q, k, v, o, lse, do, causal=True, deterministic=True)
    r2 = ea.attn_bwd(q, k, v, o, lse, do, causal=True, deterministic=True)
    torch.cuda.synchronize()
    for a, b in zip(r1, r2):
        assert torch.equal(a, b)
