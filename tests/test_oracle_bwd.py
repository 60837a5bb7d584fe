"""Pins for the fp64 backward of the oracle (dQ, dK, dV), CPU only: central
finite differences of the oracle's own fp64 forward, closed forms for one
and two keys, gradient invariants, the repeat_kv head map, and torch's fp64
CPU autograd of scaled_dot_product_attention as a library second opinion."""
import math

import numpy as np
import pytest

import oracle
import workloads as W


def f64(bits):
    return W.bf16_bits_to_f64(bits)


def rand(seed, shape):
    return f64(W.normal_bf16(seed, shape))


def loss(q, k, v, dout, **kw):
    o, _ = oracle.attn_f64(q, k, v, **kw)
    return float(np.sum(o * dout))


CASES = [
    dict(),
    dict(mask=W.MASK_CAUSAL, window=(-1, 0)),
    dict(mask=W.MASK_WINDOW, window=(3, 1), q_offset=2),
    dict(mask=W.MASK_DOCUMENT, doc_id=np.array([0, 0, 0, 1, 1, 2, 2, 2, 2], np.int32)),
    dict(mask=W.MASK_CAUSAL, window=(-1, 0), mod=W.MOD_SOFTCAP, softcap=1.5),
    dict(mask=W.MASK_CAUSAL, window=(-1, 0), mod=W.MOD_ALIBI, alibi=np.array([0.5, 0.25, 0.1, 0.03], np.float32)),
]


def test_f64_forward_equals_the_bf16_forward():
    qb, kb, vb = W.normal_bf16(1, (2, 9, 4, 8)), W.normal_bf16(2, (2, 9, 2, 8)), W.normal_bf16(3, (2, 9, 2, 8))
    for kw in CASES:
        o1, l1 = oracle.attn(qb, kb, vb, **kw)
        o2, l2 = oracle.attn_f64(f64(qb), f64(kb), f64(vb), **kw)
        assert np.max(np.abs(o1 - o2)) < 1e-14 and np.max(np.abs(np.nan_to_num(l1 - l2))) < 1e-14


@pytest.mark.parametrize("kw", CASES, ids=["none", "causal", "window", "doc", "softcap", "alibi"])
def test_backward_matches_central_finite_differences(kw):
    # L = sum(O * dout); dL/dx by (L(x + h) - L(x - h)) / 2h, h = 1e-5, on
    # sampled elements of q, k and v (GQA: 4 query heads on 2 KV heads).
    B, S, Hq, Hkv, D = 1, 9, 4, 2, 8
    q, k, v, dout = rand(11, (B, S, Hq, D)), rand(12, (B, S, Hkv, D)), rand(13, (B, S, Hkv, D)), rand(14, (B, S, Hq, D))
    dq, dk, dv = oracle.attn_bwd(q, k, v, dout, **kw)
    rng = np.random.default_rng(5)
    h = 1e-5
    for name, x, g in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        for _ in range(12):
            idx = tuple(int(rng.integers(n)) for n in x.shape)
            xp, xm = x.copy(), x.copy()
            xp[idx] += h
            xm[idx] -= h
            args = {"q": q, "k": k, "v": v}
            args[name] = xp
            lp = loss(args["q"], args["k"], args["v"], dout, **kw)
            args[name] = xm
            lm = loss(args["q"], args["k"], args["v"], dout, **kw)
            fd = (lp - lm) / (2 * h)
            assert abs(fd - g[idx]) < 1e-7 * max(1.0, abs(fd)), (name, idx, fd, g[idx])


def test_one_key_gradients():
    # A single key: O = v0 whatever q and k are, so dV = the sum of dout over
    # the rows and heads that read it, and dQ = dK = 0.
    q, k, v, dout = rand(21, (1, 3, 2, 4)), rand(22, (1, 1, 1, 4)), rand(23, (1, 1, 1, 4)), rand(24, (1, 3, 2, 4))
    dq, dk, dv = oracle.attn_bwd(q, k, v, dout)
    assert np.all(dq == 0) and np.all(dk == 0)
    assert np.max(np.abs(dv[0, 0, 0] - dout[0].sum(axis=(0, 1)))) < 1e-14


def test_two_key_logistic_gradients():
    # Scores (x, 0) with x = scale q.k0 (k1 = 0): the first key's weight is the
    # logistic s(x), O = s v0 + (1 - s) v1, so dL/dx = s (1 - s) (v0 - v1).dout,
    # dq = scale dL/dx k0, dk0 = scale dL/dx q, dk1 = -scale dL/dx q,
    # dv0 = s dout, dv1 = (1 - s) dout.
    D, scale = 3, 0.7
    q = np.array([0.5, -1.0, 2.0]).reshape(1, 1, 1, D)
    k = np.zeros((1, 2, 1, D)); k[0, 0, 0] = [1.0, 0.25, -0.5]
    v = np.zeros((1, 2, 1, D)); v[0, 0, 0] = [2.0, 0.0, 1.0]; v[0, 1, 0] = [-1.0, 3.0, 0.5]
    dout = np.array([0.3, -0.2, 1.1]).reshape(1, 1, 1, D)
    dq, dk, dv = oracle.attn_bwd(q, k, v, dout, scale=scale)
    x = scale * float(q[0, 0, 0] @ k[0, 0, 0])
    sg = 1.0 / (1.0 + math.exp(-x))
    dx = sg * (1 - sg) * float((v[0, 0, 0] - v[0, 1, 0]) @ dout[0, 0, 0])
    assert np.max(np.abs(dq[0, 0, 0] - scale * dx * k[0, 0, 0])) < 1e-15
    assert np.max(np.abs(dk[0, 0, 0] - scale * dx * q[0, 0, 0])) < 1e-15
    # the row's score gradients sum to 0, so the second key's is -dL/dx
    assert np.max(np.abs(dk[0, 1, 0] + scale * dx * q[0, 0, 0])) < 1e-15
    assert np.max(np.abs(dv[0, 0, 0] - sg * dout[0, 0, 0])) < 1e-15
    assert np.max(np.abs(dv[0, 1, 0] - (1 - sg) * dout[0, 0, 0])) < 1e-15


def test_gradient_invariants():
    # Without a score mod each softmax row's score gradients sum to 0, so
    # sum_j dK_j = scale sum_i (sum_j dz_ij) q_i = 0; and each row's
    # probabilities sum to 1, so sum_j dV_j = sum of dout over rows that see a key.
    B, S, Hq, Hkv, D = 2, 11, 4, 2, 8
    q, k, v, dout = rand(31, (B, S, Hq, D)), rand(32, (B, S, Hkv, D)), rand(33, (B, S, Hkv, D)), rand(34, (B, S, Hq, D))
    for kw in CASES[:4]:
        dq, dk, dv = oracle.attn_bwd(q, k, v, dout, **kw)
        assert np.max(np.abs(dk.sum(axis=1))) < 1e-12
        _, lse = oracle.attn_f64(q, k, v, **kw)
        seen = np.isfinite(lse).transpose(0, 2, 1)[..., None]  # [B, S, Hq, 1]
        want = (dout * seen).reshape(B, S, Hkv, Hq // Hkv, D).sum(axis=(1, 3))
        assert np.max(np.abs(dv.sum(axis=1) - want)) < 1e-12


def test_gqa_equals_repeat_kv_expanded_mha():
    # transformers issue 36218: repeat_kv puts KV head j at query heads
    # j*g .. j*g+g-1; the GQA gradient of K/V head j is the sum of the
    # expanded MHA's gradients over those heads.
    B, S, Hq, Hkv, D = 1, 10, 6, 2, 4
    q, k, v, dout = rand(41, (B, S, Hq, D)), rand(42, (B, S, Hkv, D)), rand(43, (B, S, Hkv, D)), rand(44, (B, S, Hq, D))
    g = Hq // Hkv
    ke = np.repeat(k, g, axis=2)
    ve = np.repeat(v, g, axis=2)
    kw = dict(mask=W.MASK_CAUSAL, window=(-1, 0))
    dq1, dk1, dv1 = oracle.attn_bwd(q, k, v, dout, **kw)
    dq2, dk2, dv2 = oracle.attn_bwd(q, ke, ve, dout, **kw)
    assert np.max(np.abs(dq1 - dq2)) < 1e-13
    assert np.max(np.abs(dk1 - dk2.reshape(B, S, Hkv, g, D).sum(axis=3))) < 1e-13
    assert np.max(np.abs(dv1 - dv2.reshape(B, S, Hkv, g, D).sum(axis=3))) < 1e-13


@pytest.mark.parametrize("causal", [False, True])
def test_matches_torch_fp64_autograd(causal):
    torch = pytest.importorskip("torch")
    B, S, Hq, Hkv, D = 2, 13, 4, 2, 16
    q, k, v, dout = rand(51, (B, S, Hq, D)), rand(52, (B, S, Hkv, D)), rand(53, (B, S, Hkv, D)), rand(54, (B, S, Hq, D))
    kw = dict(mask=W.MASK_CAUSAL, window=(-1, 0)) if causal else {}
    dq, dk, dv = oracle.attn_bwd(q, k, v, dout, **kw)
    tq, tk, tv = (torch.tensor(x.transpose(0, 2, 1, 3), requires_grad=True) for x in (q, k, v))
    o = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, is_causal=causal, enable_gqa=True)
    o.backward(torch.tensor(dout.transpose(0, 2, 1, 3)))
    for mine, ref in ((dq, tq.grad), (dk, tk.grad), (dv, tv.grad)):
        assert np.max(np.abs(mine - ref.numpy().transpose(0, 2, 1, 3))) < 1e-12
