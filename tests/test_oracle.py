"""Pins for the fp64 CPU oracle, checked against closed forms, invariants,
brute force on tiny inputs and torch's fp64 CPU SDPA (CPU only)."""
import math
import os

import numpy as np
import pytest

import oracle
import workloads as W

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "closed_forms.txt")


def golden():
    vals = {}
    for line in open(GOLDEN):
        line = line.split("#")[0].strip()
        if not line:
            continue
        parts = line.split()
        vals[parts[0]] = [float(x) for x in parts[1:]]
    return vals


def bf16(x):
    return W.f32_to_bf16_bits(np.asarray(x, dtype=np.float32))


def f64(b):
    return W.bf16_bits_to_f64(b)


def rand_qkv(seed, B, S, Hq, Hkv, D, Skv=None):
    Skv = S if Skv is None else Skv
    q = W.normal_bf16(seed, (B, S, Hq, D))
    k = W.normal_bf16(seed + 1, (B, Skv, Hkv, D))
    v = W.normal_bf16(seed + 2, (B, Skv, Hkv, D))
    return q, k, v


# ---------------------------------------------------------------- closed forms

def test_one_key_returns_that_value_and_its_score():
    # q = (1, 0, ...), k0 = (2, 0, ...), scale 0.5 -> the only score is exactly 1.
    D = 8
    q = np.zeros((1, 1, 1, D), np.float32); q[..., 0] = 1
    k = np.zeros((1, 1, 1, D), np.float32); k[..., 0] = 2
    v = W.normal_bf16(7, (1, 1, 1, D))
    o, lse = oracle.attn(bf16(q), bf16(k), v, scale=0.5)
    assert np.array_equal(o[0, 0, 0], f64(v)[0, 0, 0])
    assert lse[0, 0, 0] == 1.0


def test_two_keys_give_logistic_weights():
    g = golden()
    q = bf16(np.ones((1, 1, 1, 1)))
    k = bf16(np.array([1.0, 0.0]).reshape(1, 2, 1, 1))
    v = bf16(np.array([1.0, 0.0]).reshape(1, 2, 1, 1))
    o, lse = oracle.attn(q, k, v, scale=1.0)
    assert abs(o[0, 0, 0, 0] - g["logistic_1"][0]) < 1e-15
    assert abs(lse[0, 0, 0] - g["softplus_1"][0]) < 1e-15


@pytest.mark.parametrize("mask,window", [(W.MASK_NONE, (-1, -1)), (W.MASK_CAUSAL, (-1, 0)),
                                         (W.MASK_WINDOW, (5, 0)), (W.MASK_WINDOW, (3, 2)),
                                         (W.MASK_DOCUMENT, (-1, -1))])
def test_uniform_scores_average_allowed_values(mask, window):
    # q = 0 makes every score 0: O is the mean of the allowed V rows and
    # LSE = ln(number of allowed keys). The allowed counts are derived here from
    # the mask's definition by interval arithmetic, not by the oracle's predicate.
    S, H, D = 23, 2, 4
    q = np.zeros((1, S, H, D), np.uint16)
    _, k, v = rand_qkv(11, 1, S, H, H, D)
    lens = [5, 1, 9, 8]
    doc = W.doc_ids_from_lengths(lens)
    starts = np.concatenate([[0], np.cumsum(lens)[:-1]])
    o, lse = oracle.attn(q, k, v, mask=mask, window=window, doc_id=doc if mask == W.MASK_DOCUMENT else None)
    vf = f64(v)
    for i in range(S):
        if mask == W.MASK_NONE:
            lo, hi = 0, S - 1
        elif mask == W.MASK_CAUSAL:
            lo, hi = 0, i
        elif mask == W.MASK_WINDOW:
            lo, hi = max(0, i - window[0]), min(S - 1, i + window[1])
        else:
            lo, hi = starts[doc[i]], i
        n = hi - lo + 1
        assert abs(lse[0, 0, i] - math.log(n)) < 1e-14
        want = vf[0, lo:hi + 1, :, :].mean(axis=0)
        assert np.max(np.abs(o[0, i] - want)) < 1e-14


def test_uniform_scores_per_batch_documents():
    # FlexAttention's mask_mod receives the batch index (attention-gym issue 101:
    # create_block_mask(mask_mod, B, H, Q_LEN, KV_LEN)), so a batch of packed
    # sequences may have a different document layout per batch. With q = 0 the
    # row of batch b averages the V rows of its own document up to i; the
    # document start comes from that batch's lengths by interval arithmetic.
    S, H, D = 23, 2, 4
    q = np.zeros((2, S, H, D), np.uint16)
    _, k, v = rand_qkv(12, 2, S, H, H, D)
    lens = [[5, 1, 9, 8], [11, 12]]
    doc = np.stack([W.doc_ids_from_lengths(x) for x in lens])
    o, lse = oracle.attn(q, k, v, mask=W.MASK_DOCUMENT, doc_id=doc)
    vf = f64(v)
    for b in range(2):
        starts = np.concatenate([[0], np.cumsum(lens[b])[:-1]])
        for i in range(S):
            lo = starts[doc[b, i]]
            assert abs(lse[b, 1, i] - math.log(i - lo + 1)) < 1e-14
            assert np.max(np.abs(o[b, i] - vf[b, lo:i + 1].mean(axis=0))) < 1e-14
    # a [S] row is shared by every batch: equal to passing it once per batch
    o1, l1 = oracle.attn(q, k, v, mask=W.MASK_DOCUMENT, doc_id=doc[0])
    o2, l2 = oracle.attn(q, k, v, mask=W.MASK_DOCUMENT, doc_id=np.stack([doc[0], doc[0]]))
    assert np.array_equal(o1, o2) and np.array_equal(l1, l2)


def test_constant_v_rows_give_that_row():
    q, k, _ = rand_qkv(21, 2, 37, 4, 2, 16)
    row = W.normal_bf16(99, (16,))
    v = np.broadcast_to(row, (2, 37, 2, 16)).copy()
    for mask, window in [(W.MASK_NONE, (-1, -1)), (W.MASK_CAUSAL, (-1, 0)), (W.MASK_WINDOW, (7, 0))]:
        o, _ = oracle.attn(q, k, v, mask=mask, window=window)
        assert np.max(np.abs(o - f64(row))) < 1e-14


def test_causal_first_query_returns_v0():
    q, k, v = rand_qkv(31, 1, 50, 4, 4, 32)
    o, lse = oracle.attn(q, k, v, mask=W.MASK_CAUSAL, window=(-1, 0))
    assert np.array_equal(o[0, 0], f64(v)[0, 0])
    s00 = (f64(q)[0, 0] * f64(k)[0, 0]).sum(-1) / math.sqrt(32)
    assert np.max(np.abs(lse[0, :, 0] - s00)) < 1e-13


def test_fully_masked_row_is_zero_with_minus_inf_lse():
    q, k, v = rand_qkv(41, 1, 4, 1, 1, 8)
    o, lse = oracle.attn(q, k, v, mask=W.MASK_CAUSAL, window=(-1, 0), q_offset=-1)
    assert np.all(o[0, 0] == 0) and lse[0, 0, 0] == -np.inf
    assert np.isfinite(lse[0, 0, 1:]).all()


def test_probability_rows_sum_to_one():
    # With V = identity (Skv = D), output row i is the probability row itself.
    S = D = 16
    q, k, _ = rand_qkv(51, 1, S, 2, 2, D)
    eye = np.broadcast_to(np.eye(D, dtype=np.float32)[None, :, None, :], (1, S, 2, D))
    v = bf16(eye)
    for mask, window in [(W.MASK_NONE, (-1, -1)), (W.MASK_CAUSAL, (-1, 0)), (W.MASK_WINDOW, (4, 1))]:
        o, _ = oracle.attn(q, k, v, mask=mask, window=window)
        assert np.max(np.abs(o.sum(-1) - 1.0)) <= 1e-12
        assert (o >= 0).all()


# ---------------------------------------------------------------- GQA

def test_gqa_equals_repeat_kv_expanded_mha():
    # repeat_kv: x[:, :, None].expand(b, Hkv, n_rep, s, d).reshape(b, Hkv*n_rep, s, d)
    # puts KV head j at query heads j*n_rep .. j*n_rep+n_rep-1 (BHSD there; BSHD here).
    B, S, Hq, Hkv, D = 2, 29, 8, 2, 16
    q, k, v = rand_qkv(61, B, S, Hq, Hkv, D)
    g = Hq // Hkv
    k_rep = np.broadcast_to(k[:, :, :, None, :], (B, S, Hkv, g, D)).reshape(B, S, Hq, D).copy()
    v_rep = np.broadcast_to(v[:, :, :, None, :], (B, S, Hkv, g, D)).reshape(B, S, Hq, D).copy()
    for mask in (W.MASK_NONE, W.MASK_CAUSAL):
        o1, l1 = oracle.attn(q, k, v, mask=mask, window=(-1, 0))
        o2, l2 = oracle.attn(q, k_rep, v_rep, mask=mask, window=(-1, 0))
        assert np.array_equal(o1, o2) and np.array_equal(l1, l2)


def test_mqa_single_kv_head():
    B, S, Hq, D = 1, 17, 6, 8
    q, k, v = rand_qkv(71, B, S, Hq, 1, D)
    o1, _ = oracle.attn(q, k, v)
    for h in range(Hq):
        o2, _ = oracle.attn(np.ascontiguousarray(q[:, :, h:h + 1]), k, v)
        assert np.array_equal(o1[:, :, h:h + 1], o2)


# ---------------------------------------------------------------- library routine

@pytest.mark.parametrize("Hq,Hkv,Sq,Skv,causal", [(4, 4, 33, 33, False), (8, 2, 40, 40, True),
                                                 (6, 3, 19, 45, False), (4, 1, 64, 64, True)])
def test_matches_torch_sdpa_fp64(Hq, Hkv, Sq, Skv, causal):
    torch = pytest.importorskip("torch")
    q, k, v = rand_qkv(81, 2, Sq, Hq, Hkv, 32, Skv=Skv)
    o, _ = oracle.attn(q, k, v, mask=W.MASK_CAUSAL if causal else W.MASK_NONE, window=(-1, 0))
    tq, tk, tv = (torch.from_numpy(f64(x)).permute(0, 2, 1, 3) for x in (q, k, v))
    ref = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, is_causal=causal, enable_gqa=True)
    ref = ref.permute(0, 2, 1, 3).numpy()
    assert np.max(np.abs(o - ref)) < 1e-12


def test_window_matches_torch_sdpa_with_boolean_mask():
    torch = pytest.importorskip("torch")
    S, left, right = 48, 6, 3
    q, k, v = rand_qkv(91, 1, S, 2, 2, 16)
    o, _ = oracle.attn(q, k, v, mask=W.MASK_WINDOW, window=(left, right))
    i = np.arange(S)[:, None]
    j = np.arange(S)[None, :]
    allowed = torch.from_numpy((i - j <= left) & (j - i <= right))
    tq, tk, tv = (torch.from_numpy(f64(x)).permute(0, 2, 1, 3) for x in (q, k, v))
    ref = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, attn_mask=allowed)
    assert np.max(np.abs(o - ref.permute(0, 2, 1, 3).numpy())) < 1e-12


# ---------------------------------------------------------------- score mods

def test_softcap_closed_form():
    g = golden()
    q = bf16(np.ones((1, 1, 1, 1)))
    k = bf16(np.array([30.0, 0.0]).reshape(1, 2, 1, 1))
    v = bf16(np.array([1.0, 0.0]).reshape(1, 2, 1, 1))
    o, lse = oracle.attn(q, k, v, scale=1.0, mod=W.MOD_SOFTCAP, softcap=30.0)
    s0 = 30.0 * g["tanh_1"][0]
    assert abs(lse[0, 0, 0] - (s0 + math.log1p(math.exp(-s0)))) < 1e-13
    assert abs(o[0, 0, 0, 0] - 1.0 / (1.0 + math.exp(-s0))) < 1e-15


def test_softcap_large_cap_is_identity():
    q, k, v = rand_qkv(101, 1, 20, 2, 2, 16)
    o1, l1 = oracle.attn(q, k, v)
    o2, l2 = oracle.attn(q, k, v, mod=W.MOD_SOFTCAP, softcap=1e7)
    assert np.max(np.abs(o1 - o2)) < 1e-10 and np.max(np.abs(l1 - l2)) < 1e-10


def test_alibi_sign_and_closed_form():
    # query at position 1, keys at 0 and 1, all raw scores 0, slope 0.5:
    # scores become (-0.5, 0) -> weight of key 1 is logistic(0.5).
    g = golden()
    q = np.zeros((1, 2, 1, 1), np.uint16)
    k = np.zeros((1, 2, 1, 1), np.uint16)
    v = bf16(np.array([0.0, 1.0]).reshape(1, 2, 1, 1))
    o, lse = oracle.attn(q, k, v, mask=W.MASK_CAUSAL, window=(-1, 0), mod=W.MOD_ALIBI,
                         alibi=np.array([0.5], np.float32))
    assert abs(o[0, 1, 0, 0] - g["logistic_0.5"][0]) < 1e-15
    assert abs(lse[0, 0, 1] - g["softplus_-0.5"][0]) < 1e-15


def test_alibi_zero_slope_is_plain_and_per_batch_slopes():
    q, k, v = rand_qkv(111, 2, 21, 4, 2, 8)
    o1, l1 = oracle.attn(q, k, v, mask=W.MASK_CAUSAL, window=(-1, 0))
    o2, l2 = oracle.attn(q, k, v, mask=W.MASK_CAUSAL, window=(-1, 0), mod=W.MOD_ALIBI,
                         alibi=np.zeros(4, np.float32))
    assert np.array_equal(o1, o2) and np.array_equal(l1, l2)
    sl = np.array([[0.5, 0.25, 0.1, 0.0], [0.0, 0.0, 0.0, 0.0]], np.float32)
    o3, _ = oracle.attn(q, k, v, mask=W.MASK_CAUSAL, window=(-1, 0), mod=W.MOD_ALIBI, alibi=sl)
    assert np.array_equal(o3[1], o1[1]) and not np.allclose(o3[0, :, :3], o1[0, :, :3])


def _geometric_lse(slope, n):
    """ln sum_{d=0}^{n-1} exp(-slope * d): the log-sum-exp of a causal row whose
    raw scores are all 0, so that only the ALiBi bias slope * (kv - q) remains."""
    if slope == 0.0:
        return math.log(n)
    return math.log(-math.expm1(-slope * n)) - math.log(-math.expm1(-slope))


def test_alibi_slope_is_indexed_by_query_head():
    # FlashAttention overview, "Examples": alibi_slopes has shape (nheads,) with
    # nheads the number of query heads, so under GQA each query head uses its
    # own slope, not the one of the KV head it shares. Raw scores are 0 (q = 0),
    # Hq = 4 query heads share one KV head, and every row's LSE has the
    # geometric closed form of its own head's slope. An oracle that indexed the
    # slope by the KV head would give all four heads the first slope.
    S, Hq, D = 40, 4, 8
    q = np.zeros((1, S, Hq, D), np.uint16)
    k = W.normal_bf16(141, (1, S, 1, D))
    v = W.normal_bf16(142, (1, S, 1, D))
    slopes = np.array([0.5, 0.125, 0.03125, 0.0], np.float32)
    o, lse = oracle.attn(q, k, v, mask=W.MASK_CAUSAL, window=(-1, 0), mod=W.MOD_ALIBI, alibi=slopes)
    for h in range(Hq):
        for i in (0, 1, 7, S - 1):
            assert abs(lse[0, h, i] - _geometric_lse(float(slopes[h]), i + 1)) < 1e-13, (h, i)
    # only head 0 has a non-zero slope: heads 1..3 must equal the plain result
    o_plain, l_plain = oracle.attn(q, k, v, mask=W.MASK_CAUSAL, window=(-1, 0))
    one = np.array([0.5, 0.0, 0.0, 0.0], np.float32)
    o1, l1 = oracle.attn(q, k, v, mask=W.MASK_CAUSAL, window=(-1, 0), mod=W.MOD_ALIBI, alibi=one)
    assert np.array_equal(o1[:, :, 1:], o_plain[:, :, 1:]) and np.array_equal(l1[:, 1:], l_plain[:, 1:])
    assert not np.allclose(o1[:, 1:, 0], o_plain[:, 1:, 0])


def test_decode_alibi_slope_is_indexed_by_query_head():
    # The same reading for the paged decode: the single query of sequence b sits
    # at position cache_seqlens[b] - 1 and head h adds slope[h] * (t - (n - 1)).
    Hq, D, page = 4, 8, 16
    seqlens = np.array([37, 5], np.int32)
    w = W.Decode("t", B=2, Hq=Hq, Hkv=1, D=D, kv_len=48, page_size=page, seed=143)
    d = W.make_decode_inputs(w, seqlens=seqlens)
    q0 = np.zeros_like(d["q"])
    slopes = np.array([0.5, 0.125, 0.03125, 0.0], np.float32)
    _, lse = oracle.decode(q0, d["k_cache"], d["v_cache"], d["block_table"], d["cache_seqlens"],
                           mod=W.MOD_ALIBI, alibi=slopes)
    for b, n in enumerate(seqlens):
        for h in range(Hq):
            assert abs(lse[b, h] - _geometric_lse(float(slopes[h]), int(n))) < 1e-13, (b, h)


def test_alibi_slopes_for_eight_heads():
    assert np.array_equal(W.alibi_slopes(8), np.array(golden()["alibi8"], np.float32))
    s32 = W.alibi_slopes(32)
    assert s32[3] == 0.5 and s32[31] == 2.0 ** -8


# ---------------------------------------------------------------- split / combine

@pytest.mark.parametrize("cuts", [[0, 17, 40, 64], [0, 1, 2, 64], [0, 30, 30, 64], [0, 64]])
def test_lse_combine_split_invariance(cuts):
    q, k, v = rand_qkv(121, 1, 64, 2, 1, 16)
    o_full, l_full = oracle.attn(q, k, v, mask=W.MASK_CAUSAL, window=(-1, 0))
    parts = [oracle.attn(q, k, v, mask=W.MASK_CAUSAL, window=(-1, 0), kv_range=(a, b))
             for a, b in zip(cuts[:-1], cuts[1:])]
    for i in range(64):
        for h in range(2):
            lp = np.array([p[1][0, h, i] for p in parts])
            op = np.stack([p[0][0, i, h] for p in parts])
            o, lse = oracle.lse_combine(lp, op)
            assert abs(lse - l_full[0, h, i]) < 1e-12
            assert np.max(np.abs(o - o_full[0, i, h])) < 1e-12


def test_lse_combine_all_empty():
    o, lse = oracle.lse_combine(np.array([-np.inf, -np.inf]), np.zeros((2, 4)))
    assert lse == -np.inf and np.all(o == 0)


# ---------------------------------------------------------------- paged decode

@pytest.mark.parametrize("mod", [W.MOD_NONE, W.MOD_ALIBI, W.MOD_SOFTCAP])
def test_decode_paging_invariance(mod):
    w = W.Decode("t", B=3, Hq=8, Hkv=2, D=16, kv_len=70, page_size=16, seed=5)
    seqlens = np.array([70, 33, 1], np.int32)
    d = W.make_decode_inputs(w, seqlens=seqlens)
    alibi = W.alibi_slopes(8) if mod == W.MOD_ALIBI else None
    o, lse = oracle.decode(d["q"], d["k_cache"], d["v_cache"], d["block_table"], d["cache_seqlens"], mod=mod,
                           softcap=20.0, alibi=alibi)
    for b in range(3):
        n = seqlens[b]
        pages = d["block_table"][b]
        kc = d["k_cache"][pages].reshape(-1, 2, 16)[:n][None]
        vc = d["v_cache"][pages].reshape(-1, 2, 16)[:n][None]
        o2, l2 = oracle.attn(np.ascontiguousarray(d["q"][b:b + 1]), np.ascontiguousarray(kc),
                             np.ascontiguousarray(vc), q_offset=int(n - 1), mask=W.MASK_NONE, mod=mod,
                             softcap=20.0, alibi=alibi)
        assert np.array_equal(o[b], o2[0, 0]) and np.array_equal(lse[b], l2[0, :, 0])


def test_decode_rejects_bad_page_ids():
    w = W.Decode("t", B=1, Hq=2, Hkv=1, D=8, kv_len=32, page_size=16, seed=9)
    d = W.make_decode_inputs(w)
    bt = d["block_table"].copy()
    bt[0, 1] = 99
    with pytest.raises(ValueError):
        oracle.decode(d["q"], d["k_cache"], d["v_cache"], bt, d["cache_seqlens"])


# ---------------------------------------------------------------- block mask

def test_tile_classes_causal_closed_form():
    n = 8
    bm = oracle.block_mask(W.MASK_CAUSAL, n * 128, n * 128, window=(-1, 0))
    i, j = np.meshgrid(np.arange(n), np.arange(n), indexing="ij")
    want = np.where(j < i, 2, np.where(j == i, 1, 0))
    assert np.array_equal(bm["cls"], want)
    assert list(bm["full_cnt"]) == list(range(n)) and list(bm["part_cnt"]) == [1] * n
    assert list(bm["full_idx"][5, :5]) == [0, 1, 2, 3, 4] and bm["part_idx"][5, 0] == 5


def test_tile_classes_window_closed_form():
    # window 0 <= q - kv < 1024 with 128-wide tiles: diagonal partial, seven full
    # tiles below it, the eighth one below partial (q - kv spans 897..1151).
    n = 20
    bm = oracle.block_mask(W.MASK_WINDOW, n * 128, n * 128, window=(1023, 0))
    for i in range(n):
        for j in range(n):
            if j == i or j == i - 8:
                want = 1
            elif i - 7 <= j <= i - 1:
                want = 2
            else:
                want = 0
            assert bm["cls"][i, j] == want, (i, j)


def test_tile_classes_documents_interval_form():
    w = W.WORKLOADS["packed_docs_alibi_s16384"]
    S = 4096
    lens = W.doc_lengths(w.seed + 0x100, S, 128, 2048)
    doc = W.doc_ids_from_lengths(lens)
    starts = np.concatenate([[0], np.cumsum(lens)[:-1]])
    ends = np.cumsum(lens) - 1
    T = 128
    bm = oracle.block_mask(W.MASK_DOCUMENT, S, S, doc_id=doc)
    n = S // T
    for qi in range(n):
        q0, q1 = qi * T, qi * T + T - 1
        for kj in range(n):
            k0, k1 = kj * T, kj * T + T - 1
            full = k1 <= q0 and doc[k0] == doc[q1]
            any_pair = False
            for d in range(len(lens)):
                jl, jh = max(k0, starts[d]), min(k1, ends[d])
                il, ih = max(q0, starts[d]), min(q1, ends[d])
                if jl <= jh and il <= ih and jl <= ih:
                    any_pair = True
            want = 2 if full else (1 if any_pair else 0)
            assert bm["cls"][qi, kj] == want, (qi, kj)


def test_tile_classes_ragged_tail():
    # Sq = Skv = 300 with 128-wide tiles: out-of-range positions do not count.
    bm = oracle.block_mask(W.MASK_CAUSAL, 300, 300, window=(-1, 0))
    assert bm["cls"].shape == (3, 3)
    assert bm["cls"][2, 2] == 1 and bm["cls"][2, 1] == 2 and bm["cls"][1, 2] == 0
    bm = oracle.block_mask(W.MASK_NONE, 300, 200)
    assert (bm["cls"] == 2).all() and bm["cls"].shape == (3, 2)


def test_count_pairs():
    assert oracle.count_pairs(W.MASK_CAUSAL, 2048, 2048, window=(-1, 0)) == 2048 * 2049 // 2
    # window of 1024 (left 1023): row i sees min(i+1, 1024) keys
    S = 8192
    assert oracle.count_pairs(W.MASK_WINDOW, S, S, window=(1023, 0)) == sum(min(i + 1, 1024) for i in range(S))
    lens = [5, 7, 3]
    doc = W.doc_ids_from_lengths(lens)
    assert oracle.count_pairs(W.MASK_DOCUMENT, 15, 15, doc_id=doc) == sum(L * (L + 1) // 2 for L in lens)


def test_rejects_bad_arguments():
    q, k, v = rand_qkv(131, 1, 8, 3, 2, 8)
    with pytest.raises(ValueError):
        oracle.attn(q, k, v)  # 3 % 2 != 0
    q, k, v = rand_qkv(131, 1, 8, 2, 2, 8)
    with pytest.raises(ValueError):
        oracle.attn(q, k, v, mask=W.MASK_DOCUMENT)  # no doc ids
    with pytest.raises(ValueError):
        oracle.attn(q, k, v, mod=W.MOD_SOFTCAP, softcap=0.0)


def test_sampled_rows_equal_full_rows():
    q, k, v = rand_qkv(141, 2, 40, 4, 2, 16)
    o, lse = oracle.attn(q, k, v, mask=W.MASK_CAUSAL, window=(-1, 0))
    rows = np.array([[0, 0, 0], [1, 3, 39], [0, 2, 17]], np.int32)
    o2, l2 = oracle.attn(q, k, v, mask=W.MASK_CAUSAL, window=(-1, 0), rows=rows)
    for r, (b, h, i) in enumerate(rows):
        assert np.array_equal(o2[r], o[b, i, h]) and l2[r] == lse[b, h, i]


# ---------------------------------------------------------------- input recipe

def test_input_generator_is_deterministic_and_normal():
    a = W.normal_bf16(1234, (1 << 16,))
    b = W.normal_bf16(1234, (1 << 16,))
    assert np.array_equal(a, b)
    x = f64(a)
    assert abs(x.mean()) < 0.02 and abs(x.std() - 1) < 0.02
    assert W.splitmix64(0, 1)[0] == np.uint64(0xE220A8397B1DCDAF)  # splitmix64 reference first output, seed 0


def test_bf16_rounding_is_nearest_even():
    vals = np.array([1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -2.5, 1.00390625], np.float32)
    got = W.bf16_bits_to_f64(W.f32_to_bf16_bits(vals))
    assert list(got) == [1.0, 1.0, 1.015625, -2.5, 1.0]


def test_doc_lengths_and_page_permutation():
    lens = W.doc_lengths(W.WORKLOADS["packed_docs_alibi_s16384"].seed + 0x100, 16384, 128, 2048)
    assert sum(lens) == 16384 and all(128 <= L <= 2048 for L in lens[:-1]) and 1 <= lens[-1] <= 2048
    perm = W.page_permutation(77, 4096)
    assert sorted(perm.tolist()) == list(range(4096)) and not np.array_equal(perm, np.arange(4096))


# ---------------------------------------------------------------- ReLU activation wrapper
# The talk's activation wrapper (FlexAttention + FlashAttention-4, "activation
# wrapper ... a ReLU"): O = sum_j max(scale q.k_j, 0) v_j over allowed keys,
# unnormalised; the LSE slot holds ln of the summed weights.

def test_relu_activation_one_key_and_all_negative():
    q = bf16(np.array([1.0, 0.0, 0.0, 0.0]).reshape(1, 1, 1, 4))
    k = bf16(np.array([[2.0, 0.0, 0.0, 0.0], [-4.0, 0.0, 0.0, 0.0]]).reshape(1, 2, 1, 4))
    v = bf16(np.array([[3.0, -1.0, 0.5, 2.0], [7.0, 7.0, 7.0, 7.0]]).reshape(1, 2, 1, 4))
    o, lse = oracle.attn(q, k, v, scale=0.5, mod=oracle.MOD_RELU)
    # weights: relu(0.5 * 2) = 1 for key 0, relu(0.5 * -4) = 0 for key 1
    assert np.array_equal(o.ravel(), [3.0, -1.0, 0.5, 2.0]) and lse.ravel()[0] == 0.0
    o, lse = oracle.attn(q, k[:, 1:], v[:, 1:], scale=0.5, mod=oracle.MOD_RELU)
    assert np.array_equal(o.ravel(), np.zeros(4)) and lse.ravel()[0] == -np.inf


def test_relu_activation_homogeneity_linearity_and_mask():
    q, k, v = rand_qkv(61, 1, 40, 4, 2, 32)
    o1, l1 = oracle.attn(q, k, v, mod=oracle.MOD_RELU)
    # doubling q (exact in bf16) doubles every weight: O doubles, LSE gains ln 2
    o2, l2 = oracle.attn(bf16(2.0 * f64(q)), k, v, mod=oracle.MOD_RELU)
    assert np.allclose(o2, 2.0 * o1, rtol=1e-12, atol=1e-12)
    fin = np.isfinite(l1)
    assert np.allclose(l2[fin], l1[fin] + math.log(2.0), atol=1e-12)
    # doubling v doubles O and leaves the weights
    o3, l3 = oracle.attn(q, k, bf16(2.0 * f64(v)), mod=oracle.MOD_RELU)
    assert np.allclose(o3, 2.0 * o1, rtol=1e-12, atol=1e-12) and np.array_equal(l3, l1)
    # causal: row 0 sees key 0 only
    oc, lc = oracle.attn(q, k, v, mod=oracle.MOD_RELU, mask=oracle.MASK_CAUSAL, window=(-1, 0))
    s00 = max(float(np.dot(f64(q)[0, 0, 0], f64(k)[0, 0, 0])) / math.sqrt(32), 0.0)
    assert np.allclose(oc[0, 0, 0], s00 * f64(v)[0, 0, 0], atol=1e-12)
    # a row's output is the row's positive-weighted sum whatever the other rows hold
    assert np.all(np.isfinite(oc))
