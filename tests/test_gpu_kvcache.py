"""GPU parity of flash_attn_with_kvcache semantics (FlashAttention overview,
"Examples") against the fp64 oracle: the in-place cache update with rotary
embedding (paged and batch-indexed caches, both pair layouts), decode of
several new tokens per sequence packed into one MMA tile (causal and not,
with mods), contiguous caches read through cache_batch_idx, and the
end-to-end update-then-attend call."""
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

F = W.bf16_bits_to_f64


def _round_bf16(x):
    return torch.from_numpy(np.asarray(x, dtype=np.float32)).to(torch.bfloat16).to(torch.float64).numpy()


def _tables(P, R, base=10000.0):
    j = np.arange(R // 2)
    ang = np.arange(P)[:, None] * (base ** (-2.0 * j / R))[None, :]
    return np.cos(ang).astype(np.float32), np.sin(ang).astype(np.float32)


def _gather(cache, bt, page, L):
    """Rows 0 .. L-1 of one sequence from a paged cache [P, page, H, D]."""
    pos = np.arange(L)
    return cache[bt[pos // page], pos % page]


# Rotated values are computed in fp32 and rounded to bf16: within one bf16
# unit in the last place of the fp64 rotation.
def _close_bf16(got, ref, what):
    err = np.abs(got - ref)
    tol = 2.0 ** -7 * np.abs(ref) + 1e-6
    assert (err <= tol).all(), "%s: max excess %.3e" % (what, float((err - tol).max()))


@pytest.mark.parametrize("interleaved,D,R", [(True, 128, 128), (False, 128, 64), (False, 64, 64), (True, 64, 32)])
def test_cache_update_paged_rotary(interleaved, D, R):
    rng = np.random.default_rng(7 + D + R)
    B, Snew, Hq, Hkv, page, P = 3, 5, 8, 2, 64, 24
    kc = W.normal_bf16(300, (P, page, Hkv, D))
    vc = W.normal_bf16(301, (P, page, Hkv, D))
    kn, vn = W.normal_bf16(302, (B, Snew, Hkv, D)), W.normal_bf16(303, (B, Snew, Hkv, D))
    q = W.normal_bf16(304, (B, Snew, Hq, D))
    bt = rng.permutation(P)[:B * 8].reshape(B, 8).astype(np.int32)
    seqlens = np.array([0, 61, 300], np.int32)  # an empty cache, a page boundary inside the update, a long one
    cos, sin = _tables(512, R)
    tk, tv = dev_bf16(kc), dev_bf16(vc)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    new_len = torch.zeros(B, dtype=torch.int32, device="cuda")
    q_out = ea.attn_kvcache_update(tk, tv, torch.from_numpy(seqlens).cuda(), q=dev_bf16(q), k=dev_bf16(kn),
                                   v=dev_bf16(vn), block_table=torch.from_numpy(bt).cuda(),
                                   rotary_cos=torch.from_numpy(cos).cuda(), rotary_sin=torch.from_numpy(sin).cuda(),
                                   rotary_interleaved=interleaved, seqlens_out=new_len, status=status)
    torch.cuda.synchronize()
    assert status.item() == 0
    assert new_len.cpu().numpy().tolist() == (seqlens + Snew).tolist()
    k_ref, v_ref = oracle.kvcache_append(F(kc), F(vc), F(kn), F(vn), seqlens, block_table=bt, page_size=page,
                                         rotary_cos=cos.astype(np.float64), rotary_sin=sin.astype(np.float64),
                                         interleaved=interleaved)
    pos = seqlens[:, None] + np.arange(Snew)[None, :]
    q_ref = oracle.rotary(F(q), cos.astype(np.float64), sin.astype(np.float64), pos, interleaved)
    got_k, got_v = host_f64(tk), host_f64(tv)
    assert np.array_equal(got_v, v_ref)  # v is copied bit for bit, the rest of both caches untouched
    row, slot = oracle.cache_rows(B, Snew, seqlens, block_table=bt, page_size=page)
    touched = np.zeros((P, page), dtype=bool)
    touched[row, slot] = True
    assert np.array_equal(got_k[~touched], F(kc)[~touched])
    _close_bf16(got_k[touched], k_ref[touched], "k rows")
    _close_bf16(host_f64(q_out), q_ref, "q")


def test_cache_update_contiguous_batch_idx_and_errors():
    B, Snew, Hkv, D, Bc, S = 3, 4, 2, 128, 5, 256
    kc, vc = W.normal_bf16(310, (Bc, S, Hkv, D)), W.normal_bf16(311, (Bc, S, Hkv, D))
    kn, vn = W.normal_bf16(312, (B, Snew, Hkv, D)), W.normal_bf16(313, (B, Snew, Hkv, D))
    idx = np.array([4, 0, 2], np.int32)
    seqlens = np.array([10, 0, 200], np.int32)
    tk, tv = dev_bf16(kc), dev_bf16(vc)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    ea.attn_kvcache_update(tk, tv, torch.from_numpy(seqlens).cuda(), k=dev_bf16(kn), v=dev_bf16(vn),
                           cache_batch_idx=torch.from_numpy(idx).cuda(), status=status)
    torch.cuda.synchronize()
    assert status.item() == 0
    k_ref, v_ref = oracle.kvcache_append(F(kc), F(vc), F(kn), F(vn), seqlens, cache_batch_idx=idx)
    assert np.array_equal(host_f64(tk), k_ref) and np.array_equal(host_f64(tv), v_ref)  # no rotary: exact copies
    # a position past the cache is reported and skipped; so is a page id out of range
    status.zero_()
    before = tk.clone()
    ea.attn_kvcache_update(tk, tv, torch.tensor([S - 2, 0, 0], dtype=torch.int32, device="cuda"), k=dev_bf16(kn),
                           v=dev_bf16(vn), cache_batch_idx=torch.tensor([1, 9, 3], dtype=torch.int32, device="cuda"),
                           status=status)
    torch.cuda.synchronize()
    assert status.item() & ea.ATTN_DEV_BAD_LEN and status.item() & ea.ATTN_DEV_BAD_PAGE
    changed = (tk != before).any(dim=3).any(dim=2).cpu().numpy()
    # sequence 0 writes its two positions that fit, sequence 2 its four; sequence 1 nothing
    assert changed[1].sum() == 2 and changed[1, S - 2:].all()
    assert changed[3].sum() == 4 and not changed[0].any() and not changed[2].any() and not changed[4].any()


def _decode_ref(q, kc, vc, bt, page, seqlens, causal, mod=oracle.MOD_NONE, softcap=0.0, alibi=None,
                cache_batch_idx=None):
    """Per sequence: the oracle on the gathered keys, the q_len tokens at the last positions."""
    B, T, Hq, D = q.shape
    o = np.zeros((B, T, Hq, D))
    lse = np.zeros((B, T, Hq))
    for b in range(B):
        L = int(seqlens[b])
        if bt is not None:
            k, v = _gather(kc, bt[b], page, L), _gather(vc, bt[b], page, L)
        else:
            r = b if cache_batch_idx is None else int(cache_batch_idx[b])
            k, v = kc[r, :L], vc[r, :L]
        kw = dict(mod=mod, softcap=softcap, alibi=alibi, q_offset=L - T)
        if causal:
            kw.update(mask=oracle.MASK_CAUSAL, window=(-1, 0))
        ro, rl = oracle.attn_f64(np.ascontiguousarray(q[b:b + 1]), np.ascontiguousarray(k[None]),
                                 np.ascontiguousarray(v[None]), **kw)
        o[b], lse[b] = ro[0], rl[0].T
    return o, lse


@pytest.mark.parametrize("Hq,Hkv,T,causal", [(16, 4, 4, True), (32, 1, 4, True), (12, 2, 3, False), (8, 8, 16, True)])
def test_decode_several_new_tokens(Hq, Hkv, T, causal):
    D, page, P = 128, 64, 64
    rng = np.random.default_rng(Hq + T)
    B = 3
    kc, vc = W.normal_bf16(320, (P, page, Hkv, D)), W.normal_bf16(321, (P, page, Hkv, D))
    q = W.normal_bf16(322, (B, T, Hq, D))
    bt = rng.permutation(P)[:B * 20].reshape(B, 20).astype(np.int32)
    seqlens = np.array([T, 700, 1280], np.int32)  # the first sequence holds only its new tokens
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    o, lse = ea.attn_decode(dev_bf16(q), dev_bf16(kc), dev_bf16(vc), torch.from_numpy(bt).cuda(),
                            torch.from_numpy(seqlens).cuda(), max_seqlen=1280, causal=causal, status=status)
    torch.cuda.synchronize()
    assert status.item() == 0
    o_ref, l_ref = _decode_ref(F(q), F(kc), F(vc), bt, page, seqlens, causal)
    compare(host_f64(o), o_ref, lse.cpu().numpy().astype(np.float64), l_ref, "decode T=%d g=%d" % (T, Hq // Hkv))


def test_decode_several_tokens_with_mods():
    Hq, Hkv, T, D, page, P, B = 16, 2, 5, 128, 128, 40, 2
    rng = np.random.default_rng(9)
    kc, vc = W.normal_bf16(330, (P, page, Hkv, D)), W.normal_bf16(331, (P, page, Hkv, D))
    q = W.normal_bf16(332, (B, T, Hq, D))
    bt = rng.permutation(P)[:B * 12].reshape(B, 12).astype(np.int32)
    seqlens = np.array([1000, 333], np.int32)
    slopes = W.alibi_slopes(Hq)
    for mod, kw in ((oracle.MOD_SOFTCAP, dict(softcap=30.0)),
                    (oracle.MOD_ALIBI, dict(alibi_slopes=torch.from_numpy(slopes).cuda()))):
        o, lse = ea.attn_decode(dev_bf16(q), dev_bf16(kc), dev_bf16(vc), torch.from_numpy(bt).cuda(),
                                torch.from_numpy(seqlens).cuda(), max_seqlen=1536, causal=True, **kw)
        torch.cuda.synchronize()
        o_ref, l_ref = _decode_ref(F(q), F(kc), F(vc), bt, page, seqlens, True, mod=mod, softcap=30.0,
                                   alibi=slopes.astype(np.float64) if mod == oracle.MOD_ALIBI else None)
        compare(host_f64(o), o_ref, lse.cpu().numpy().astype(np.float64), l_ref, "decode mods %d" % mod)


@pytest.mark.parametrize("T", [1, 4])
def test_decode_contiguous_cache_with_batch_idx(T):
    Hq, Hkv, D, Bc, S, B = 8, 2, 128, 4, 900, 3
    kc, vc = W.normal_bf16(340, (Bc, S, Hkv, D)), W.normal_bf16(341, (Bc, S, Hkv, D))
    q = W.normal_bf16(342, (B, T, Hq, D))
    idx = np.array([3, 0, 2], np.int32)
    seqlens = np.array([900, 129, 17], np.int32)
    qd = dev_bf16(q)
    o, lse = ea.attn_decode(qd if T > 1 else qd[:, 0], dev_bf16(kc), dev_bf16(vc), None,
                            torch.from_numpy(seqlens).cuda(), causal=True,
                            cache_batch_idx=torch.from_numpy(idx).cuda())
    torch.cuda.synchronize()
    o_ref, l_ref = _decode_ref(F(q), F(kc), F(vc), None, 0, seqlens, True, cache_batch_idx=idx)
    og = host_f64(o).reshape(B, T, Hq, D)
    compare(og, o_ref, lse.cpu().numpy().astype(np.float64).reshape(B, T, Hq), l_ref, "contiguous T=%d" % T)


@pytest.mark.parametrize("paged", [True, False])
def test_with_kvcache_update_then_attend(paged):
    """flash_attn_with_kvcache in one call: rotate q and the new k, append k/v,
    attend causally over the updated cache."""
    Hq, Hkv, D, B, T, R = 16, 4, 128, 2, 3, 128
    rng = np.random.default_rng(11)
    if paged:
        P, page = 32, 128
        kc, vc = W.normal_bf16(350, (P, page, Hkv, D)), W.normal_bf16(351, (P, page, Hkv, D))
        bt = rng.permutation(P)[:B * 8].reshape(B, 8).astype(np.int32)
        idx = None
    else:
        P, page = 3, 1024
        kc, vc = W.normal_bf16(350, (P, page, Hkv, D)), W.normal_bf16(351, (P, page, Hkv, D))
        bt, idx = None, np.array([2, 0], np.int32)
    q = W.normal_bf16(352, (B, T, Hq, D))
    kn, vn = W.normal_bf16(353, (B, T, Hkv, D)), W.normal_bf16(354, (B, T, Hkv, D))
    seqlens = np.array([255, 700], np.int32)
    cos, sin = _tables(1024, R)
    tk, tv = dev_bf16(kc), dev_bf16(vc)
    o, lse = ea.attn_with_kvcache(dev_bf16(q), tk, tv, torch.from_numpy(seqlens).cuda(), k=dev_bf16(kn),
                                  v=dev_bf16(vn), rotary_cos=torch.from_numpy(cos).cuda(),
                                  rotary_sin=torch.from_numpy(sin).cuda(), rotary_interleaved=False,
                                  block_table=None if bt is None else torch.from_numpy(bt).cuda(),
                                  cache_batch_idx=None if idx is None else torch.from_numpy(idx).cuda(), causal=True)
    torch.cuda.synchronize()
    c64, s64 = cos.astype(np.float64), sin.astype(np.float64)
    k_ref, v_ref = oracle.kvcache_append(F(kc), F(vc), F(kn), F(vn), seqlens, block_table=bt, page_size=page,
                                         cache_batch_idx=idx, rotary_cos=c64, rotary_sin=s64, interleaved=False,
                                         round_bf16=_round_bf16)
    pos = seqlens[:, None] + np.arange(T)[None, :]
    q_ref = _round_bf16(oracle.rotary(F(q), c64, s64, pos, False))
    o_ref, l_ref = _decode_ref(q_ref, k_ref, v_ref, bt, page, seqlens + T, True, cache_batch_idx=idx)
    compare(host_f64(o), o_ref, lse.cpu().numpy().astype(np.float64), l_ref, "with_kvcache paged=%s" % paged)
