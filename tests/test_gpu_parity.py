"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle on
the same seeded inputs. Small cases are compared element by element; the
full-size workloads are compared on sampled rows the oracle computes one by one."""
import numpy as np
import pytest

import oracle
import workloads as W
from tests._gpu_util import compare, dev_bf16, host_f64, sample_rows

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

import exact_attention_145_b200 as ea  # noqa: E402


def run_fwd(q, k, v, **kw):
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    doc = kw.pop("doc_id_np", None)
    alibi = kw.pop("alibi_np", None)
    if doc is not None:
        kw["doc_id"] = torch.from_numpy(doc).cuda()
    if alibi is not None:
        kw["alibi_slopes"] = torch.from_numpy(alibi).cuda()
    o, lse = ea.attn_fwd(dev_bf16(q), dev_bf16(k), dev_bf16(v), status=status, **kw)
    torch.cuda.synchronize()
    assert status.item() == 0, "device status %d" % status.item()
    return host_f64(o), lse.cpu().numpy().astype(np.float64)


def oracle_kw(kw):
    """Translate binding keywords into oracle keywords."""
    ok = {}
    if kw.get("causal"):
        ok["mask"], ok["window"] = W.MASK_CAUSAL, (-1, 0)
    elif kw.get("window") is not None:
        ok["mask"], ok["window"] = W.MASK_WINDOW, kw["window"]
    if kw.get("doc_id_np") is not None:
        ok["mask"], ok["doc_id"] = W.MASK_DOCUMENT, kw["doc_id_np"]
    if kw.get("q_offset"):
        ok["q_offset"] = kw["q_offset"]
    if kw.get("softcap") is not None:
        ok["mod"], ok["softcap"] = W.MOD_SOFTCAP, kw["softcap"]
    if kw.get("alibi_np") is not None:
        ok["mod"], ok["alibi"] = W.MOD_ALIBI, kw["alibi_np"]
    if kw.get("scale") is not None:
        ok["scale"] = kw["scale"]
    return ok


def full_case(B, Sq, Hq, Hkv, D, Skv=None, seed=1, **kw):
    Skv = Sq if Skv is None else Skv
    q = W.normal_bf16(seed, (B, Sq, Hq, D))
    k = W.normal_bf16(seed + 1, (B, Skv, Hkv, D))
    v = W.normal_bf16(seed + 2, (B, Skv, Hkv, D))
    o_ref, lse_ref = oracle.attn(q, k, v, **oracle_kw(kw))
    o, lse = run_fwd(q, k, v, **kw)
    return compare(o, o_ref, lse, lse_ref, what=str((B, Sq, Hq, Hkv, D, Skv, kw.keys())))


# ------------------------------------------------------------ small, element by element

def test_tiny_mha_workload():
    w = W.WORKLOADS["tiny_mha_s128_d64"]
    d = W.make_prefill_inputs(w)
    o_ref, lse_ref = oracle.attn(d["q"], d["k"], d["v"])
    o, lse = run_fwd(d["q"], d["k"], d["v"])
    compare(o, o_ref, lse, lse_ref, "tiny")


@pytest.mark.parametrize("Hq,Hkv", [(8, 8), (8, 2), (6, 2), (4, 1), (3, 3)])
@pytest.mark.parametrize("D", [64, 128])
def test_no_mask_heads_and_dims(Hq, Hkv, D):
    full_case(2, 300, Hq, Hkv, D, seed=10 + Hq + D)


@pytest.mark.parametrize("S", [1, 17, 128, 129, 383, 640])
def test_causal_lengths(S):
    full_case(1, S, 4, 2, 128, seed=20 + S, causal=True)


def test_causal_gqa_medium_all_rows():
    full_case(1, 1000, 8, 2, 128, seed=31, causal=True)


def test_cross_lengths_and_offset():
    full_case(1, 200, 4, 4, 128, Skv=700, seed=41)
    full_case(1, 200, 4, 4, 128, Skv=700, seed=42, causal=True, q_offset=500)
    full_case(2, 90, 2, 1, 64, Skv=333, seed=43, window=(50, 10), q_offset=120)


def test_fully_masked_rows():
    # causal with q_offset = -64: the first 64 query rows see no key at all
    full_case(1, 300, 2, 2, 128, seed=51, causal=True, q_offset=-64)


@pytest.mark.parametrize("window", [(1023, 0), (100, 100), (0, 0), (-1, 37)])
def test_windows_softcap(window):
    full_case(1, 1500, 2, 2, 128, seed=60, window=window, softcap=30.0)


def test_softcap_small_cap():
    full_case(1, 400, 2, 2, 64, seed=61, softcap=2.0, causal=True)


def test_alibi_causal_and_per_batch():
    full_case(1, 700, 8, 2, 128, seed=70, causal=True, alibi_np=W.alibi_slopes(8))
    sl = np.stack([W.alibi_slopes(4), W.alibi_slopes(4)[::-1].copy()]).astype(np.float32)
    full_case(2, 300, 4, 4, 64, seed=71, alibi_np=sl)


def test_documents_alibi_gqa():
    S = 3000
    lens = W.doc_lengths(99, S, 128, 700)
    doc = W.doc_ids_from_lengths(lens)
    full_case(1, S, 8, 2, 128, seed=80, doc_id_np=doc, alibi_np=W.alibi_slopes(8))
    full_case(1, S, 3, 3, 64, seed=81, doc_id_np=doc)


@pytest.mark.parametrize("S", [129, 130, 131, 387])
def test_documents_ragged_tail(S):
    """Sequence lengths that are not a multiple of 4: the last group of
    document ids is partial. Documents start inside the last key tile, so the
    final rows depend on those ids."""
    lens = [S - 3, 1, 2] if S < 200 else [100, 150, S - 250 - 1, 1]
    doc = W.doc_ids_from_lengths(lens)
    full_case(1, S, 4, 2, 128, seed=85 + S, doc_id_np=doc)
    full_case(1, S, 2, 2, 64, seed=86 + S, doc_id_np=doc, alibi_np=W.alibi_slopes(2))


def test_bhsd_strided_inputs():
    B, S, H, D = 2, 260, 4, 128
    q = W.normal_bf16(90, (B, H, S, D))
    k = W.normal_bf16(91, (B, H, S, D))
    v = W.normal_bf16(92, (B, H, S, D))
    tq, tk, tv = (dev_bf16(x).transpose(1, 2) for x in (q, k, v))  # BSHD views of BHSD storage
    o, lse = ea.attn_fwd(tq, tk, tv, causal=True)
    torch.cuda.synchronize()
    qs, ks, vs = (np.ascontiguousarray(x.transpose(0, 2, 1, 3)) for x in (q, k, v))
    o_ref, lse_ref = oracle.attn(qs, ks, vs, mask=W.MASK_CAUSAL, window=(-1, 0))
    compare(host_f64(o), o_ref, lse.cpu().numpy().astype(np.float64), lse_ref, "bhsd")


def test_explicit_scale():
    full_case(1, 256, 2, 2, 128, seed=95, scale=0.3, causal=True)


# ------------------------------------------------------------ block mask builder (exact)

def _bm_compare(bm, ref, b=0, h=0):
    """Slice (b, h) of a device block mask against the oracle's tables."""
    cls = bm.cls.cpu().numpy()[b, h]
    assert np.array_equal(cls, ref["cls"])
    pc, fc = bm.part_cnt.cpu().numpy()[b, h], bm.full_cnt.cpu().numpy()[b, h]
    assert np.array_equal(pc, ref["part_cnt"]) and np.array_equal(fc, ref["full_cnt"])
    pi, fi = bm.part_idx.cpu().numpy()[b, h], bm.full_idx.cpu().numpy()[b, h]
    for r in range(cls.shape[0]):
        assert np.array_equal(pi[r, :pc[r]], ref["part_idx"][r, :pc[r]])
        assert np.array_equal(fi[r, :fc[r]], ref["full_idx"][r, :fc[r]])


@pytest.mark.parametrize("name", ["causal_gqa_llama8b_s2048", "window1024_softcap30_s8192",
                                  "packed_docs_alibi_s16384"])
def test_block_mask_full_size_exact(name):
    w = W.WORKLOADS[name]
    S = w.S
    doc = None
    if w.mask == W.MASK_DOCUMENT:
        doc = W.doc_ids_from_lengths(W.doc_lengths(w.seed + 0x100, S, *w.doc_range))
    ref = oracle.block_mask(w.mask, S, S, window=(w.window_left, w.window_right), doc_id=doc)
    bm = ea.attn_build_block_mask(S, S, causal=w.mask == W.MASK_CAUSAL,
                                  window=(w.window_left, w.window_right) if w.mask == W.MASK_WINDOW else None,
                                  doc_id=None if doc is None else torch.from_numpy(doc).cuda())
    torch.cuda.synchronize()
    _bm_compare(bm, ref)


@pytest.mark.parametrize("Sq,Skv,blk", [(300, 300, 128), (1000, 555, 64), (77, 1200, 16)])
def test_block_mask_ragged_exact(Sq, Skv, blk):
    for kind, window, q_off in [(W.MASK_CAUSAL, (-1, 0), 0), (W.MASK_WINDOW, (90, 7), 13), (W.MASK_NONE, (-1, -1), 0)]:
        ref = oracle.block_mask(kind, Sq, Skv, blk, blk, window=window, q_offset=q_off)
        bm = ea.attn_build_block_mask(Sq, Skv, causal=kind == W.MASK_CAUSAL,
                                      window=window if kind == W.MASK_WINDOW else None, q_offset=q_off,
                                      blk_q=blk, blk_kv=blk)
        torch.cuda.synchronize()
        _bm_compare(bm, ref)


@pytest.mark.parametrize("S,blk,ids", [(1000, 64, "sorted"), (777, 16, "unsorted"), (1500, 128, "unsorted"),
                                       (2048, 128, "two"), (300, 128, "one")])
def test_block_mask_document_exact(S, blk, ids):
    """Document classes: tiles decided from id ranges (sorted, one or two
    documents) and tiles evaluated pair by pair (unsorted ids mix every tile)."""
    if ids == "sorted":
        doc = W.doc_ids_from_lengths(W.doc_lengths(99, S, 20, 300))
    elif ids == "unsorted":
        doc = W.uniform_ints(123 + S, S, 0, 3)
    elif ids == "two":
        doc = np.zeros(S, np.int32)
        doc[S // 3:] = 1
    else:
        doc = np.full(S, 7, np.int32)
    ref = oracle.block_mask(W.MASK_DOCUMENT, S, S, blk, blk, doc_id=doc)
    bm = ea.attn_build_block_mask(S, S, doc_id=torch.from_numpy(doc).cuda(), blk_q=blk, blk_kv=blk)
    torch.cuda.synchronize()
    _bm_compare(bm, ref)


@pytest.mark.parametrize("window,q_off", [((0, 0), 0), ((0, 0), -5), ((3, 40), 200), ((-1, 5), -300), ((200, -1), 0)])
def test_block_mask_window_edges_exact(window, q_off):
    """Interval classification at narrow bands, offsets that push rows off the key range, one-sided windows."""
    for Sq, Skv, blk in [(500, 700, 64), (129, 128, 16), (1024, 1024, 128)]:
        ref = oracle.block_mask(W.MASK_WINDOW, Sq, Skv, blk, blk, window=window, q_offset=q_off)
        bm = ea.attn_build_block_mask(Sq, Skv, window=window, q_offset=q_off, blk_q=blk, blk_kv=blk)
        torch.cuda.synchronize()
        _bm_compare(bm, ref)


def test_block_mask_per_batch_documents_and_head_slices_exact():
    """Bm = 2 batches with different document layouts, Hm = 3 head slices: each
    slice equals the oracle's tables for its batch's document row."""
    S = 1500
    doc = np.stack([W.doc_ids_from_lengths(W.doc_lengths(7, S, 60, 500)),
                    W.doc_ids_from_lengths(W.doc_lengths(8, S, 200, 900))])
    bm = ea.attn_build_block_mask(S, S, doc_id=torch.from_numpy(doc).cuda(), H=3)
    torch.cuda.synchronize()
    assert bm.shape[:2] == (2, 3)
    for b in range(2):
        ref = oracle.block_mask(W.MASK_DOCUMENT, S, S, doc_id=doc[b])
        for h in range(3):
            _bm_compare(bm, ref, b, h)
    # window mask with head slices (no batch dependence): every slice equal
    bm = ea.attn_build_block_mask(1000, 1000, window=(300, 0), B=2, H=2)
    torch.cuda.synchronize()
    ref = oracle.block_mask(W.MASK_WINDOW, 1000, 1000, window=(300, 0))
    for b in range(2):
        for h in range(2):
            _bm_compare(bm, ref, b, h)


def _runs_and_order(doc_row, ref):
    """Document run starts, the never-decreasing flag and the heaviest-first
    q-tile order, from their definitions (host reference for the builder)."""
    S = len(doc_row)
    start = np.zeros(S, np.int32)
    for i in range(1, S):
        start[i] = start[i - 1] if doc_row[i] == doc_row[i - 1] else i
    sorted_ = int(np.all(np.diff(doc_row) >= 0))
    wgt = ref["part_cnt"] + ref["full_cnt"]
    order = np.array(sorted(range(len(wgt)), key=lambda i: (-wgt[i], i)), np.int32)
    return start, sorted_, order


@pytest.mark.parametrize("ids", ["sorted", "unsorted"])
def test_block_mask_document_runs_and_work_order_exact(ids):
    S = 3001
    if ids == "sorted":
        doc = np.stack([W.doc_ids_from_lengths(W.doc_lengths(27, S, 100, 900)),
                        W.doc_ids_from_lengths(W.doc_lengths(28, S, 30, 200))])
    else:
        doc = np.stack([W.uniform_ints(29, S, 0, 3), W.doc_ids_from_lengths(W.doc_lengths(30, S, 30, 200))])
    bm = ea.attn_build_block_mask(S, S, doc_id=torch.from_numpy(doc).cuda())
    torch.cuda.synchronize()
    for b in range(2):
        ref = oracle.block_mask(W.MASK_DOCUMENT, S, S, doc_id=doc[b])
        start, sorted_, order = _runs_and_order(doc[b], ref)
        assert np.array_equal(bm.doc_start.cpu().numpy()[b], start)
        assert int(bm.doc_sorted.cpu().numpy()[b]) == sorted_
        assert np.array_equal(bm.row_order.cpu().numpy()[b], order)
    assert int(bm.doc_sorted.cpu().numpy()[0]) == (1 if ids == "sorted" else 0)


@pytest.mark.parametrize("S", [777, 1030])
def test_documents_unsorted_ids_forward(S):
    """Ids that go up and down (every position compared by id, the path for
    documents that are not one run each), ragged lengths included."""
    doc = W.uniform_ints(31 + S, S, 0, 2)
    full_case(1, S, 4, 2, 128, seed=87 + S, doc_id_np=doc)
    full_case(1, S, 2, 2, 64, seed=88 + S, doc_id_np=doc, alibi_np=W.alibi_slopes(2))


def test_per_batch_documents_forward():
    """B = 2 packed-document batches with different layouts through attn_fwd
    (doc_id [B, S], block mask with Bm = 2), GQA and ALiBi, against the oracle."""
    S = 1300
    doc = np.stack([W.doc_ids_from_lengths(W.doc_lengths(17, S, 128, 700)),
                    W.doc_ids_from_lengths(W.doc_lengths(18, S, 40, 300))])
    full_case(2, S, 8, 2, 128, seed=88, doc_id_np=doc, alibi_np=W.alibi_slopes(8))
    full_case(2, S, 3, 3, 64, seed=89, doc_id_np=doc)


def test_per_head_block_sparse_tables_filled_by_the_caller():
    """A caller-filled block mask with Hm = Hq over MASK_NONE: heads 0 and 2
    attend block-causally (every key of tiles up to the query's own tile),
    heads 1 and 3 to every key. The oracle computes each row over its allowed
    key range (kv_range), the plain definition on a key subset."""
    B, S, Hq, Hkv, D = 1, 700, 4, 2, 128
    nT = -(-S // 128)
    cls = np.zeros((1, Hq, nT, nT), np.uint8)
    for h in range(Hq):
        for i in range(nT):
            for j in range(nT):
                full = j < nT - 1 or S % 128 == 0
                allowed = (j <= i) if h % 2 == 0 else True
                cls[0, h, i, j] = 0 if not allowed else (2 if full else 1)
    bm = ea.BlockMask(S, S, 128, 128, torch.device("cuda"), Bm=1, Hm=Hq)
    bm.cls.copy_(torch.from_numpy(cls))
    pc = (cls == 1).sum(-1).astype(np.int32)
    fc = (cls == 2).sum(-1).astype(np.int32)
    pi = np.zeros(cls.shape, np.int32)
    fi = np.zeros(cls.shape, np.int32)
    for h in range(Hq):
        for i in range(nT):
            p_, f_ = np.nonzero(cls[0, h, i] == 1)[0], np.nonzero(cls[0, h, i] == 2)[0]
            pi[0, h, i, :len(p_)] = p_
            fi[0, h, i, :len(f_)] = f_
    for name, arr in (("part_cnt", pc), ("full_cnt", fc), ("part_idx", pi), ("full_idx", fi)):
        getattr(bm, name).copy_(torch.from_numpy(arr))
    q = W.normal_bf16(91, (B, S, Hq, D))
    k = W.normal_bf16(92, (B, S, Hkv, D))
    v = W.normal_bf16(93, (B, S, Hkv, D))
    o_plain, l_plain = oracle.attn(q, k, v)
    ref_o = np.empty((S, Hq, D))
    ref_l = np.empty((Hq, S))
    for h in range(Hq):
        for i in range(S):
            if h % 2 == 1:
                ref_o[i, h], ref_l[h, i] = o_plain[0, i, h], l_plain[0, h, i]
            else:
                ro, rl = oracle.attn(q, k, v, rows=np.array([[0, h, i]]), kv_range=(0, min(S, (i // 128 + 1) * 128)))
                ref_o[i, h], ref_l[h, i] = ro[0], rl[0]
    # no work order (NULL), then an explicit permutation of the q-tiles
    bm.c.row_order = None
    o, lse = run_fwd(q, k, v, block_mask=bm)
    compare(o[0], ref_o, lse[0], ref_l, "per-head tables, no order")
    bm2 = ea.attn_build_block_mask(S, S, device=torch.device("cuda"))  # only its order table is used
    bm.c.row_order = bm2.c.row_order
    bm2.row_order.copy_(torch.tensor([[3, 0, 5, 1, 4, 2]], dtype=torch.int32))
    o, lse = run_fwd(q, k, v, block_mask=bm)
    compare(o[0], ref_o, lse[0], ref_l, "per-head tables, permuted order")
    # an order entry outside the q-tiles is reported and not followed
    bm2.row_order.copy_(torch.tensor([[3, 0, 99, 1, 4, 2]], dtype=torch.int32))
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    o3, _ = ea.attn_fwd(dev_bf16(q), dev_bf16(k), dev_bf16(v), block_mask=bm, status=status)
    torch.cuda.synchronize()
    assert status.item() & ea.ATTN_DEV_BAD_MASK


def test_block_mask_drives_causal_like_analytic():
    S = 900
    q = W.normal_bf16(101, (1, S, 4, 128))
    k = W.normal_bf16(102, (1, S, 2, 128))
    v = W.normal_bf16(103, (1, S, 2, 128))
    bm = ea.attn_build_block_mask(S, S, causal=True)
    o1, l1 = ea.attn_fwd(dev_bf16(q), dev_bf16(k), dev_bf16(v), causal=True, block_mask=bm)
    o2, l2 = ea.attn_fwd(dev_bf16(q), dev_bf16(k), dev_bf16(v), causal=True)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


# ------------------------------------------------------------ decode

def run_decode(d, Hkv, **kw):
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    alibi = kw.pop("alibi_np", None)
    if alibi is not None:
        kw["alibi_slopes"] = torch.from_numpy(alibi).cuda()
    o, lse = ea.attn_decode(dev_bf16(d["q"]), dev_bf16(d["k_cache"]), dev_bf16(d["v_cache"]),
                            torch.from_numpy(d["block_table"]).cuda(), torch.from_numpy(d["cache_seqlens"]).cuda(),
                            status=status, **kw)
    torch.cuda.synchronize()
    return host_f64(o), lse.cpu().numpy().astype(np.float64), status.item()


@pytest.mark.parametrize("page", [16, 64, 128, 256])
def test_decode_pages_and_ragged_lengths(page):
    w = W.Decode("t", B=5, Hq=16, Hkv=2, D=128, kv_len=2000, page_size=page, seed=110 + page)
    seqlens = np.array([2000, 1, 777, 128, 1300], np.int32)
    d = W.make_decode_inputs(w, seqlens=seqlens)
    o_ref, lse_ref = oracle.decode(d["q"], d["k_cache"], d["v_cache"], d["block_table"], d["cache_seqlens"])
    o, lse, st = run_decode(d, 2, max_seqlen=2000)
    assert st == 0
    compare(o, o_ref, lse, lse_ref, "decode page %d" % page)


@pytest.mark.parametrize("splits", [1, 3, 7, 0])
def test_decode_mqa_splits(splits):
    w = W.Decode("t", B=3, Hq=128, Hkv=1, D=128, kv_len=4096 + 100, page_size=256, seed=120)
    d = W.make_decode_inputs(w)
    o_ref, lse_ref = oracle.decode(d["q"], d["k_cache"], d["v_cache"], d["block_table"], d["cache_seqlens"])
    o, lse, st = run_decode(d, 1, num_splits=splits)
    assert st == 0
    compare(o, o_ref, lse, lse_ref, "decode splits %d" % splits)


def test_decode_mods_and_d64():
    w = W.Decode("t", B=2, Hq=8, Hkv=8, D=64, kv_len=600, page_size=64, seed=130)
    d = W.make_decode_inputs(w, seqlens=np.array([600, 333], np.int32))
    o_ref, lse_ref = oracle.decode(d["q"], d["k_cache"], d["v_cache"], d["block_table"], d["cache_seqlens"],
                                   mod=W.MOD_SOFTCAP, softcap=15.0)
    o, lse, st = run_decode(d, 8, softcap=15.0)
    compare(o, o_ref, lse, lse_ref, "decode softcap")
    sl = W.alibi_slopes(8)
    o_ref, lse_ref = oracle.decode(d["q"], d["k_cache"], d["v_cache"], d["block_table"], d["cache_seqlens"],
                                   mod=W.MOD_ALIBI, alibi=sl)
    o, lse, st = run_decode(d, 8, alibi_np=sl)
    compare(o, o_ref, lse, lse_ref, "decode alibi")


@pytest.mark.parametrize("Hq,Hkv", [(128, 1), (8, 2)])
@pytest.mark.parametrize("mod", ["alibi", "softcap"])
def test_decode_mods_grouped_heads(Hq, Hkv, mod):
    """Score mods when several query heads share a KV head: in decode each MMA
    row is a different query head (row r of KV head hk is head hk*g + r), so the
    ALiBi slope must follow the row. MQA (g = 128) and GQA (g = 4)."""
    w = W.Decode("t", B=3, Hq=Hq, Hkv=Hkv, D=128, kv_len=1500, page_size=128, seed=135 + Hq + Hkv)
    d = W.make_decode_inputs(w, seqlens=np.array([1500, 700, 129], np.int32))
    if mod == "alibi":
        sl = W.alibi_slopes(Hq)
        okw, kw = dict(mod=W.MOD_ALIBI, alibi=sl), dict(alibi_np=sl)
    else:
        okw, kw = dict(mod=W.MOD_SOFTCAP, softcap=5.0), dict(softcap=5.0)
    o_ref, lse_ref = oracle.decode(d["q"], d["k_cache"], d["v_cache"], d["block_table"], d["cache_seqlens"], **okw)
    o, lse, st = run_decode(d, Hkv, **kw)
    assert st == 0
    compare(o, o_ref, lse, lse_ref, "decode %s g=%d" % (mod, Hq // Hkv))


def test_decode_length_above_max_seqlen_is_reported_and_clamped():
    """A cache_seqlens entry above max_seqlen (or negative) sets ATTN_DEV_BAD_LEN;
    the other sequences stay exact and the bad one is computed over its first
    max_seqlen keys. Made on the host: nothing faults."""
    w = W.Decode("t", B=3, Hq=8, Hkv=1, D=128, kv_len=1024, page_size=128, seed=145)
    d = W.make_decode_inputs(w, seqlens=np.array([1024, 600, 300], np.int32))
    o, lse, st = run_decode(d, 1, max_seqlen=600)
    assert st & ea.ATTN_DEV_BAD_LEN and not st & ea.ATTN_DEV_BAD_PAGE
    clamped = d["cache_seqlens"].copy()
    clamped[0] = 600
    o_ref, lse_ref = oracle.decode(d["q"], d["k_cache"], d["v_cache"], d["block_table"], clamped)
    compare(o, o_ref, lse, lse_ref, "decode clamped")
    d2 = dict(d, cache_seqlens=np.array([-5, 600, 300], np.int32))
    o, lse, st = run_decode(d2, 1, max_seqlen=600)
    assert st & ea.ATTN_DEV_BAD_LEN
    assert np.all(o[0] == 0) and np.all(lse[0] == -np.inf)
    o_ref, lse_ref = oracle.decode(d["q"], d["k_cache"], d["v_cache"], d["block_table"], d["cache_seqlens"])
    compare(o[1:], o_ref[1:], lse[1:], lse_ref[1:], "decode negative length")
    # within bounds: no report
    _, _, st = run_decode(d, 1, max_seqlen=1024)
    assert st == 0


def test_decode_zero_length_sequence():
    w = W.Decode("t", B=2, Hq=4, Hkv=1, D=128, kv_len=300, page_size=128, seed=140)
    d = W.make_decode_inputs(w, seqlens=np.array([0, 300], np.int32))
    o, lse, st = run_decode(d, 1)
    assert st == 0
    assert np.all(o[0] == 0) and np.all(lse[0] == -np.inf)
    o_ref, lse_ref = oracle.decode(d["q"], d["k_cache"], d["v_cache"], d["block_table"], d["cache_seqlens"])
    compare(o[1:], o_ref[1:], lse[1:], lse_ref[1:], "decode len 0")


def test_decode_bad_page_id_sets_status_without_fault():
    w = W.Decode("t", B=2, Hq=8, Hkv=1, D=128, kv_len=512, page_size=128, seed=150)
    d = W.make_decode_inputs(w)
    d["block_table"] = d["block_table"].copy()
    d["block_table"][1, 2] = 10_000_000
    o, lse, st = run_decode(d, 1)
    assert st & ea.ATTN_DEV_BAD_PAGE
    assert np.isfinite(o).all()


def test_lse_combine_entry_point():
    rng = np.random.default_rng(5)
    rows, n, D = 37, 5, 128
    op = rng.standard_normal((rows, n, D)).astype(np.float32)
    lp = (rng.standard_normal((rows, n)) * 3).astype(np.float32)
    lp[3, :] = -np.inf
    lp[4, 1] = -np.inf
    o, lse = ea.attn_lse_combine(torch.from_numpy(op).cuda(), torch.from_numpy(lp).cuda())
    torch.cuda.synchronize()
    o, lse = host_f64(o), lse.cpu().numpy().astype(np.float64)
    for r in range(rows):
        oo, ll = oracle.lse_combine(lp[r].astype(np.float64), op[r].astype(np.float64))
        if ll == -np.inf:
            assert lse[r] == -np.inf and np.all(o[r] == 0)
        else:
            assert abs(lse[r] - ll) < 1e-5 and np.max(np.abs(o[r] - oo)) < 2e-2


# ------------------------------------------------------------ full-size workloads, sampled rows

def _full_prefill(name, n_rows=384):
    w = W.WORKLOADS[name]
    d = W.make_prefill_inputs(w)
    kw = {}
    if w.mask == W.MASK_CAUSAL:
        kw["causal"] = True
    if w.mask == W.MASK_WINDOW:
        kw["window"] = (w.window_left, w.window_right)
    if w.mask == W.MASK_DOCUMENT:
        kw["doc_id_np"] = d["doc_id"]
    if w.mod == W.MOD_SOFTCAP:
        kw["softcap"] = w.softcap
    if w.mod == W.MOD_ALIBI:
        kw["alibi_np"] = d["alibi"]
    o, lse = run_fwd(d["q"], d["k"], d["v"], **dict(kw))
    rng = np.random.default_rng(w.seed)
    extra = [127, 128, 255, 256, w.S // 2]
    if d["doc_lens"] is not None:
        ends = np.cumsum(d["doc_lens"])
        extra += [int(e) for e in ends[:6]] + [int(e) - 1 for e in ends[:6]]
    rows = sample_rows(rng, w.B, w.Hq, w.S, n_rows, extra)
    o_ref, lse_ref = oracle.attn(d["q"], d["k"], d["v"], rows=rows, **oracle_kw(kw))
    o_s = np.stack([o[b, i, h] for b, h, i in rows])
    l_s = np.array([lse[b, h, i] for b, h, i in rows])
    return compare(o_s, o_ref, l_s, lse_ref, name)


def test_full_causal_gqa_llama8b_sampled():
    _full_prefill("causal_gqa_llama8b_s2048")


def test_full_window_softcap_sampled():
    _full_prefill("window1024_softcap30_s8192")


def test_full_packed_docs_alibi_sampled():
    _full_prefill("packed_docs_alibi_s16384")


def test_full_mqa_paged_decode_sampled_sequences():
    w = W.WORKLOADS["mqa_paged_decode_b32_kv32768"]
    d = W.make_decode_inputs(w)
    o, lse, st = run_decode(d, w.Hkv, max_seqlen=w.kv_len)
    assert st == 0
    pick = [0, 13, 31]
    sub = dict(q=d["q"][pick], k_cache=d["k_cache"], v_cache=d["v_cache"], block_table=d["block_table"][pick],
               cache_seqlens=d["cache_seqlens"][pick])
    o_ref, lse_ref = oracle.decode(sub["q"], sub["k_cache"], sub["v_cache"], sub["block_table"], sub["cache_seqlens"])
    compare(o[pick], o_ref, lse[pick], lse_ref, "full decode")


# ------------------------------------------------------------ 256 x 128 tables

@pytest.mark.parametrize("S,Hq,Hkv,docs", [(300, 4, 2, None), (1000, 8, 2, [300, 77, 500, 123]),
                                            (900, 3, 1, [450, 450]), (700, 2, 2, None)])
def test_block_mask_256_row_tables(S, Hq, Hkv, docs):
    """A 256 x 128 table (one row per two-subtile CTA, the talk's Blackwell
    block-sparse granularity) gives the same result as the 128 x 128 table
    and the oracle; odd tile counts leave an empty unit, odd groups use the
    256-row single-head units."""
    q, k, v = (W.normal_bf16(500 + S, (1, S, Hq, 128)), W.normal_bf16(501 + S, (1, S, Hkv, 128)),
               W.normal_bf16(502 + S, (1, S, Hkv, 128)))
    kw, okw = {}, {}
    if docs is None:
        kw["causal"] = True
        okw = dict(mask=oracle.MASK_CAUSAL, window=(-1, 0))
        bm256 = ea.attn_build_block_mask(S, S, causal=True, blk_q=256, blk_kv=128, device=torch.device("cuda"))
        bm128 = ea.attn_build_block_mask(S, S, causal=True, device=torch.device("cuda"))
    else:
        doc = W.doc_ids_from_lengths(docs)
        kw["doc_id"] = torch.from_numpy(doc).cuda()
        okw = dict(mask=oracle.MASK_DOCUMENT, doc_id=doc)
        bm256 = ea.attn_build_block_mask(S, S, doc_id=kw["doc_id"], blk_q=256, blk_kv=128)
        bm128 = ea.attn_build_block_mask(S, S, doc_id=kw["doc_id"])
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    o1, l1 = ea.attn_fwd(dev_bf16(q), dev_bf16(k), dev_bf16(v), block_mask=bm256, status=status, **kw)
    o2, l2 = ea.attn_fwd(dev_bf16(q), dev_bf16(k), dev_bf16(v), block_mask=bm128, **kw)
    torch.cuda.synchronize()
    assert status.item() == 0
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
    ro, rl = oracle.attn(q, k, v, **okw)
    compare(host_f64(o1)[0], ro[0], l1.cpu().numpy().astype(np.float64)[0], rl[0], "256-row table S=%d" % S)
