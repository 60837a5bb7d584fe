"""Host-side logic that needs no GPU: the decode split heuristic exported by
the library and the bench's kernel-code digest (which decides whether the
recorded DRAM traffic still describes the kernel)."""
import pytest

from exact_attention_145_b200 import _lib
from exact_attention_145_b200.build import build

import bench


@pytest.fixture(scope="module")
def lib():
    build()
    return _lib.load()


def test_decode_splits_fill_one_wave_when_they_can(lib):
    # 32 sequences x 1 KV head: 4 splits give 128 units, one wave of 148 SMs
    assert lib.attn_decode_num_splits(32, 128, 1, 32768, 0) == 4
    # a few long sequences: as many splits as fit one wave
    assert lib.attn_decode_num_splits(4, 128, 1, 32768, 0) == 37
    # sequences already fill the GPU: no split
    assert lib.attn_decode_num_splits(148, 128, 1, 2048, 0) == 1
    assert lib.attn_decode_num_splits(64, 64, 8, 4096, 0) == 1


def test_decode_explicit_splits_are_clamped_to_key_tiles(lib):
    assert lib.attn_decode_num_splits(2, 8, 1, 1000, 5) == 5
    assert lib.attn_decode_num_splits(2, 8, 1, 1000, 64) == 8  # 1000 keys = 8 tiles of 128
    assert lib.attn_decode_num_splits(0, 8, 1, 1000, 0) == 1


def test_code_digest_ignores_comments_and_whitespace_only():
    a = "int f(int x) {\n  return x + 1;  // one more\n}\n"
    b = "/* header */ int f(int x) { return x + 1; }"
    c = "int f(int x) { return x + 2; }"
    assert bench.code_digest(a) == bench.code_digest(b)
    assert bench.code_digest(a) != bench.code_digest(c)


@pytest.mark.parametrize("name", ["tiny_mha_s128_d64", "causal_gqa_llama8b_s2048", "window1024_softcap30_s8192",
                                  "packed_docs_alibi_s16384"])
def test_bench_flop_accounting_matches_the_oracle_pair_count(name):
    """bench.py's closed-form pair counts (the FLOP numerator of every
    TFLOP/s figure) against the oracle's brute-force count, on the workloads'
    own masks at a reduced length where the workload allows it."""
    import oracle
    import workloads as W
    w = W.WORKLOADS[name]
    S = min(w.S, 3000)
    ws = W.Prefill(**{**w.__dict__, "S": S})
    doc_lens = None
    kw = {}
    if w.mask == W.MASK_CAUSAL:
        kw = dict(window=(-1, 0))
    elif w.mask == W.MASK_WINDOW:
        kw = dict(window=(w.window_left, w.window_right))
    elif w.mask == W.MASK_DOCUMENT:
        doc_lens = W.doc_lengths(w.seed + 0x100, S, *w.doc_range)
        kw = dict(doc_id=W.doc_ids_from_lengths(doc_lens))
    per_head = oracle.count_pairs(w.mask, S, S, **kw)
    assert bench.unmasked_pairs(ws, doc_lens) == per_head * w.B * w.Hq


def test_trace_summary_on_synthetic_records():
    """The cycle-trace summarizer (trace build analysis) on a hand-made record
    stream: one CTA, two units of 2 and 1 steps on subtile 0."""
    import numpy as np
    from exact_attention_145_b200 import trace as T
    E = T.EV
    per = 64
    raw = np.zeros((1, T.N_ROLES, per, 2), np.uint32)

    def put(role, recs):
        for i, (t, e, aux) in enumerate(recs):
            raw[0, role, i] = (t, (e << 24) | aux)

    put(0, [(10, E["S_WAIT"], 0), (100, E["S_READY"], 0 | (2 << 20)), (1100, E["P_DONE"], 0),
            (1110, E["S_WAIT"], 1), (2000, E["S_READY"], 1 | (1 << 20)), (3500, E["P_DONE"], 1),
            (3510, E["O_WAIT"], 0), (3800, E["EPI_BEGIN"], 0), (4400, E["EPI_END"], 0),
            (4410, E["S_WAIT"], 2), (6000, E["S_READY"], 2 | (2 << 20)), (7000, E["P_DONE"], 2),
            (7010, E["O_WAIT"], 1), (7300, E["EPI_BEGIN"], 1), (7900, E["EPI_END"], 1),
            (8000, E["KERNEL_END"], 0)])
    put(T.MMA, [(900, E["P_WAIT"], 0), (1150, E["PV"], 0)])
    # warps 1-3 of subtile 0 hand over P of step 0 later than warp 0
    for w, late in ((1, 40), (2, 300), (3, 10)):
        put(w, [(1100 + late, E["P_DONE"], 0)])
    s = T.summarize(T.decode_records(raw, 1, per))
    assert s["prologue_to_first_s"] == 100
    assert s["softmax_full_tile"] == 1000 and s["softmax_partial_tile"] == 1500
    assert s["p_to_next_s"] == 900 and s["step_period_per_subtile"] == 1900
    assert s["unit_boundary"] == 6000 - 3500
    assert s["epilogue"] == 600 and s["o_wait_before_epilogue"] == 290
    assert s["mma_wait_for_p"] == 250
    assert s["p_handover_skew_across_warps"] == 300
    assert s["critical_cta"] == {"cycles": 8000, "steps": 3, "units": 2}
