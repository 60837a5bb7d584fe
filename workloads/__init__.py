"""Seeded synthetic inputs for the exact-attention forward path.

This module is shared by the CUDA path's tests/bench and by the fp64 oracle's
tests. It holds random-number generation and workload shapes only: none of the
attention arithmetic (scores, masks, softmax, combine) lives here.

Recipe (the same on both sides):
  * PRNG: splitmix64 (Steele, Lea & Flood, "Fast splittable pseudorandom number
    generators", OOPSLA 2014): state_i = seed + (i+1)*0x9E3779B97F4A7C15, then the
    three xor-shift-multiply finalisation rounds.
  * Normals: Box-Muller on pairs of 53-bit uniforms.
  * bf16: float32 rounded to nearest-even bf16; stored as uint16 bit patterns.
  * Document lengths: integers uniform in [lo, hi] (x mod (hi-lo+1)), drawn until
    the running sum reaches the total; the last document is cut to fit.
  * Page table: Fisher-Yates shuffle of all physical page ids, reshaped row-major.

The five workloads mirror the shapes the pages discuss: a tiny MHA case, a
Llama-3.1-8B-shaped causal GQA prefill (FlexAttention memory issue repro,
train_length 2048, 32 query / 8 KV heads), a long-context sliding-window +
softcap case, packed documents with ALiBi under a block mask, and an MQA decode
over a paged KV cache (flash_attn_with_kvcache with block_table).
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import numpy as np

_GOLDEN = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)


def splitmix64(seed: int, n: int, start: int = 0) -> np.ndarray:
    """Return outputs start..start+n-1 of the splitmix64 sequence for `seed`."""
    with np.errstate(over="ignore"):
        idx = np.arange(start + 1, start + n + 1, dtype=np.uint64)
        z = np.uint64(seed & 0xFFFFFFFFFFFFFFFF) + idx * _GOLDEN
        z = (z ^ (z >> np.uint64(30))) * _M1
        z = (z ^ (z >> np.uint64(27))) * _M2
        z = z ^ (z >> np.uint64(31))
    return z


def uniform53(bits: np.ndarray) -> np.ndarray:
    """Map 64-bit words to doubles in [0, 1) with 53 random bits."""
    return (bits >> np.uint64(11)).astype(np.float64) * (1.0 / 9007199254740992.0)


def normal_f32(seed: int, n: int) -> np.ndarray:
    """n standard normals (float32) by Box-Muller from splitmix64(seed)."""
    m = (n + 1) // 2
    out = np.empty(2 * m, dtype=np.float32)
    chunk = 1 << 22
    for c0 in range(0, m, chunk):
        c = min(chunk, m - c0)
        bits = splitmix64(seed, 2 * c, start=2 * c0)
        u1 = 1.0 - uniform53(bits[0::2])  # (0, 1]
        u2 = uniform53(bits[1::2])
        r = np.sqrt(-2.0 * np.log(u1))
        t = 2.0 * math.pi * u2
        out[2 * c0: 2 * c0 + c] = (r * np.cos(t)).astype(np.float32)
        out[2 * c0 + c: 2 * c0 + 2 * c] = (r * np.sin(t)).astype(np.float32)
    # fixed layout per chunk: the c cosine outputs, then the c sine outputs
    return out[:n]


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 to nearest-even bf16; return the uint16 bit patterns."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    u = (u + np.uint64(0x7FFF) + ((u >> np.uint64(16)) & np.uint64(1))) >> np.uint64(16)
    return u.astype(np.uint16)


def bf16_bits_to_f64(b: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns to float64."""
    return (b.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)


def normal_bf16(seed: int, shape) -> np.ndarray:
    """bf16 (uint16 bits) N(0,1) array of the given shape."""
    n = int(np.prod(shape))
    return f32_to_bf16_bits(normal_f32(seed, n)).reshape(shape)


def doc_lengths(seed: int, total: int, lo: int, hi: int) -> list:
    """Document lengths uniform in [lo, hi], last one truncated so they sum to total."""
    lens, s, i = [], 0, 0
    span = hi - lo + 1
    while s < total:
        x = int(splitmix64(seed, 1, start=i)[0])
        i += 1
        L = lo + x % span
        L = min(L, total - s)
        lens.append(L)
        s += L
    return lens


def doc_ids_from_lengths(lens) -> np.ndarray:
    return np.repeat(np.arange(len(lens), dtype=np.int32), lens)


def uniform_ints(seed: int, n: int, lo: int, hi: int) -> np.ndarray:
    """n int32 values uniform in [lo, hi] (splitmix64 modulo the span)."""
    return (lo + splitmix64(seed, n) % np.uint64(hi - lo + 1)).astype(np.int32)


def page_permutation(seed: int, num_pages: int) -> np.ndarray:
    """Fisher-Yates shuffle of range(num_pages) driven by splitmix64(seed)."""
    perm = np.arange(num_pages, dtype=np.int32)
    bits = splitmix64(seed, max(num_pages - 1, 0))
    for t, i in enumerate(range(num_pages - 1, 0, -1)):
        j = int(bits[t] % np.uint64(i + 1))
        perm[i], perm[j] = perm[j], perm[i]
    return perm


# ------------------------------------------------------------------ workloads

MASK_NONE, MASK_CAUSAL, MASK_WINDOW, MASK_DOCUMENT = 0, 1, 2, 3
MOD_NONE, MOD_SOFTCAP, MOD_ALIBI = 0, 1, 2


@dataclasses.dataclass
class Prefill:
    name: str
    B: int
    Hq: int
    Hkv: int
    S: int
    D: int
    mask: int = MASK_NONE
    window_left: int = -1
    window_right: int = -1
    mod: int = MOD_NONE
    softcap: float = 0.0
    doc_range: Optional[tuple] = None  # (lo, hi) for packed documents
    seed: int = 0


@dataclasses.dataclass
class Decode:
    name: str
    B: int
    Hq: int
    Hkv: int
    D: int
    kv_len: int
    page_size: int
    seed: int = 0


def _seed(c: int) -> int:
    return 0xA77E0000 + c


WORKLOADS = {
    "tiny_mha_s128_d64": Prefill("tiny_mha_s128_d64", B=1, Hq=2, Hkv=2, S=128, D=64, seed=_seed(1)),
    "causal_gqa_llama8b_s2048": Prefill("causal_gqa_llama8b_s2048", B=1, Hq=32, Hkv=8, S=2048, D=128,
                                        mask=MASK_CAUSAL, window_left=-1, window_right=0, seed=_seed(2)),
    "window1024_softcap30_s8192": Prefill("window1024_softcap30_s8192", B=2, Hq=16, Hkv=16, S=8192, D=128,
                                          mask=MASK_WINDOW, window_left=1023, window_right=0,
                                          mod=MOD_SOFTCAP, softcap=30.0, seed=_seed(3)),
    "packed_docs_alibi_s16384": Prefill("packed_docs_alibi_s16384", B=1, Hq=32, Hkv=8, S=16384, D=128,
                                        mask=MASK_DOCUMENT, mod=MOD_ALIBI, doc_range=(128, 2048), seed=_seed(4)),
    "mqa_paged_decode_b32_kv32768": Decode("mqa_paged_decode_b32_kv32768", B=32, Hq=128, Hkv=1, D=128,
                                           kv_len=32768, page_size=256, seed=_seed(5)),
}


def alibi_slopes(Hq: int) -> np.ndarray:
    """ALiBi slopes 2^(-8(h+1)/Hq), h = 0..Hq-1, as float32 (the stored input)."""
    h = np.arange(Hq, dtype=np.float64)
    return np.exp2(-8.0 * (h + 1.0) / Hq).astype(np.float32)


def make_prefill_inputs(w: Prefill, S: Optional[int] = None) -> dict:
    """Q, K, V (bf16 bits, BSHD) plus doc ids / slopes for a prefill workload.

    Q, K, V are drawn in that order from consecutive seeds; documents come
    from seed + 0x100. `S` overrides the sequence length (smaller parity cases).
    """
    S = w.S if S is None else S
    q = normal_bf16(w.seed, (w.B, S, w.Hq, w.D))
    k = normal_bf16(w.seed + 1, (w.B, S, w.Hkv, w.D))
    v = normal_bf16(w.seed + 2, (w.B, S, w.Hkv, w.D))
    out = dict(q=q, k=k, v=v, doc_id=None, alibi=None, doc_lens=None)
    if w.mask == MASK_DOCUMENT:
        lo, hi = w.doc_range
        lens = doc_lengths(w.seed + 0x100, S, lo, hi)
        out["doc_lens"] = lens
        out["doc_id"] = doc_ids_from_lengths(lens)
    if w.mod == MOD_ALIBI:
        out["alibi"] = alibi_slopes(w.Hq)
    return out


def make_decode_inputs(w: Decode, B: Optional[int] = None, kv_len: Optional[int] = None,
                       seqlens: Optional[np.ndarray] = None) -> dict:
    """q [B,1,Hq,D], paged k/v caches [num_pages, page, Hkv, D], block_table, cache_seqlens."""
    B = w.B if B is None else B
    kv_len = w.kv_len if kv_len is None else kv_len
    pages_per_seq = (kv_len + w.page_size - 1) // w.page_size
    num_pages = B * pages_per_seq
    q = normal_bf16(w.seed, (B, 1, w.Hq, w.D))
    kc = normal_bf16(w.seed + 1, (num_pages, w.page_size, w.Hkv, w.D))
    vc = normal_bf16(w.seed + 2, (num_pages, w.page_size, w.Hkv, w.D))
    perm = page_permutation(w.seed + 0x100, num_pages)
    block_table = perm.reshape(B, pages_per_seq).astype(np.int32)
    if seqlens is None:
        seqlens = np.full(B, kv_len, dtype=np.int32)
    return dict(q=q, k_cache=kc, v_cache=vc, block_table=block_table,
                cache_seqlens=np.asarray(seqlens, dtype=np.int32))
