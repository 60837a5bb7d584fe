"""Pins of the oracle's kv-cache update (rotary embedding and in-place append,
FlashAttention overview, "Examples": flash_attn_with_kvcache) against hand
results and properties the mathematics fixes: a plane rotation by a known
angle, the identity at angle 0, composition of rotations, norm preservation,
the permutation between the interleaved and the half layouts, and the cache
rows a paged and a batch-indexed cache give."""
import math

import numpy as np
import pytest

import oracle


def _tables(P, R, base=10000.0):
    j = np.arange(R // 2)
    theta = base ** (-2.0 * j / R)
    ang = np.arange(P)[:, None] * theta[None, :]
    return np.cos(ang), np.sin(ang)


def test_rotary_hand_examples():
    x = np.array([1.0, 2.0, 5.0, 7.0]).reshape(1, 1, 1, 4)
    pos = np.zeros((1, 1), dtype=np.int64)
    # interleaved, rotary_dim 2: pair (x0, x1) rotated by cos 0.6 / sin 0.8, the rest unchanged
    got = oracle.rotary(x, np.array([[0.6]]), np.array([[0.8]]), pos, True).ravel()
    assert np.allclose(got, [1 * 0.6 - 2 * 0.8, 1 * 0.8 + 2 * 0.6, 5.0, 7.0], atol=1e-15)
    # half layout, rotary_dim 4: pairs (x0, x2) by (0.6, 0.8) and (x1, x3) by a quarter turn
    got = oracle.rotary(x, np.array([[0.6, 0.0]]), np.array([[0.8, 1.0]]), pos, False).ravel()
    assert np.allclose(got, [1 * 0.6 - 5 * 0.8, 2 * 0.0 - 7 * 1.0, 1 * 0.8 + 5 * 0.6, 2 * 1.0 + 7 * 0.0], atol=1e-15)


@pytest.mark.parametrize("interleaved", [True, False])
def test_rotary_identity_norm_and_composition(interleaved):
    rng = np.random.default_rng(3)
    B, T, H, D, R = 2, 5, 3, 16, 12
    cos, sin = _tables(64, R)
    x = rng.standard_normal((B, T, H, D))
    zero = np.zeros((B, T), dtype=np.int64)
    assert np.array_equal(oracle.rotary(x, cos, sin, zero, interleaved), x)
    p1 = rng.integers(0, 30, size=(B, T))
    p2 = rng.integers(0, 30, size=(B, T))
    y = oracle.rotary(x, cos, sin, p1, interleaved)
    # dims past rotary_dim untouched, each rotated pair keeps its length
    assert np.array_equal(y[..., R:], x[..., R:])
    if interleaved:
        n0 = x[..., 0:R:2] ** 2 + x[..., 1:R:2] ** 2
        n1 = y[..., 0:R:2] ** 2 + y[..., 1:R:2] ** 2
    else:
        n0 = x[..., :R // 2] ** 2 + x[..., R // 2:R] ** 2
        n1 = y[..., :R // 2] ** 2 + y[..., R // 2:R] ** 2
    assert np.allclose(n0, n1, rtol=1e-13)
    # R(p2) R(p1) = R(p1 + p2) for tables cos / sin of theta_j * p
    assert np.allclose(oracle.rotary(y, cos, sin, p2, interleaved), oracle.rotary(x, cos, sin, p1 + p2, interleaved),
                       atol=1e-12)


def test_rotary_layouts_are_a_permutation_apart():
    rng = np.random.default_rng(4)
    D, R = 8, 8
    cos, sin = _tables(16, R)
    x = rng.standard_normal((1, 3, 2, D))
    pos = np.array([[1, 7, 11]])
    perm = np.concatenate([np.arange(0, R, 2), np.arange(1, R, 2)])  # interleaved pair j -> (j, j + R/2)
    inter = oracle.rotary(x, cos, sin, pos, True)
    halves = oracle.rotary(x[..., perm], cos, sin, pos, False)
    assert np.allclose(inter[..., perm], halves, atol=1e-14)


def test_cache_rows_paged_and_batch_indexed():
    # page size 4: sequence 0 holds 3 tokens on logical page 0 -> physical 5, page 1 -> 2
    row, slot = oracle.cache_rows(2, 3, [3, 0], block_table=[[5, 2], [7, 1]], page_size=4)
    assert row.tolist() == [[5, 2, 2], [7, 7, 7]]
    assert slot.tolist() == [[3, 0, 1], [0, 1, 2]]
    row, slot = oracle.cache_rows(2, 2, [4, 1], cache_batch_idx=[3, 0])
    assert row.tolist() == [[3, 3], [0, 0]] and slot.tolist() == [[4, 5], [1, 2]]


def test_kvcache_append_writes_only_the_new_rows():
    rng = np.random.default_rng(5)
    P, page, H, D = 6, 4, 2, 8
    kc, vc = rng.standard_normal((P, page, H, D)), rng.standard_normal((P, page, H, D))
    kn, vn = rng.standard_normal((2, 3, H, D)), rng.standard_normal((2, 3, H, D))
    bt = np.array([[5, 2], [0, 3]])
    cos, sin = _tables(16, 4)
    k2, v2 = oracle.kvcache_append(kc, vc, kn, vn, [3, 5], block_table=bt, page_size=page, rotary_cos=cos,
                                   rotary_sin=sin, interleaved=False)
    touched = np.zeros((P, page), dtype=bool)
    row, slot = oracle.cache_rows(2, 3, [3, 5], block_table=bt, page_size=page)
    touched[row, slot] = True
    assert np.array_equal(k2[~touched], kc[~touched]) and np.array_equal(v2[~touched], vc[~touched])
    kr = oracle.rotary(kn, cos, sin, np.array([[3, 4, 5], [5, 6, 7]]), False)
    for b in range(2):
        for i in range(3):
            assert np.array_equal(k2[row[b, i], slot[b, i]], kr[b, i])
            assert np.array_equal(v2[row[b, i], slot[b, i]], vn[b, i])
    # a quarter turn at angle j = 0 for position 1 (cos 0, sin 1) swaps and negates
    q = np.zeros((1, 1, 1, 4))
    q[..., 0] = 1.0
    out = oracle.rotary(q, np.array([[1.0, 1.0], [0.0, 1.0]]), np.array([[0.0, 0.0], [1.0, 0.0]]),
                        np.array([[1]]), False).ravel()
    assert np.allclose(out, [0.0, 0.0, 1.0, 0.0], atol=1e-15) and math.isclose(np.linalg.norm(out), 1.0)
