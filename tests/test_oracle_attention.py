"""Pins for the oracle's fp64 attention (CPU only).

Closed forms worked by hand, special cases the pages' steps reduce to
(uniform keys, one dominant key, the quantised cache on its own grid, the
full residual window, idx = all positions, verification row = prefix
decode), and an independent library implementation of the textbook
operation (torch scaled_dot_product_attention in float64)."""

import math

import numpy as np
import pytest
import torch

from oracle import attention as A
from oracle import quant


def test_two_key_closed_form():
    o, lse = A.softmax_attention(np.array([[1.0, 0.0]]), np.eye(2), np.eye(2), 1.0)
    e = math.e
    assert np.allclose(o[0], [e / (1 + e), 1 / (1 + e)], rtol=0, atol=1e-15)
    assert abs(lse[0] - math.log(1 + e)) < 1e-15


def test_three_key_closed_form():
    # scores 0.5 * [2, 2, 4] = [1, 1, 2]; weights [1, 1, e] / (2 + e);
    # the weighted values [2,0], [0,2], [1,1] average to exactly [1, 1].
    q = np.array([[2.0, 2.0]])
    k = np.array([[1.0, 0.0], [0.0, 1.0], [1.0, 1.0]])
    v = np.array([[2.0, 0.0], [0.0, 2.0], [1.0, 1.0]])
    o, lse = A.softmax_attention(q, k, v, 0.5)
    assert np.allclose(o[0], [1.0, 1.0], rtol=0, atol=1e-15)
    assert abs(lse[0] - (1.0 + math.log(2.0 + math.e))) < 1e-14


def test_equal_keys_give_mean_of_values():
    rng = np.random.default_rng(1)
    k = np.tile(rng.standard_normal(16), (50, 1))
    v = rng.standard_normal((50, 16))
    o, _ = A.softmax_attention(rng.standard_normal((3, 16)), k, v, 0.25)
    assert np.allclose(o, v.mean(0)[None], rtol=0, atol=1e-14)


def test_dominant_key_gives_its_value_row():
    rng = np.random.default_rng(2)
    D = 8
    k = rng.standard_normal((40, D)) * 0.01
    q = np.zeros((1, D))
    q[0, 0] = 1.0
    k[17, 0] = 1e4            # score gap >> 100 / sm_scale
    v = rng.standard_normal((40, D))
    o, _ = A.softmax_attention(q, k, v, 1.0)
    assert np.allclose(o[0], v[17], rtol=2.0 ** -24, atol=0)


def _sdpa(q, k, v, scale, mask=None):
    t = lambda x: torch.from_numpy(np.ascontiguousarray(x, np.float64))
    return torch.nn.functional.scaled_dot_product_attention(
        t(q), t(k), t(v), attn_mask=None if mask is None else torch.from_numpy(mask), scale=scale).numpy()


def test_dense_decode_matches_torch_sdpa():
    rng = np.random.default_rng(4)
    B, Hq, Hkv, N, D = 2, 8, 2, 37, 16
    q = rng.standard_normal((B, Hq, D))
    k = rng.standard_normal((B, Hkv, N, D))
    v = rng.standard_normal((B, Hkv, N, D))
    o = A.draft_attention_dense(q, k, v, 0.3)
    g = Hq // Hkv
    kk = np.repeat(k, g, axis=1)
    vv = np.repeat(v, g, axis=1)
    ref = _sdpa(q[:, :, None, :], kk, vv, 0.3)[:, :, 0, :]
    assert np.allclose(o, ref, rtol=1e-12, atol=1e-13)


def test_verify_matches_torch_sdpa_with_causal_mask():
    rng = np.random.default_rng(5)
    B, nq, Hq, Hkv, T, D = 2, 5, 6, 3, 23, 8
    q = rng.standard_normal((B, nq, Hq, D))
    k = rng.standard_normal((B, Hkv, T, D))
    v = rng.standard_normal((B, Hkv, T, D))
    o, lse = A.verify_attention(q, k, v, None)
    g = Hq // Hkv
    mask = np.arange(T)[None, :] <= (T - nq + np.arange(nq))[:, None]
    ref = _sdpa(q.transpose(0, 2, 1, 3), np.repeat(k, g, 1), np.repeat(v, g, 1), 1 / math.sqrt(D), mask)
    assert np.allclose(o, ref.transpose(0, 2, 1, 3), rtol=1e-12, atol=1e-13)
    # lse closed form on one row
    s = q[1, 2, 4] @ k[1, 2, :T - nq + 3].T / math.sqrt(D)
    assert abs(lse[1, 2, 4] - np.log(np.exp(s).sum())) < 1e-12


def test_verify_causal_hand_example():
    # nq = 2, T = 3, scores [0, 0, ln 2]: row 0 sees keys 0..1 -> mean(0, 4) = 2,
    # row 1 sees all -> (0 + 4 + 2*8) / 4 = 5.
    q = np.ones((1, 2, 1, 1))
    k = np.array([0.0, 0.0, math.log(2.0)]).reshape(1, 1, 3, 1)
    v = np.array([0.0, 4.0, 8.0]).reshape(1, 1, 3, 1)
    o, _ = A.verify_attention(q, k, v, 1.0)
    assert abs(o[0, 0, 0, 0] - 2.0) < 1e-14 and abs(o[0, 1, 0, 0] - 5.0) < 1e-14


def test_verify_rows_equal_prefix_decode():
    rng = np.random.default_rng(6)
    B, nq, Hq, Hkv, T, D = 1, 4, 4, 2, 30, 16
    q = rng.standard_normal((B, nq, Hq, D))
    k = rng.standard_normal((B, Hkv, T, D))
    v = rng.standard_normal((B, Hkv, T, D))
    o, _ = A.verify_attention(q, k, v, None)
    for i in range(nq):
        n = T - nq + i + 1
        d = A.draft_attention_dense(q[:, i], k[:, :, :n], v[:, :, :n], None)
        assert np.allclose(o[:, i], d, rtol=1e-13, atol=1e-15)   # BLAS may sum in another order


def test_quant_on_grid_equals_dense():
    """Keys and values on the quantisation grid: the quantised draft equals
    dense attention over the same data, bit for bit."""
    rng = np.random.default_rng(8)
    B, Hq, Hkv, T, D, G, R = 1, 4, 2, 96, 64, 32, 32
    Lq = T - R
    codes = rng.integers(0, 4, size=(B, Hkv, Lq, D))
    codes[..., 0::G, :] = 0
    codes[..., 1::G, :] = 3
    codes[..., :, 0::G] = 0
    codes[..., :, 1::G] = 3
    x = -1.0 + codes * 0.5
    k = np.concatenate([x, rng.standard_normal((B, Hkv, R, D)).astype(np.float32)], 2)
    v = np.concatenate([x * 2, rng.standard_normal((B, Hkv, R, D)).astype(np.float32)], 2)
    cache = quant.build_quant_cache(k, v, 2, G, R)
    q = rng.standard_normal((B, Hq, D))
    assert np.array_equal(A.draft_attention_quant(q, cache), A.draft_attention_dense(q, k, v))


def test_quant_all_residual_equals_dense():
    rng = np.random.default_rng(9)
    k = rng.standard_normal((2, 2, 40, 64)).astype(np.float32)
    v = rng.standard_normal((2, 2, 40, 64)).astype(np.float32)
    cache = quant.build_quant_cache(k, v, 2, 32, 40)
    q = rng.standard_normal((2, 6, 64))
    assert np.array_equal(A.draft_attention_quant(q, cache), A.draft_attention_dense(q, k, v))


def test_sparse_all_positions_equals_dense_and_gather_is_exact():
    rng = np.random.default_rng(10)
    B, Hq, Hkv, T, D = 2, 4, 2, 50, 16
    k = rng.standard_normal((B, Hkv, T, D))
    v = rng.standard_normal((B, Hkv, T, D))
    q = rng.standard_normal((B, Hq, D))
    idx = np.broadcast_to(np.arange(T), (B, Hkv, T))
    assert np.array_equal(A.draft_attention_sparse(q, k, v, idx), A.draft_attention_dense(q, k, v))
    idx2 = np.sort(rng.choice(T, size=(B, Hkv, 9)), axis=-1)
    rows = A.gather_rows(k, idx2)
    assert rows[1, 1, 3].tolist() == k[1, 1, idx2[1, 1, 3]].tolist()
    with pytest.raises(ValueError):
        A.gather_rows(k, np.full((B, Hkv, 2), T))


def test_empty_key_set_refused():
    with pytest.raises(ValueError):
        A.softmax_attention(np.ones((1, 4)), np.zeros((0, 4)), np.zeros((0, 4)), 1.0)
