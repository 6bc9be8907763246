"""Pins for the oracle's masked attention (CPU only).

The attention oracle is checked against torch's scaled_dot_product_attention
run in float64 on the CPU (a library routine), in the special cases where
DMS reduces to a textbook attention:
  * every alpha = 0          -> dense causal attention;
  * every alpha = 1          -> sliding-window attention of width w;
  * w >= context, any alpha  -> dense attention;
and with an explicit boolean mask for mixed alpha. Closed forms (one
visible token, two visible tokens) and the GQA head mapping are pinned too.
"""
import math

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle


def _sdpa_last(q, K, V, mask_last_row, scale):
    """fp64 SDPA of g query rows at the last position. mask: [T] bool (True = attend)."""
    qt = torch.from_numpy(q)[None, :, None, :]                      # [1, g, 1, d]
    kt = torch.from_numpy(K)[None, None].expand(1, q.shape[0], -1, -1)
    vt = torch.from_numpy(V)[None, None].expand(1, q.shape[0], -1, -1)
    m = torch.from_numpy(np.asarray(mask_last_row, dtype=bool))[None, None, None, :]
    return F.scaled_dot_product_attention(qt, kt, vt, attn_mask=m, scale=scale)[0, :, 0].numpy()


def _rand(rng, T, g, d):
    return (rng.standard_normal((g, d)), rng.standard_normal((T, d)), rng.standard_normal((T, d)))


@pytest.mark.parametrize("T,d,g", [(1, 64, 4), (17, 64, 4), (300, 128, 7), (1000, 64, 1)])
def test_all_kept_is_dense(T, d, g):
    rng = np.random.default_rng(T + d)
    q, K, V = _rand(rng, T, g, d)
    a = np.zeros(T, np.uint8)
    scale = 1.0 / math.sqrt(d)
    got = oracle.attention(q, K, V, a, window=16, scale=scale)
    ref = _sdpa_last(q, K, V, np.ones(T, bool), scale)
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("T,w", [(40, 1), (40, 16), (300, 256), (600, 256), (10, 10)])
def test_all_marked_is_sliding_window(T, w):
    rng = np.random.default_rng(T * 7 + w)
    q, K, V = _rand(rng, T, 5, 64)
    a = np.ones(T, np.uint8)
    scale = 0.125
    got = oracle.attention(q, K, V, a, window=w, scale=scale)
    band = np.arange(T) >= T - w      # the last w positions, the query's own included
    ref = _sdpa_last(q, K, V, band, scale)
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-12)


def test_window_covering_context_is_dense_for_any_alpha():
    rng = np.random.default_rng(1)
    T = 200
    q, K, V = _rand(rng, T, 4, 64)
    a = rng.integers(0, 2, T).astype(np.uint8)
    got = oracle.attention(q, K, V, a, window=T, scale=0.1)
    ref = _sdpa_last(q, K, V, np.ones(T, bool), 0.1)
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("w", [1, 3, 16, 64])
def test_mixed_alpha_matches_masked_sdpa(w):
    rng = np.random.default_rng(w)
    T = 257
    q, K, V = _rand(rng, T, 7, 128)
    a = (rng.random(T) < 0.7).astype(np.uint8)
    mask = np.zeros(T, bool)
    mask[oracle.visible_positions(a, T - 1, w)] = True
    got = oracle.attention(q, K, V, a, window=w, scale=1 / math.sqrt(128))
    ref = _sdpa_last(q, K, V, mask, 1 / math.sqrt(128))
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-12)


def test_single_visible_token_returns_its_value_exactly():
    rng = np.random.default_rng(2)
    T, w = 9, 1
    q, K, V = _rand(rng, T, 3, 64)
    a = np.ones(T, np.uint8)      # everything marked, w = 1: only the query's own token
    got = oracle.attention(q, K, V, a, window=w, scale=0.3)
    np.testing.assert_array_equal(got, np.repeat(V[-1:], 3, axis=0))


def test_two_tokens_closed_form():
    q = np.array([[1.0, 2.0]])
    K = np.array([[0.5, 0.0], [0.0, 1.0]])
    V = np.array([[1.0, -1.0], [3.0, 5.0]])
    a = np.zeros(2, np.uint8)
    scale = 0.7
    s0, s1 = scale * 0.5, scale * 2.0
    p1 = math.exp(s1) / (math.exp(s0) + math.exp(s1))
    expect = (1 - p1) * V[0] + p1 * V[1]
    got = oracle.attention(q, K, V, a, window=4, scale=scale)[0]
    np.testing.assert_allclose(got, expect, rtol=1e-15, atol=1e-15)


def test_empty_stream_gives_zeros():
    out = oracle.attention(np.ones((2, 64)), np.zeros((0, 64)), np.zeros((0, 64)),
                           np.zeros(0, np.uint8), window=4, scale=1.0)
    assert np.all(out == 0)


def test_gqa_mapping_matches_sdpa_enable_gqa():
    rng = np.random.default_rng(9)
    T, hq, hkv, d = 120, 28, 4, 128
    q = rng.standard_normal((hq, d))
    K = rng.standard_normal((T, hkv, d))
    V = rng.standard_normal((T, hkv, d))
    a = np.zeros((T, hkv), np.uint8)
    scale = 1 / math.sqrt(d)
    got = oracle.decode_gqa(q, K, V, a, window=256, scale=scale)
    ref = F.scaled_dot_product_attention(
        torch.from_numpy(q)[None, :, None, :],
        torch.from_numpy(K).permute(1, 0, 2)[None],
        torch.from_numpy(V).permute(1, 0, 2)[None],
        scale=scale, enable_gqa=True)[0, :, 0].numpy()
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-12)


def test_per_kv_head_decisions_are_independent():
    """A decision on KV head 0 must not change what KV head 1 sees."""
    rng = np.random.default_rng(4)
    T, d = 50, 64
    q = rng.standard_normal((4, d))
    K = rng.standard_normal((T, 2, d))
    V = rng.standard_normal((T, 2, d))
    a0 = np.zeros((T, 2), np.uint8)
    a1 = a0.copy()
    a1[:, 0] = 1
    o0 = oracle.decode_gqa(q, K, V, a0, 8, 0.1)
    o1 = oracle.decode_gqa(q, K, V, a1, 8, 0.1)
    np.testing.assert_array_equal(o0[2:], o1[2:])
    assert not np.allclose(o0[:2], o1[:2])


def test_batch_equals_single():
    rng = np.random.default_rng(12)
    items = []
    for T in (1, 33, 200):
        q, K, V = _rand(rng, T, 4, 64)
        items.append((q, K, V, (rng.random(T) < 0.5).astype(np.uint8)))
    outs, threads = oracle.attention_batch(items, window=16, scale=0.125)
    assert threads >= 1
    for (q, K, V, a), o in zip(items, outs):
        np.testing.assert_array_equal(o, oracle.attention(q, K, V, a, 16, 0.125))
