"""Checks of the seeded input generators (CPU only)."""
import numpy as np
import torch

from learned_kv_cache_decode_b200 import workloads as W


def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.standard_normal(100000).astype(np.float32),
                        np.array([1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -2.5, 0.0, 1e-30], np.float32)])
    ours = W.bf16_bits(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(ours, ref)
    back = W.bf16_to_f64(ours)
    np.testing.assert_array_equal(back, torch.from_numpy(ref.view(np.int16)).view(torch.bfloat16).double().numpy())


def test_kv_random_access_is_consistent():
    wl = W.WORKLOADS["llama3.2-1b"]
    K, V = W.kv(wl, 3, 0, 2500)
    K2, V2 = W.kv(wl, 3, 1000, 1300)
    np.testing.assert_array_equal(K[1000:2300], K2)
    np.testing.assert_array_equal(V[1000:2300], V2)
    assert K.dtype == np.uint16 and K.shape == (2500, 8, 64)
    assert not np.array_equal(K, V)
    K3, _ = W.kv(wl, 4, 0, 10)
    assert not np.array_equal(K[:10], K3)


def test_alpha_random_access_and_rates():
    wl = W.WORKLOADS["qwen-r1-7b-32k"]
    a = W.alpha(wl, 0, 0, 20000)
    np.testing.assert_array_equal(a[5000:9000], W.alpha(wl, 0, 5000, 4000))
    p = W.alpha_prob(wl, 0, np.array([0, 5000, 10000, 20000]))
    np.testing.assert_allclose(p[:, 0], [0.5, 0.5 + 0.4375 * 0.5, 0.9375, 0.9375])
    late = a[12000:].mean()
    assert abs(late - 0.9375) < 0.01
    assert abs(a[:1000].mean() - 0.5) < 0.05


def test_per_stream_rates_and_contexts():
    wl = W.WORKLOADS["qwen-r1-32b-chains"]
    ctx = W.contexts(wl)
    assert ctx.shape == (64,) and ctx.min() >= 8192 and ctx.max() <= 32768
    np.testing.assert_array_equal(ctx, W.contexts(wl))
    r = W.stream_rates(wl, 5)
    assert r.shape == (8,) and np.all((r >= 0.8) & (r <= 0.95))
    a = W.alpha(wl, 5, 0, 30000)
    np.testing.assert_allclose(a.mean(axis=0), r, atol=0.01)


def test_query_shapes():
    for wl in W.WORKLOADS.values():
        q = W.query(wl, 0)
        assert q.shape == (wl.batch, wl.num_q_heads, wl.head_dim)
        assert q.dtype == (np.uint16 if wl.dtype == "bf16" else np.float32)
        assert wl.num_q_heads % wl.num_kv_heads == 0


def test_depth_layers_compress_more_with_depth():
    """The per-layer schedule of depth-wise compression: alpha rates give long-context
    ratios linear from the first to the last layer, each layer its own draws."""
    base = W.WORKLOADS["qwen-r1-7b-32k"]
    layers = W.depth_layers(base, 4, 2.0, 8.0)
    assert [round(1.0 / (1.0 - x.alpha_args[0]), 9) for x in layers] == [2.0, 4.0, 6.0, 8.0]
    assert len({x.seed for x in layers} | {base.seed}) == 5
    rates = [float(W.alpha(x, 0, 0, 20000).mean()) for x in layers]
    for x, r in zip(layers, rates):
        assert abs(r - x.alpha_args[0]) < 0.01
    assert rates == sorted(rates)
    one = W.depth_layers(base, 1, 3.0, 9.0)
    assert abs(1.0 / (1.0 - one[0].alpha_args[0]) - 3.0) < 1e-12
