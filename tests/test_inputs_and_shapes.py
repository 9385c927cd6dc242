"""Seeded input generator and the shape arithmetic the pages print (CPU only)."""
import numpy as np

import moe_inputs as mi
import oracle
from oracle_checks import read_golden


def test_generator_is_deterministic_and_chunk_independent(monkeypatch):
    cfg = mi.custom_config(T=33, d=128, ffn=192, n=4, K=2, dtype="bf16")
    a = mi.make_layer(cfg, seed=5)
    monkeypatch.setattr(mi, "_threads", lambda: 1)
    b = mi.make_layer(cfg, seed=5)
    for k in a:
        assert np.array_equal(a[k], b[k]), k
    c = mi.make_layer(cfg, seed=6)
    assert not np.array_equal(a["w1"], c["w1"])
    assert a["x"].dtype == np.uint16 and a["W_g"].dtype == np.float32
    assert a["w1"].shape == (4, 128, 192) and a["w2"].shape == (4, 192, 128)


def test_multi_chunk_tensor(monkeypatch):
    monkeypatch.setattr(mi, "CHUNK", 1000)
    cfg = mi.custom_config(T=40, d=64, ffn=64, n=3, K=2, dtype="f32")
    a = mi.make_layer(cfg, seed=1)
    monkeypatch.setattr(mi, "_threads", lambda: 1)
    b = mi.make_layer(cfg, seed=1)
    assert np.array_equal(a["w1"], b["w1"])
    # std close to 1/sqrt(d) for w1, 1/sqrt(ffn) for w2
    assert abs(a["w1"].std() * 8 - 1) < 0.05 and abs(a["w2"].std() * 8 - 1) < 0.05


def test_bf16_rounding_is_nearest_even():
    vals = np.array([1.0, 1.00390625, 1.01171875, 1.0039062500001, -2.5, 3.0e38, 1e-40],
                    np.float32)
    got = mi.bf16_bits_to_f32(mi.f32_to_bf16_bits(vals))
    # 1 + 2^-8 is halfway between 1 and 1 + 2^-7: ties to even -> 1.0
    assert got[0] == 1.0 and got[1] == 1.0
    # 1 + 3*2^-8 is halfway between 1+2^-7 and 1+2^-6: ties to even -> 1+2^-6
    assert got[2] == np.float32(1.015625)
    assert got[4] == -2.5
    assert np.all(np.isfinite(got[:6]))
    x = np.random.default_rng(0).standard_normal(10000).astype(np.float32)
    r = mi.bf16_bits_to_f32(mi.f32_to_bf16_bits(x))
    assert np.all(np.abs(r - x) <= np.abs(x) * 2.0 ** -8)


def test_parameter_counts_match_the_pages():
    """Part 4 of the neobadger page: 3 x 4,096 x 14,336 parameters per expert
    (about 176 million), about 45.1 billion over 8 experts x 32 layers, and
    routers of 4,096 x 8 per layer, about 1 million in total."""
    g = read_golden("parameter_counts.txt")
    d, F = int(g["d"][0]), int(g["ffn"][0])
    layers, n = int(g["layers"][0]), int(g["experts"][0])
    cfg = mi.CONFIGS["decode"]
    assert (cfg.d, cfg.ffn, cfg.n, cfg.K) == (d, F, n, int(g["experts_per_token"][0]))
    per_expert = 3 * d * F
    assert per_expert == 176_160_768
    assert round(per_expert / 1e6) == round(g["per_expert_params_approx"][0] / 1e6)
    assert round(per_expert * n * layers / 1e8) == round(g["all_expert_params_approx"][0] / 1e8)
    assert round(d * n * layers / 1e6) == round(g["router_params_total_approx"][0] / 1e6)
    assert cfg.expert_bytes() == 2 * per_expert
    assert mi.CONFIGS["prefill"].active_flops() == 6.0 * 4096 * 2 * d * F + 2.0 * 4096 * d * 8


def test_skewed_generator_histogram():
    """The skewed config gives expert 0 at least 40% of routed rows and one
    expert under 2% (checked with the oracle's routing on 2048 tokens)."""
    cfg = mi.CONFIGS["skew_prefill"]
    sub = mi.custom_config(T=2048, d=cfg.d, ffn=64, n=cfg.n, K=cfg.K, dtype="bf16", skew=True)
    L = mi.make_layer(sub, seed=0, only=("x", "W_g"))
    assert np.all(mi.bf16_bits_to_f32(L["x"][:, -1]) == 1.0)
    idx, gate, _ = oracle.router(L["x"], L["W_g"], cfg.K)
    share = np.bincount(idx.ravel(), minlength=cfg.n) / idx.size
    assert share[0] >= 0.40, share
    assert share.min() < 0.02, share


def test_uniform_routing_many_expert_shape():
    """Without skew the routing is close to uniform (many-expert shape, fewer tokens)."""
    sub = mi.custom_config(T=4096, d=2048, ffn=64, n=128, K=2, dtype="bf16")
    L = mi.make_layer(sub, seed=0, only=("x", "W_g"))
    idx, _, _ = oracle.router(L["x"], L["W_g"], 2)
    c = np.bincount(idx.ravel(), minlength=128)
    assert c.min() > 20 and c.max() < 120 and c.sum() == 8192
