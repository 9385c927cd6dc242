"""CUDA path vs the fp64 oracle, through the C ABI (needs a B200).

Small cases span several tiles and ragged tails and are compared element by
element; the five workloads run at full size in the launch configuration the
benchmark times, with routing checked on every token and y on a sample that
reaches every (expert, M-block) tile row of the grouped GEMMs."""
import zlib

import numpy as np
import pytest

import moe_inputs as mi
import oracle
from gpu_helpers import (NEAR_TIE, PER_TOKEN_FACTOR, TOL_Y, agreeing_tokens, block_covering_sample,
                         blocks_covered, compare_routing, dev, host, near_tie_mask, rel_l2, require_cuda,
                         y_as_f64, y_check_with_alternatives)

pytestmark = pytest.mark.gpu

SMALL = [
    # name, T, d, ffn, n, K, dtype
    ("bf16_ragged", 300, 256, 384, 8, 2, "bf16"),
    ("bf16_k3_n16", 1000, 512, 640, 16, 3, "bf16"),
    ("bf16_tails", 77, 320, 192, 4, 1, "bf16"),
    ("bf16_n1", 130, 128, 256, 1, 1, "bf16"),
    ("bf16_dense_K_eq_n", 50, 192, 128, 4, 4, "bf16"),
    ("bf16_T1", 1, 256, 256, 8, 2, "bf16"),
    ("bf16_many_experts", 500, 128, 128, 64, 2, "bf16"),
    ("bf16_n256", 700, 64, 64, 256, 8, "bf16"),
    # tensor-core router: top-K fused over a cluster of 2 and 4 d-splits, and
    # K > 8 (logits to memory, then the top-K kernel)
    ("bf16_router_split2", 600, 1024, 128, 40, 3, "bf16"),
    ("bf16_router_split4", 1000, 2048, 128, 8, 2, "bf16"),
    ("bf16_router_K10", 600, 1024, 64, 32, 10, "bf16"),
    # tensor-core router accumulators: one MMA of N = 3 Npad (Npad = 80), two
    # (N = 2 Npad + Npad; Npad = 112 with padding rows, 128), three into one
    # accumulator (Npad = 144)
    ("bf16_router_n80", 600, 256, 64, 80, 2, "bf16"),
    ("bf16_router_n100", 520, 512, 64, 100, 4, "bf16"),
    ("bf16_router_n128", 600, 256, 128, 128, 2, "bf16"),
    ("bf16_router_n130", 530, 256, 64, 130, 2, "bf16"),
    ("f32_tiny", 64, 128, 256, 8, 2, "f32"),
    ("f32_n40_k4", 200, 64, 128, 40, 4, "f32"),
    ("f32_n1", 33, 64, 64, 1, 1, "f32"),
]


def run_layer(cfg, L):
    import sparse_mixture_experts_24_b200 as m
    torch = require_cuda()
    layer = m.MoELayer(cfg.n, cfg.K, cfg.d, cfg.ffn, cfg.dtype)
    try:
        xs = [dev(L[k]) for k in ("x", "W_g", "w1", "w3", "w2")]
        y, idx, w = layer.forward(*xs)
        layer.sync_status()
        torch.cuda.synchronize()
        return host(y), host(idx), host(w)
    finally:
        layer.close()


@pytest.mark.parametrize("case", SMALL, ids=[c[0] for c in SMALL])
def test_small_layer_matches_oracle(case):
    name, T, d, F, n, K, dt = case
    cfg = mi.custom_config(name, T=T, d=d, ffn=F, n=n, K=K, dtype=dt)
    L = mi.make_layer(cfg, seed=zlib.crc32(name.encode()) % 1000)
    y, idx, w = run_layer(cfg, L)
    o_idx, o_gate, o_logits = oracle.router(L["x"], L["W_g"], K)
    rep = compare_routing(idx, w, o_idx, o_gate, o_logits, L["x"], L["W_g"], K)
    # y against the oracle's own layer on the tokens whose routing agrees
    y_ref, _, _ = oracle.moe_forward(L["x"], L["W_g"], L["w1"], L["w3"], L["w2"], K)
    agree = agreeing_tokens(idx, o_idx)
    yg = y_as_f64(y)[agree]
    y_ref = y_ref[agree]
    err = rel_l2(yg, y_ref)
    assert err <= TOL_Y[dt], (name, err, rep)
    # per-token relative error stays bounded too (no single bad row hides in the norm)
    per_tok = np.linalg.norm(yg - y_ref, axis=1) / np.maximum(np.linalg.norm(y_ref, axis=1), 1e-30)
    assert per_tok.max() <= 5 * TOL_Y[dt], per_tok.max()


@pytest.mark.parametrize("path", ["single", "pair"])
@pytest.mark.parametrize("case", [("pair_big_segments", 2048, 256, 512, 4, 2),
                                  ("pair_ragged", 700, 192, 320, 2, 1),
                                  ("pair_odd_blocks", 1333, 128, 384, 3, 2)], ids=lambda c: c[0])
def test_gemm_paths_match_oracle(case, path, monkeypatch):
    """Both GEMM tilings (single SM, CTA pair) against the oracle on cases with
    large, ragged and odd-numbered 256-row segments."""
    monkeypatch.setenv("MOE_GEMM_PATH", path)
    name, T, d, F, n, K = case
    cfg = mi.custom_config(name, T=T, d=d, ffn=F, n=n, K=K, dtype="bf16")
    L = mi.make_layer(cfg, seed=zlib.crc32(name.encode()) % 1000)
    y, idx, w = run_layer(cfg, L)
    o_idx, o_gate, o_logits = oracle.router(L["x"], L["W_g"], K)
    compare_routing(idx, w, o_idx, o_gate, o_logits, L["x"], L["W_g"], K)
    y_ref, _, _ = oracle.moe_forward(L["x"], L["W_g"], L["w1"], L["w3"], L["w2"], K)
    agree = agreeing_tokens(idx, o_idx)
    yg, y_ref = y_as_f64(y)[agree], y_ref[agree]
    err = rel_l2(yg, y_ref)
    assert err <= TOL_Y["bf16"], (name, path, err)
    per_tok = np.linalg.norm(yg - y_ref, axis=1) / np.maximum(np.linalg.norm(y_ref, axis=1), 1e-30)
    assert per_tok.max() <= 5 * TOL_Y["bf16"], per_tok.max()


def test_route_entry_point_matches_forward_routing():
    import sparse_mixture_experts_24_b200 as m
    cfg = mi.custom_config("route", T=257, d=256, ffn=128, n=8, K=2, dtype="bf16")
    L = mi.make_layer(cfg, seed=3)
    layer = m.MoELayer(cfg.n, cfg.K, cfg.d, cfg.ffn, "bf16")
    try:
        x, Wg = dev(L["x"]), dev(L["W_g"])
        idx, w = layer.route(x, Wg)
        y, idx2, w2 = layer.forward(x, Wg, dev(L["w1"]), dev(L["w3"]), dev(L["w2"]))
        layer.sync_status()
        assert np.array_equal(host(idx), host(idx2)) and np.array_equal(host(w), host(w2))
    finally:
        layer.close()


# up to 4,096 pairs: the one-block kernel; above: rank, scan, scatter
@pytest.mark.parametrize("T,n,K", [(1, 1, 1), (5, 8, 2), (300, 8, 2), (1000, 16, 3), (777, 256, 8),
                                   (64, 4, 4), (4096, 128, 2), (9000, 8, 2), (40000, 64, 2)])
def test_dispatch_matches_oracle_bit_exact(T, n, K):
    import sparse_mixture_experts_24_b200 as m
    torch = require_cuda()
    rng = np.random.default_rng(T * 31 + n)
    idx = np.stack([rng.permutation(n)[:K] for _ in range(T)]).astype(np.int32)
    layer = m.MoELayer(n, K, 64, 64, "bf16")
    try:
        counts, offsets, row_token, token_row = layer.dispatch(dev(idx))
        layer.sync_status()
        c, o, rt, tr = oracle.dispatch(idx, n)
        assert np.array_equal(host(counts), c)
        assert np.array_equal(host(offsets), o)
        assert np.array_equal(host(row_token), rt)
        assert np.array_equal(host(token_row), tr)
    finally:
        layer.close()
    torch.cuda.synchronize()


def test_forward_with_routing_dense_and_handmade():
    """Caller-supplied routing: every expert for every token (K = n), and a
    hand-made routing with uneven segments, against the oracle."""
    import sparse_mixture_experts_24_b200 as m
    torch = require_cuda()
    cfg = mi.custom_config("fwr", T=190, d=256, ffn=256, n=6, K=6, dtype="bf16")
    L = mi.make_layer(cfg, seed=11)
    g = np.random.default_rng(0).random((cfg.T, cfg.K)).astype(np.float32)
    g /= g.sum(1, keepdims=True)
    idx = np.stack([np.random.default_rng(t).permutation(6) for t in range(cfg.T)]).astype(np.int32)
    layer = m.MoELayer(cfg.n, cfg.K, cfg.d, cfg.ffn, "bf16")
    try:
        y = layer.forward_with_routing(dev(L["x"]), dev(idx), dev(g), dev(L["w1"]), dev(L["w3"]),
                                       dev(L["w2"]))
        layer.sync_status()
        ref = oracle.forward_with_routing(L["x"], idx, g.astype(np.float64), L["w1"], L["w3"], L["w2"])
        assert rel_l2(y_as_f64(host(y)), ref) <= TOL_Y["bf16"]
    finally:
        layer.close()
    # skewed hand-made routing: expert 0 for every token, the others rarely
    cfg2 = mi.custom_config("fwr2", T=600, d=128, ffn=384, n=5, K=2, dtype="bf16")
    L2 = mi.make_layer(cfg2, seed=12)
    idx2 = np.zeros((cfg2.T, 2), np.int32)
    idx2[:, 1] = 1 + (np.arange(cfg2.T) % 97 == 0) * 3
    g2 = np.tile(np.array([[0.7, 0.3]], np.float32), (cfg2.T, 1))
    layer = m.MoELayer(cfg2.n, cfg2.K, cfg2.d, cfg2.ffn, "bf16")
    try:
        y2 = layer.forward_with_routing(dev(L2["x"]), dev(idx2), dev(g2), dev(L2["w1"]), dev(L2["w3"]),
                                        dev(L2["w2"]))
        layer.sync_status()
        ref2 = oracle.forward_with_routing(L2["x"], idx2, g2.astype(np.float64), L2["w1"], L2["w3"],
                                           L2["w2"])
        assert rel_l2(y_as_f64(host(y2)), ref2) <= TOL_Y["bf16"]
    finally:
        layer.close()
    torch.cuda.synchronize()


# ----- full-size workloads in the benchmark's launch configuration ---------

_LAYERS = {}


def _layer_inputs(name):
    if name not in _LAYERS:
        _LAYERS.clear()
        _LAYERS[name] = mi.make_layer(mi.CONFIGS[name], seed=0)
    return _LAYERS[name]


@pytest.mark.parametrize("name", ["tiny_fp32", "decode", "prefill", "skew_prefill", "many_expert"])
def test_full_size_workload(name):
    """Routing on every token; y on every token (T <= 64) or on at least 512
    tokens that put a row in every (expert, 128-row M-block) of both grouped
    GEMMs, the last, ragged row of every segment included, plus every
    near-tie token, each against the oracle's layer (near-ties: the closest
    of the oracle's own alternative routings)."""
    cfg = mi.CONFIGS[name]
    L = _layer_inputs(name)
    y, idx, w = run_layer(cfg, L)
    o_idx, o_gate, o_logits = oracle.router(L["x"], L["W_g"], cfg.K)
    rep = compare_routing(idx, w, o_idx, o_gate, o_logits, L["x"], L["W_g"], cfg.K)
    print("\n%s routing: %s" % (name, rep))
    agreeing_tokens(idx, o_idx)
    near = near_tie_mask(o_logits, cfg.K)
    if cfg.T <= 64:
        sample, nblk = np.arange(cfg.T), None
    else:
        sample, nblk = block_covering_sample(o_idx, cfg.n, count=512)
        sample = np.union1d(sample, np.nonzero(near | (idx != o_idx).any(axis=1))[0])
        covered = blocks_covered(sample, o_idx, cfg.n)
        print("%s sample: %d tokens covering %d of %d (expert, M-block) pairs"
              % (name, sample.size, covered, nblk))
        assert covered == nblk and sample.size >= 512
    err, worst, tied = y_check_with_alternatives(y, idx, o_logits, o_idx, o_gate, sample, L, cfg.K,
                                                 TOL_Y[cfg.dtype])
    print("%s y rel-L2 on %d tokens: %.3e (worst token %.3e; %d near-tie tokens against the "
          "oracle's alternatives)" % (name, sample.size, err, worst, tied))
    assert err <= TOL_Y[cfg.dtype]
    assert worst <= PER_TOKEN_FACTOR * TOL_Y[cfg.dtype]
    # properties that hold at any size: finite output, gates sum to 1,
    # every token routed to K distinct experts
    yf = y_as_f64(y)
    assert np.isfinite(yf).all()
    assert (np.sort(idx, 1)[:, 1:] != np.sort(idx, 1)[:, :-1]).all() if cfg.K > 1 else True
    # every token whose routing differs from the oracle's is a near-tie whose
    # GPU routing is one of the oracle's alternatives
    for t in np.nonzero((idx != o_idx).any(axis=1))[0]:
        alts = oracle.routing_alternatives(o_logits[t], cfg.K, NEAR_TIE)
        assert tuple(idx[t]) in {tuple(int(e) for e in i) for i, _ in alts}, t
    if cfg.skew:
        share = np.bincount(idx.ravel(), minlength=cfg.n) / idx.size
        assert share[0] >= 0.40 and share.min() < 0.02, share
