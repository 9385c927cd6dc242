"""Seeded random layer shapes vs the fp64 oracle, through the C ABI (needs a
B200): T, d, ffn, n and K drawn over the ranges the library accepts (d and ffn
multiples of 64; 256 for the 4-bit weight-and-activation path), so that tile
edges, ragged segments, empty experts and the router variants are met in
combinations no hand-written case names.  Routing bit-exact outside near-ties;
y within the bf16 bar of the oracle's layer on the tokens routed alike."""
import numpy as np
import pytest

import moe_inputs as mi
import oracle
from gpu_helpers import TOL_Y, agreeing_tokens, compare_routing, dev, host, rel_l2, require_cuda, y_as_f64

pytestmark = pytest.mark.gpu


def draw(seed, step=64):
    rng = np.random.default_rng(1000 + seed)
    n = int(rng.choice([1, 2, 3, 5, 8, 13, 16, 33, 64, 100]))
    K = int(rng.integers(1, min(n, 8) + 1))
    T = int(rng.choice([1, 2, 31, 64, 127, 300, 513, 700]))
    d = int(step * rng.integers(1, 1024 // step + 1))
    F = int(step * rng.integers(1, 1024 // step + 1))
    return T, d, F, n, K


@pytest.mark.parametrize("seed", range(12))
def test_bf16_layer_random_shapes(seed):
    import sparse_mixture_experts_24_b200 as m
    torch = require_cuda()
    T, d, F, n, K = draw(seed)
    cfg = mi.custom_config("fuzz%d" % seed, T=T, d=d, ffn=F, n=n, K=K, dtype="bf16")
    L = mi.make_layer(cfg, seed=seed)
    layer = m.MoELayer(n, K, d, F, "bf16")
    try:
        y, idx, w = layer.forward(*(dev(L[k]) for k in ("x", "W_g", "w1", "w3", "w2")))
        layer.sync_status()
        torch.cuda.synchronize()
        y, idx, w = host(y), host(idx), host(w)
    finally:
        layer.close()
    o_idx, o_gate, o_logits = oracle.router(L["x"], L["W_g"], K)
    compare_routing(idx, w, o_idx, o_gate, o_logits, L["x"], L["W_g"], K)
    agree = agreeing_tokens(idx, o_idx)
    y_ref = oracle.forward_with_routing(L["x"], o_idx, o_gate, L["w1"], L["w3"], L["w2"])
    assert rel_l2(y_as_f64(y)[agree], y_ref[agree]) <= TOL_Y["bf16"], (T, d, F, n, K)


@pytest.mark.parametrize("seed", range(6))
def test_w4a4_layer_random_shapes(seed):
    import sparse_mixture_experts_24_b200 as m
    torch = require_cuda()
    T, d, F, n, K = draw(100 + seed, step=256)
    cfg = mi.custom_config("fuzz_w4_%d" % seed, T=T, d=d, ffn=F, n=n, K=K, dtype="bf16")
    L = mi.make_layer(cfg, seed=seed)
    q = [oracle.quantize_weights_fp4(L[k]) for k in ("w1", "w3", "w2")]
    w13 = m.pack_weights_w4a4(*(dev(a) for a in q[0]), pair=tuple(dev(a) for a in q[1]))
    w2 = m.pack_weights_w4a4(*(dev(a) for a in q[2]))
    layer = m.MoELayer(n, K, d, F, "bf16")
    try:
        y, idx, w = layer.forward_w4a4(dev(L["x"]), dev(L["W_g"]), w13, w2)
        layer.sync_status()
        torch.cuda.synchronize()
        y, idx = host(y), host(idx)
    finally:
        layer.close()
    o_idx, o_gate, _ = oracle.router(L["x"], L["W_g"], K)
    agree = agreeing_tokens(idx, o_idx)
    y_ref = oracle.forward_w4a4(L["x"], o_idx, o_gate, *q)
    assert rel_l2(y_as_f64(y)[agree], y_ref[agree]) <= TOL_Y["bf16"], (T, d, F, n, K)
