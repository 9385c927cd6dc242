"""Expert capacity and load-balancing statistics (Part 5 of the neobadger page)
on the GPU against the oracle, through the C ABI (needs a B200)."""
import math
import zlib

import numpy as np
import pytest

import moe_inputs as mi
import oracle
from gpu_helpers import TOL_Y, dev, host, rel_l2, require_cuda, y_as_f64

pytestmark = pytest.mark.gpu

CAP_CASES = [
    # name, T, d, ffn, n, K, dtype, skew, factor
    ("cap_skew_bf16", 600, 256, 256, 8, 2, "bf16", True, 1.0),
    ("cap_tight_bf16", 500, 128, 192, 4, 2, "bf16", False, 0.5),
    ("cap_loose_bf16", 300, 128, 128, 8, 2, "bf16", True, 8.0),
    ("cap_skew_f32", 200, 64, 128, 8, 2, "f32", True, 1.0),
    ("cap_many_bf16", 700, 128, 128, 64, 2, "bf16", False, 1.0),
    # 6,000 pairs: the three-kernel dispatch with a capacity
    ("cap_mid_bf16", 3000, 64, 64, 16, 2, "bf16", True, 1.0),
]


@pytest.mark.parametrize("case", CAP_CASES, ids=[c[0] for c in CAP_CASES])
def test_capacity_forward_and_dispatch(case):
    import sparse_mixture_experts_24_b200 as m
    require_cuda()
    name, T, d, F, n, K, dt, skew, factor = case
    cfg = mi.custom_config(name, T=T, d=d, ffn=F, n=n, K=K, dtype=dt, skew=skew)
    L = mi.make_layer(cfg, seed=zlib.crc32(name.encode()) % 1000)
    C = math.ceil(factor * T * K / n)
    layer = m.MoELayer(n, K, d, F, dt)
    try:
        layer.set_capacity_factor(factor)
        y, idx_d, w_d = layer.forward(*[dev(L[k]) for k in ("x", "W_g", "w1", "w3", "w2")])
        counts, offsets, row_token, token_row = (host(t) for t in layer.dispatch(idx_d))
        layer.sync_status()
        y, idx, w = host(y), host(idx_d), host(w_d)
    finally:
        layer.close()
    o_idx, o_gate, _ = oracle.router(L["x"], L["W_g"], K)
    # capacity makes every later pair depend on the routing of all earlier
    # tokens, so these cases are chosen to route exactly as the oracle does
    assert np.array_equal(idx, o_idx), "routing differs from the oracle's"
    c, o, rt, tr = oracle.dispatch_capacity(o_idx, n, C)
    assert np.array_equal(counts, c) and np.array_equal(offsets, o)
    assert np.array_equal(token_row, tr)
    assert np.array_equal(row_token[:o[-1]], rt[:o[-1]])
    dropped = tr < 0
    if factor <= 1.0:
        assert dropped.any(), "the case should overflow an expert"
    gate = np.where(dropped, 0.0, o_gate)
    y_ref = oracle.forward_with_routing(L["x"], o_idx, gate, L["w1"], L["w3"], L["w2"])
    err = rel_l2(y_as_f64(y), y_ref)
    assert err <= TOL_Y[dt], (name, err)
    fully = dropped.all(axis=1)
    if fully.any():  # tokens whose every pair overflowed get y = 0 exactly
        assert np.all(y_as_f64(y)[fully] == 0.0)


STAT_CASES = [
    ("stats_bf16_n8", 1000, 256, 8, 2, "bf16", False),
    ("stats_bf16_skew", 700, 512, 8, 2, "bf16", True),
    ("stats_bf16_n128", 900, 256, 128, 2, "bf16", False),
    ("stats_f32_n8", 300, 128, 8, 2, "f32", False),
    ("stats_f32_n40_k3", 257, 64, 40, 3, "f32", False),
]


@pytest.mark.parametrize("case", STAT_CASES, ids=[c[0] for c in STAT_CASES])
def test_router_stats_match_oracle(case):
    import sparse_mixture_experts_24_b200 as m
    require_cuda()
    name, T, d, n, K, dt, skew = case
    cfg = mi.custom_config(name, T=T, d=d, ffn=64, n=n, K=K, dtype=dt, skew=skew)
    L = mi.make_layer(cfg, seed=zlib.crc32(name.encode()) % 1000, only=("x", "W_g"))
    layer = m.MoELayer(n, K, d, 64, dt)
    try:
        # the statistics take the routing as an input: both sides get the oracle's
        o_idx, _, _ = oracle.router(L["x"], L["W_g"], K)
        x, Wg, idx_d = dev(L["x"]), dev(L["W_g"]), dev(o_idx)
        f, P, aux = (host(t) for t in layer.router_stats(x, Wg, idx_d, alpha=0.02))
        f2, P2, aux2 = (host(t) for t in layer.router_stats(x, Wg, idx_d, alpha=0.02))
        layer.sync_status()
    finally:
        layer.close()
    of, oP, oaux = oracle.router_stats(L["x"], L["W_g"], o_idx, 0.02)
    # integer counts: f is exact up to the one fp32 division
    assert np.allclose(f, of, rtol=1e-6, atol=0)
    # P: fp32 logits and softmax, fp32 sum over T tokens
    assert np.allclose(P, oP, rtol=1e-4, atol=1e-6), np.abs(P - oP).max()
    assert abs(float(aux[0]) - oaux) <= 1e-4 * oaux
    # deterministic: a second call gives bit-identical results
    assert np.array_equal(f, f2) and np.array_equal(P, P2) and np.array_equal(aux, aux2)
    assert abs(float(P.sum()) - 1.0) < 1e-4
