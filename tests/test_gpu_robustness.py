"""Failure detection, workspace reuse and growth, pointer changes, streams and
extreme sizes, through the C ABI (needs a B200)."""
import numpy as np
import pytest

import moe_inputs as mi
import oracle
from gpu_helpers import TOL_Y, agreeing_tokens, compare_routing, dev, host, rel_l2, require_cuda, y_as_f64

pytestmark = pytest.mark.gpu


def _check_layer(cfg, L, y, idx, w):
    o_idx, o_gate, o_logits = oracle.router(L["x"], L["W_g"], cfg.K)
    compare_routing(idx, w, o_idx, o_gate, o_logits, L["x"], L["W_g"], cfg.K)
    y_ref, _, _ = oracle.moe_forward(L["x"], L["W_g"], L["w1"], L["w3"], L["w2"], cfg.K)
    agree = agreeing_tokens(idx, o_idx)
    assert rel_l2(y_as_f64(y)[agree], y_ref[agree]) <= TOL_Y[cfg.dtype]


def test_bounded_wait_runs_out_and_the_context_stays_usable():
    """A kernel waits on a barrier nothing completes; its bounded wait gives up
    after ~2 ms, the host reads MOE_ERR_TIMEOUT, the flag clears, and the next
    layer call is correct."""
    import sparse_mixture_experts_24_b200 as m
    torch = require_cuda()
    cfg = mi.custom_config("after_timeout", T=100, d=128, ffn=128, n=4, K=2, dtype="bf16")
    L = mi.make_layer(cfg, seed=2)
    layer = m.MoELayer(cfg.n, cfg.K, cfg.d, cfg.ffn, "bf16")
    try:
        m.moe_selftest_timeout(layer.h, 2000)
        with pytest.raises(m.MoEError) as ei:
            layer.sync_status()
        assert ei.value.status == m.MOE_ERR_TIMEOUT
        layer.sync_status()  # cleared
        y, idx, w = layer.forward(*[dev(L[k]) for k in ("x", "W_g", "w1", "w3", "w2")])
        layer.sync_status()
        _check_layer(cfg, L, host(y), host(idx), host(w))
        with pytest.raises(m.MoEError):
            m.moe_selftest_timeout(layer.h, 0)
    finally:
        layer.close()
    torch.cuda.synchronize()


def test_workspace_grows_and_is_reused():
    import sparse_mixture_experts_24_b200 as m
    require_cuda()
    d, F, n, K = 128, 128, 8, 2
    layer = m.MoELayer(n, K, d, F, "bf16")
    try:
        big = mi.make_layer(mi.custom_config("g", T=700, d=d, ffn=F, n=n, K=K, dtype="bf16"), seed=8)
        W = [dev(big[k]) for k in ("W_g", "w1", "w3", "w2")]
        ptrs = []
        for T in (10, 700, 50, 700, 1):
            cfg = mi.custom_config("g%d" % T, T=T, d=d, ffn=F, n=n, K=K, dtype="bf16")
            L = dict(big, x=big["x"][:T].copy())
            y, idx, w = layer.forward(dev(L["x"]), *W)
            layer.sync_status()
            _check_layer(cfg, L, host(y), host(idx), host(w))
            ptrs.append(m.moe_workspace_view(layer.h, "H")[0])
        assert ptrs[2] == ptrs[1] and ptrs[3] == ptrs[1] and ptrs[4] == ptrs[1]  # no reallocation
    finally:
        layer.close()


def test_reserve_then_forward_allocates_nothing_more():
    import sparse_mixture_experts_24_b200 as m
    require_cuda()
    cfg = mi.custom_config("res", T=300, d=128, ffn=256, n=8, K=2, dtype="bf16")
    L = mi.make_layer(cfg, seed=9)
    layer = m.MoELayer(cfg.n, cfg.K, cfg.d, cfg.ffn, "bf16")
    try:
        layer.reserve(1000)
        p0 = m.moe_workspace_view(layer.h, "O")
        y, idx, w = layer.forward(*[dev(L[k]) for k in ("x", "W_g", "w1", "w3", "w2")])
        layer.sync_status()
        assert m.moe_workspace_view(layer.h, "O") == p0 and p0[1] == 2000
        _check_layer(cfg, L, host(y), host(idx), host(w))
    finally:
        layer.close()


def test_new_weight_and_activation_pointers_are_picked_up():
    """The TMA descriptors over caller tensors follow pointer changes (weights,
    and x on the tensor-core router path, T >= 512)."""
    import sparse_mixture_experts_24_b200 as m
    require_cuda()
    cfg = mi.custom_config("ptr", T=600, d=128, ffn=128, n=4, K=2, dtype="bf16")
    layer = m.MoELayer(cfg.n, cfg.K, cfg.d, cfg.ffn, "bf16")
    try:
        for seed in (21, 22, 23):
            L = mi.make_layer(cfg, seed=seed)
            y, idx, w = layer.forward(*[dev(L[k]) for k in ("x", "W_g", "w1", "w3", "w2")])
            layer.sync_status()
            _check_layer(cfg, L, host(y), host(idx), host(w))
    finally:
        layer.close()


def test_two_handles_and_a_side_stream():
    import sparse_mixture_experts_24_b200 as m
    torch = require_cuda()
    c1 = mi.custom_config("h1", T=200, d=128, ffn=192, n=8, K=2, dtype="bf16")
    c2 = mi.custom_config("h2", T=90, d=64, ffn=128, n=5, K=3, dtype="f32")
    L1, L2 = mi.make_layer(c1, seed=31), mi.make_layer(c2, seed=32)
    a = m.MoELayer(c1.n, c1.K, c1.d, c1.ffn, "bf16")
    b = m.MoELayer(c2.n, c2.K, c2.d, c2.ffn, "f32")
    s = torch.cuda.Stream()
    try:
        t1 = [dev(L1[k]) for k in ("x", "W_g", "w1", "w3", "w2")]
        t2 = [dev(L2[k]) for k in ("x", "W_g", "w1", "w3", "w2")]
        torch.cuda.synchronize()
        with torch.cuda.stream(s):
            y1, i1, w1 = a.forward(*t1, stream=s)
            y2, i2, w2 = b.forward(*t2, stream=s)
            y1b, i1b, w1b = a.forward(*t1, stream=s)
        s.synchronize()
        a.sync_status(s)
        b.sync_status(s)
        _check_layer(c1, L1, host(y1), host(i1), host(w1))
        _check_layer(c2, L2, host(y2), host(i2), host(w2))
        assert np.array_equal(host(y1), host(y1b))  # deterministic
    finally:
        a.close()
        b.close()


@pytest.mark.parametrize("case", [
    ("all_256_experts_dense", 20, 64, 64, 256, 256, "bf16"),
    ("many_tokens", 70000, 64, 64, 8, 2, "bf16"),
    ("many_tokens_f32", 20000, 64, 64, 16, 3, "f32"),
    ("wide_d", 64, 8192, 128, 4, 2, "bf16"),
], ids=lambda c: c[0])
def test_extreme_sizes(case):
    import sparse_mixture_experts_24_b200 as m
    require_cuda()
    name, T, d, F, n, K, dt = case
    cfg = mi.custom_config(name, T=T, d=d, ffn=F, n=n, K=K, dtype=dt)
    L = mi.make_layer(cfg, seed=5)
    layer = m.MoELayer(n, K, d, F, dt)
    try:
        y, idx, w = layer.forward(*[dev(L[k]) for k in ("x", "W_g", "w1", "w3", "w2")])
        layer.sync_status()
        y, idx, w = host(y), host(idx), host(w)
    finally:
        layer.close()
    o_idx, o_gate, o_logits = oracle.router(L["x"], L["W_g"], K)
    compare_routing(idx, w, o_idx, o_gate, o_logits, L["x"], L["W_g"], K)
    agree = agreeing_tokens(idx, o_idx)
    sample = np.arange(T) if T <= 300 else np.random.default_rng(0).choice(T, 300, replace=False)
    sample = sample[agree[sample]]
    y_ref = oracle.forward_with_routing(L["x"][sample], o_idx[sample], o_gate[sample],
                                        L["w1"], L["w3"], L["w2"])
    assert rel_l2(y_as_f64(y[sample]), y_ref) <= TOL_Y[dt]


def test_zero_tokens_launch_nothing():
    import sparse_mixture_experts_24_b200 as m
    require_cuda()
    layer = m.MoELayer(8, 2, 64, 64, "bf16")
    try:
        c0 = m.moe_launch_count(layer.h)
        m.moe_forward(layer.h, 0, None, None, None, None, None, None, None, None)
        assert m.moe_launch_count(layer.h) == c0
    finally:
        layer.close()


NONFINITE_CASES = [
    # name, T, d, ffn, n, K, dtype: the token router, the tensor-core router (T >= 512
    # and n > 32), and the fp32 routers
    ("nf_token_router", 64, 256, 128, 8, 2, "bf16"),
    ("nf_tc_router", 600, 256, 128, 8, 2, "bf16"),
    ("nf_tc_router_n64", 300, 128, 128, 64, 4, "bf16"),
    ("nf_f32", 100, 128, 128, 8, 2, "f32"),
    ("nf_f32_n40", 100, 64, 64, 40, 3, "f32"),
]


@pytest.mark.parametrize("case", NONFINITE_CASES, ids=[c[0] for c in NONFINITE_CASES])
def test_nonfinite_tokens_stay_contained(case):
    """Rows of x holding NaN, +-inf or huge values: their results are
    unspecified, but every routing index stays a valid, distinct expert, the
    call reports no error, and every other token's routing and output equal
    the oracle's (tokens never mix)."""
    import sparse_mixture_experts_24_b200 as m
    require_cuda()
    name, T, d, F, n, K, dt = case
    cfg = mi.custom_config(name, T=T, d=d, ffn=F, n=n, K=K, dtype=dt)
    L = mi.make_layer(cfg, seed=9)
    xf = mi.as_f32(L["x"]).copy()
    bad = np.array([3, 7, 11, T - 1])
    xf[3, :] = np.nan
    xf[7, 0] = np.inf
    xf[11, 5] = -np.inf
    xf[T - 1, :] = 1e30
    x = mi.f32_to_bf16_bits(xf) if dt == "bf16" else xf
    layer = m.MoELayer(n, K, d, F, dt)
    try:
        y, idx, w = layer.forward(dev(x), *[dev(L[k]) for k in ("W_g", "w1", "w3", "w2")])
        layer.sync_status()
        y, idx, w = host(y), host(idx), host(w)
    finally:
        layer.close()
    assert ((idx >= 0) & (idx < n)).all()
    assert all(len(set(row)) == K for row in idx.tolist())
    good = np.setdiff1d(np.arange(T), bad)
    xg = x[good]
    o_idx, o_gate, o_logits = oracle.router(xg, L["W_g"], K)
    compare_routing(idx[good], w[good], o_idx, o_gate, o_logits, xg, L["W_g"], K)
    y_ref, _, _ = oracle.moe_forward(xg, L["W_g"], L["w1"], L["w3"], L["w2"], K)
    agree = agreeing_tokens(idx[good], o_idx)
    assert rel_l2(y_as_f64(y[good])[agree], y_ref[agree]) <= TOL_Y[dt]
