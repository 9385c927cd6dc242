"""4-bit expert path vs the fp64 oracle, through the C ABI (needs a B200).

Weight quantisation is compared code for code with the oracle's (codes, block
scales, matrix scales); the layer runs on the oracle's codes and is compared
with the oracle's layer of the dequantised weights under the oracle's
routing (tokens whose GPU routing agrees); the hidden layer H after GEMM1 is
compared row by row with numpy on the dequantised weights, which locates any
wrong column or row of the converted weight tiles."""
import zlib

import numpy as np
import pytest

import moe_inputs as mi
import oracle
from gpu_helpers import (TOL_Y, agreeing_tokens, compare_routing, dev, host, read_workspace, rel_l2,
                         require_cuda, stratified_sample, y_as_f64)

pytestmark = pytest.mark.gpu


def seed_of(name: str) -> int:
    return zlib.crc32(name.encode()) % 1000


def quantize_gpu(w: np.ndarray):
    import sparse_mixture_experts_24_b200 as m
    torch = require_cuda()
    q = m.quantize_weights_fp4(dev(w))
    torch.cuda.synchronize()
    return tuple(host(t) for t in q)


WQ_CASES = [
    # name, n, rows, cols, dtype
    ("fp4q_bf16", 3, 64, 96, "bf16"),
    ("fp4q_f32", 2, 32, 64, "f32"),
    ("fp4q_bf16_wide", 1, 128, 4160, "bf16"),
    ("fp4q_bf16_tall", 2, 1024, 32, "bf16"),
]


@pytest.mark.parametrize("case", WQ_CASES, ids=[c[0] for c in WQ_CASES])
def test_fp4_quantization_matches_oracle(case):
    name, n, rows, cols, dt = case
    rng = np.random.default_rng(seed_of(name))
    w = (rng.standard_normal((n, rows, cols)) * rng.choice([1e-3, 1.0, 40.0], size=(n, 1, cols))).astype(np.float32)
    w[0, :16, 3] = 0.0                 # a zero block: scale code 0, codes 0
    w[0, 16:32, 4] = -0.0
    w[-1, :, 7] *= 1e-6                # blocks whose scale underflows towards the E4M3 subnormals
    w = mi.f32_to_bf16_bits(w) if dt == "bf16" else w
    c, b, t = quantize_gpu(w)
    c_ref, b_ref, t_ref = oracle.quantize_weights_fp4(w)
    assert np.array_equal(t, t_ref), (t, t_ref)
    assert np.array_equal(b, b_ref), "%d block scales differ" % int((b != b_ref).sum())
    diff = np.nonzero(c != c_ref)
    assert diff[0].size == 0, "%d code bytes differ, first at %s: %s vs %s" % (
        diff[0].size, [int(a[0]) for a in diff], int(c[tuple(a[0] for a in diff)]), int(c_ref[tuple(a[0] for a in diff)]))


def test_fp4_quantization_ties_and_saturation():
    """Columns whose values sit on E2M1 halfway points after scaling: a column
    with maximum 6 * 448 * st has block scale 448 and matrix scale st, so the
    quotients are the chosen values exactly."""
    vals = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 0.1, 2.9, 4.9, 5.9, 6.0, -0.25, -1.75, -5.0, 0.0],
                    np.float32)
    cols = 32
    w = np.zeros((1, 16, cols), np.float32)
    for c in range(cols):
        w[0, :, c] = np.roll(vals, c)
    w *= np.float32(1.75)              # 1.75 = 448 * 2^-8: quotient = value, scale exact
    w[0, 0, :] = 6.0 * 1.75            # every block maximum 6 * 1.75 -> matrix scale 2^-8
    c, b, t = quantize_gpu(w)
    c_ref, b_ref, t_ref = oracle.quantize_weights_fp4(w)
    assert t_ref[0] == np.float32(2.0 ** -8) and np.array_equal(t, t_ref)
    assert np.array_equal(b, b_ref) and np.array_equal(c, c_ref)


def run_fp4(cfg, L, q, factor=0.0):
    import sparse_mixture_experts_24_b200 as m
    torch = require_cuda()
    layer = m.MoELayer(cfg.n, cfg.K, cfg.d, cfg.ffn, "bf16")
    try:
        if factor:
            layer.set_capacity_factor(factor)
        qd = [tuple(dev(a) for a in t) for t in q]
        y, idx, w = layer.forward_fp4(dev(L["x"]), dev(L["W_g"]), *qd)
        layer.sync_status()
        torch.cuda.synchronize()
        R = cfg.T * cfg.K
        H = read_workspace(layer, "H", R, cfg.ffn, np.uint16)
        _, offsets, row_token, token_row = (host(a) for a in layer.dispatch(idx))
        return host(y), host(idx), host(w), H, offsets, row_token, token_row
    finally:
        layer.close()


def silu(z):
    return z / (1.0 + np.exp(-z))


FWD_CASES = [
    # name, T, d, ffn, n, K
    ("fp4_ragged", 300, 256, 320, 8, 2),
    ("fp4_tails", 77, 320, 192, 4, 1),
    ("fp4_T1", 1, 256, 256, 8, 2),
    ("fp4_d64_n64", 700, 64, 64, 64, 4),
    ("fp4_big_segments", 1500, 384, 512, 4, 2),
]


@pytest.mark.parametrize("case", FWD_CASES, ids=[c[0] for c in FWD_CASES])
def test_fp4_layer_matches_oracle(case):
    name, T, d, F, n, K = case
    cfg = mi.custom_config(name, T=T, d=d, ffn=F, n=n, K=K, dtype="bf16")
    L = mi.make_layer(cfg, seed=seed_of(name))
    q = [oracle.quantize_weights_fp4(L[w]) for w in ("w1", "w3", "w2")]
    deq = [oracle.dequantize_fp4(*t) for t in q]
    y, idx, w, H, offsets, row_token, _ = run_fp4(cfg, L, q)
    o_idx, o_gate, o_logits = oracle.router(L["x"], L["W_g"], K)
    compare_routing(idx, w, o_idx, o_gate, o_logits, L["x"], L["W_g"], K)
    # H rows against numpy on the dequantised weights (GEMM1 and the converters)
    R = int(offsets[-1])
    seg = np.searchsorted(offsets, np.arange(R), side="right") - 1
    xr = mi.as_f32(L["x"]).astype(np.float64)[row_token[:R]]
    Hg = mi.as_f32(H[:R]).astype(np.float64)
    for e in np.unique(seg):
        rows = seg == e
        a = xr[rows] @ deq[0][e]
        b = xr[rows] @ deq[1][e]
        ref = silu(a) * b
        err = np.linalg.norm(Hg[rows] - ref, axis=1) / np.maximum(np.linalg.norm(ref, axis=1), 1e-30)
        assert err.max() < 2e-2, (e, err.max(), np.argmax(err))
    # the layer against the oracle's 4-bit layer under its own routing
    agree = agreeing_tokens(idx, o_idx)
    y_ref = oracle.forward_fp4(L["x"], o_idx, o_gate, *q)
    yg = y_as_f64(y)
    err = rel_l2(yg[agree], y_ref[agree])
    assert err <= TOL_Y["bf16"], err
    per_tok = np.linalg.norm(yg - y_ref, axis=1)[agree] / np.maximum(np.linalg.norm(y_ref, axis=1)[agree], 1e-30)
    assert per_tok.max() <= 5 * TOL_Y["bf16"], per_tok.max()


def test_fp4_capacity_drops_like_bf16():
    name, T, d, F, n, K = "fp4_capacity", 600, 128, 192, 8, 2
    cfg = mi.custom_config(name, T=T, d=d, ffn=F, n=n, K=K, dtype="bf16", skew=True)
    L = mi.make_layer(cfg, seed=seed_of(name))
    q = [oracle.quantize_weights_fp4(L[w]) for w in ("w1", "w3", "w2")]
    C = int(np.ceil(1.0 * T * K / n))
    y, idx, w, _, offsets, _, token_row = run_fp4(cfg, L, q, factor=1.0)
    o_idx, o_gate, _ = oracle.router(L["x"], L["W_g"], K)
    assert (idx == o_idx).all(), "skewed case should route without near-ties"
    _, o_off, _, o_tr = oracle.dispatch_capacity(o_idx, n, C)
    assert np.array_equal(offsets, o_off) and np.array_equal(token_row, o_tr)
    dropped = o_tr < 0
    assert dropped.any()
    y_ref = oracle.forward_fp4(L["x"], o_idx, np.where(dropped, 0.0, o_gate), *q)
    assert rel_l2(y_as_f64(y), y_ref) <= TOL_Y["bf16"]


def test_fp4_rejects_fp32_handle_and_bad_shapes():
    import sparse_mixture_experts_24_b200 as m
    torch = require_cuda()
    layer = m.MoELayer(8, 2, 128, 128, "f32")
    try:
        x = torch.zeros((4, 128), dtype=torch.float32, device="cuda")
        z = (x, x, x)
        with pytest.raises(m.MoEError) as ei:
            layer.forward_fp4(x, x, z, z, z)
        assert ei.value.status == m.MOE_ERR_UNSUPPORTED
    finally:
        layer.close()
    w = torch.zeros((1, 24, 64), dtype=torch.bfloat16, device="cuda")   # rows not a multiple of 16
    with pytest.raises(m.MoEError) as ei:
        m.quantize_weights_fp4(w)
    assert ei.value.status == m.MOE_ERR_INVALID_ARG


def test_fp4_full_size_decode():
    """The decode workload with 4-bit experts: GPU quantisation of the full
    weights equals the oracle's, and y on an expert-stratified token sample
    equals the oracle's 4-bit layer."""
    import sparse_mixture_experts_24_b200 as m
    torch = require_cuda()
    cfg = mi.CONFIGS["decode"]
    L = mi.make_layer(cfg, seed=0)
    q = [oracle.quantize_weights_fp4(L[w]) for w in ("w1", "w3", "w2")]
    for wname, ref in zip(("w1", "w3", "w2"), q):
        got = m.quantize_weights_fp4(dev(L[wname]))
        torch.cuda.synchronize()
        for g, r in zip(got, ref):
            assert np.array_equal(host(g), r), wname
        del got
    layer = m.MoELayer(cfg.n, cfg.K, cfg.d, cfg.ffn, "bf16")
    try:
        y, idx, w = layer.forward_fp4(dev(L["x"]), dev(L["W_g"]), *[tuple(dev(a) for a in t) for t in q])
        layer.sync_status()
        y, idx, w = host(y), host(idx), host(w)
    finally:
        layer.close()
    o_idx, o_gate, o_logits = oracle.router(L["x"], L["W_g"], cfg.K)
    compare_routing(idx, w, o_idx, o_gate, o_logits, L["x"], L["W_g"], cfg.K)
    pick = stratified_sample(o_idx, cfg.n, 16)
    pick = pick[(idx[pick] == o_idx[pick]).all(axis=1)]
    y_ref = oracle.forward_fp4(L["x"][pick], o_idx[pick], o_gate[pick], *q)
    assert rel_l2(y_as_f64(y)[pick], y_ref) <= TOL_Y["bf16"]
