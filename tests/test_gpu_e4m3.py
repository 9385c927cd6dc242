"""E4M3 expert path vs the fp64 oracle, through the C ABI (needs a B200).

Weight quantisation is compared code for code and scale for scale with the
oracle's; the layer is compared with the oracle's E4M3 layer under the
oracle's own routing (on the tokens whose GPU routing agrees), the gathered x
codes with the oracle's codes of the same tokens, and the hidden-row codes by
the properties that define them (the row scale, and each code a nearest E4M3
value of the fp32 quotient, ties to even)."""
import zlib

import numpy as np
import pytest

import moe_inputs as mi
import oracle
from gpu_helpers import (PER_TOKEN_FACTOR, TOL_Y, block_covering_sample, blocks_covered, compare_routing, dev,
                         host, read_workspace, rel_l2, require_cuda, stratified_sample, y_as_f64)

pytestmark = pytest.mark.gpu

TABLE = np.array([oracle.e4m3_decode(c) for c in range(256)])
FINITE = np.unique(TABLE[np.isfinite(TABLE)])


def seed_of(name: str) -> int:
    return zlib.crc32(name.encode()) % 1000


def quantize_gpu(w: np.ndarray):
    import sparse_mixture_experts_24_b200 as m
    torch = require_cuda()
    q, s = m.quantize_weights_e4m3(dev(w))
    torch.cuda.synchronize()
    return host(q), host(s)


def check_nearest_codes(vals: np.ndarray, scales: np.ndarray, codes: np.ndarray) -> None:
    """Each code is an E4M3 value nearest to fp32(v / scale) (saturating at
    +-448), and a code halfway between two values has an even mantissa."""
    q = (vals.astype(np.float32) / scales.astype(np.float32)[:, None]).astype(np.float64)
    qc = np.clip(q, -448.0, 448.0)
    pos = np.clip(np.searchsorted(FINITE, qc), 1, FINITE.size - 1)
    lo, hi = FINITE[pos - 1], FINITE[pos]
    d_lo, d_hi = np.abs(qc - lo), np.abs(hi - qc)
    best = np.minimum(d_lo, d_hi)
    got = TABLE[codes]
    assert np.all(np.abs(got - qc) == best), "a code is not a nearest E4M3 value"
    tie = (d_lo == d_hi) & (lo != hi)
    assert np.all((codes[tie] & 1) == 0), "a tie did not round to the even mantissa"


def check_row_scales(vals: np.ndarray, scales: np.ndarray) -> None:
    amax = np.abs(vals.astype(np.float32)).max(axis=1)
    want = np.where(amax > 0, amax / np.float32(448.0), np.float32(1.0)).astype(np.float32)
    assert np.array_equal(scales, want)


WQ_CASES = [
    # name, n, rows, cols, dtype
    ("wq_bf16", 3, 200, 96, "bf16"),
    ("wq_bf16_one_row", 2, 1, 64, "bf16"),
    ("wq_f32_ragged_rows", 2, 130, 48, "f32"),
    ("wq_bf16_wide", 1, 64, 4160, "bf16"),
]


@pytest.mark.parametrize("case", WQ_CASES, ids=[c[0] for c in WQ_CASES])
def test_weight_quantization_matches_oracle(case):
    name, n, rows, cols, dt = case
    rng = np.random.default_rng(seed_of(name))
    w = (rng.standard_normal((n, rows, cols)) * rng.choice([1e-3, 1.0, 30.0], size=(n, 1, cols))).astype(np.float32)
    w[0, :, 1] = 0.0                  # an all-zero column: scale 1, codes 0
    if rows > 1:
        w[-1, 0, 2] = -0.0
    w = mi.f32_to_bf16_bits(w) if dt == "bf16" else w
    q, s = quantize_gpu(w)
    q_ref, s_ref = oracle.quantize_weights_e4m3(w)
    assert np.array_equal(s, s_ref), np.abs(s - s_ref).max()
    assert np.array_equal(q, q_ref), "%d codes differ" % int((q != q_ref).sum())


def test_codec_matches_oracle():
    """Columns whose maximum is 448 have scale 1, so every other value of the
    column is coded as itself: the E4M3 rounding of chosen fp32 values
    (halfway cases, subnormals, the top of the range) against the oracle."""
    special = [1.0 + 1 / 16, 1.125 + 1 / 16, 2.0 ** -10, 3 * 2.0 ** -10, 5 * 2.0 ** -10, 2.0 ** -6,
               np.nextafter(np.float32(2.0 ** -6), np.float32(0)), 2.0 ** -9, 2.0 ** -11, 1e-30, 0.0,
               440.0, 447.0, 432.0 + 8.0, np.nextafter(np.float32(448), np.float32(0)), 416.0 + 8.0,
               17.0, 18.0, 19.0, 0.3, 1 / 3, 2.5, 3.5, 7.75, 240.0, 248.0]
    rng = np.random.default_rng(7)
    vals = np.concatenate([special, [-v for v in special],
                           rng.standard_normal(2000) * 10.0 ** rng.uniform(-4, 2.6, 2000)]).astype(np.float32)
    vals = np.clip(vals, -448.0, 448.0)
    cols = 16
    rows_per_col = -(-vals.size // cols)
    w = np.zeros((1, rows_per_col + 1, cols), np.float32)
    w[0, 0, :] = 448.0
    w[0, 1:, :].reshape(-1)[:vals.size] = vals
    q, s = quantize_gpu(w)
    q_ref, s_ref = oracle.quantize_weights_e4m3(w)
    assert np.all(s == 1.0) and np.array_equal(s, s_ref)
    assert np.array_equal(q, q_ref), [(float(w.reshape(-1)[i]), int(q.reshape(-1)[i]), int(q_ref.reshape(-1)[i]))
                                      for i in np.nonzero(q.reshape(-1) != q_ref.reshape(-1))[0][:5]]


def run_e4m3(cfg, L, q, factor=0.0):
    """GPU E4M3 layer on the oracle's codes; returns y, idx, w and the
    workspace buffers X8, XS, H8, HS, H and the dispatch row_token."""
    import sparse_mixture_experts_24_b200 as m
    torch = require_cuda()
    layer = m.MoELayer(cfg.n, cfg.K, cfg.d, cfg.ffn, "bf16")
    try:
        if factor:
            layer.set_capacity_factor(factor)
        qd = [dev(a) for a in q]
        y, idx, w = layer.forward_e4m3(dev(L["x"]), dev(L["W_g"]), *qd)
        layer.sync_status()
        torch.cuda.synchronize()
        R = cfg.T * cfg.K
        out = {name: read_workspace(layer, name, R, cols, dt)
               for name, dt, cols in (("X8", np.uint8, cfg.d), ("H8", np.uint8, cfg.ffn), ("XS", np.float32, 1),
                                      ("HS", np.float32, 1), ("H", np.uint16, cfg.ffn))}
        _, offsets, row_token, token_row = (host(a) for a in layer.dispatch(idx))
        return host(y), host(idx), host(w), out, offsets, row_token, token_row
    finally:
        layer.close()


def oracle_codes(L):
    return [a for w in ("w1", "w3", "w2") for a in oracle.quantize_weights_e4m3(L[w])]


FWD_CASES = [
    # name, T, d, ffn, n, K
    ("e4m3_ragged", 300, 256, 320, 8, 2),
    ("e4m3_tails", 77, 320, 192, 4, 1),
    ("e4m3_T1", 1, 256, 256, 8, 2),
    ("e4m3_d64_n64", 700, 64, 64, 64, 4),
    ("e4m3_big_segments", 1500, 384, 512, 4, 2),
    ("e4m3_many_long_rows", 1200, 256, 4608, 8, 2),   # 2,400 H rows of 4,608: 128-thread blocks, two passes
]


@pytest.mark.parametrize("case", FWD_CASES, ids=[c[0] for c in FWD_CASES])
def test_e4m3_layer_matches_oracle(case):
    name, T, d, F, n, K = case
    cfg = mi.custom_config(name, T=T, d=d, ffn=F, n=n, K=K, dtype="bf16")
    L = mi.make_layer(cfg, seed=seed_of(name))
    q = oracle_codes(L)
    y, idx, w, ws, offsets, row_token, _ = run_e4m3(cfg, L, q)
    o_idx, o_gate, o_logits = oracle.router(L["x"], L["W_g"], K)
    compare_routing(idx, w, o_idx, o_gate, o_logits, L["x"], L["W_g"], K)
    R = int(offsets[-1])
    assert R == T * K
    # gathered x codes: the oracle's codes of each row's token
    xq, xs = oracle.quantize_weights_e4m3(mi.as_f32(L["x"]).T[None].copy())
    xq, xs = xq[0].T, xs[0]
    assert np.array_equal(ws["XS"][:R, 0], xs[row_token[:R]])
    assert np.array_equal(ws["X8"][:R], xq[row_token[:R]])
    # hidden-row codes: scale and nearest-value properties on the GPU's own H
    H = mi.as_f32(ws["H"][:R])
    check_row_scales(H, ws["HS"][:R, 0])
    check_nearest_codes(H, ws["HS"][:R, 0], ws["H8"][:R])
    # the layer against the oracle's E4M3 layer under the oracle's routing
    agree = (idx == o_idx).all(axis=1)
    assert agree.mean() > 0.99
    y_ref = oracle.forward_e4m3(L["x"], o_idx, o_gate, *q)
    yg = y_as_f64(y)
    err = rel_l2(yg[agree], y_ref[agree])
    assert err <= TOL_Y["bf16"], err
    per_tok = np.linalg.norm(yg - y_ref, axis=1)[agree] / np.maximum(np.linalg.norm(y_ref, axis=1)[agree], 1e-30)
    assert per_tok.max() <= 5 * TOL_Y["bf16"], per_tok.max()
    # and it is a quantised layer: away from the exact one, within E4M3's band
    y_exact = oracle.forward_with_routing(L["x"], o_idx, o_gate, L["w1"], L["w3"], L["w2"])
    band = rel_l2(yg[agree], y_exact[agree])
    assert 2e-3 < band < 0.1, band


def test_e4m3_capacity_drops_like_bf16():
    """With a capacity factor the E4M3 path keeps the same pairs as the
    oracle's capacity dispatch; dropped pairs add nothing."""
    name, T, d, F, n, K = "e4m3_capacity", 600, 128, 192, 8, 2
    cfg = mi.custom_config(name, T=T, d=d, ffn=F, n=n, K=K, dtype="bf16", skew=True)
    L = mi.make_layer(cfg, seed=seed_of(name))
    q = oracle_codes(L)
    factor = 1.0
    C = int(np.ceil(factor * T * K / n))
    y, idx, w, _, offsets, _, token_row = run_e4m3(cfg, L, q, factor=factor)
    o_idx, o_gate, o_logits = oracle.router(L["x"], L["W_g"], K)
    assert (idx == o_idx).all(), "skewed case should route without near-ties"
    _, o_off, _, o_tr = oracle.dispatch_capacity(o_idx, n, C)
    assert np.array_equal(offsets, o_off) and np.array_equal(token_row, o_tr)
    dropped = o_tr < 0
    assert dropped.any()
    y_ref = oracle.forward_e4m3(L["x"], o_idx, np.where(dropped, 0.0, o_gate), *q)
    assert rel_l2(y_as_f64(y), y_ref) <= TOL_Y["bf16"]


def test_e4m3_rejects_fp32_handle_and_accepts_T0():
    import sparse_mixture_experts_24_b200 as m
    torch = require_cuda()
    layer = m.MoELayer(8, 2, 128, 128, "f32")
    try:
        x = torch.zeros((4, 128), dtype=torch.float32, device="cuda")
        with pytest.raises(m.MoEError) as ei:
            layer.forward_e4m3(x, x, x, x, x, x, x, x)
        assert ei.value.status == m.MOE_ERR_UNSUPPORTED
    finally:
        layer.close()
    layer = m.MoELayer(8, 2, 128, 128, "bf16")
    try:
        x = torch.zeros((0, 128), dtype=torch.bfloat16, device="cuda")
        z = torch.zeros(16, dtype=torch.uint8, device="cuda")
        y, _, _ = layer.forward_e4m3(x, z, z, z, z, z, z, z)
        assert y.shape == (0, 128)
    finally:
        layer.close()


def test_e4m3_full_size_decode():
    """The decode workload (Mixtral 8x7B layer shapes) with E4M3 experts: the
    GPU quantisation of the full weights equals the oracle's, and y on an
    expert-stratified token sample equals the oracle's E4M3 layer."""
    import sparse_mixture_experts_24_b200 as m
    torch = require_cuda()
    cfg = mi.CONFIGS["decode"]
    L = mi.make_layer(cfg, seed=0)
    q = oracle_codes(L)
    for w, (qr, sr) in zip(("w1", "w3", "w2"), ((q[0], q[1]), (q[2], q[3]), (q[4], q[5]))):
        qg, sg = m.quantize_weights_e4m3(dev(L[w]))
        torch.cuda.synchronize()
        assert np.array_equal(host(sg), sr), w
        assert np.array_equal(host(qg), qr), w
        del qg, sg
    layer = m.MoELayer(cfg.n, cfg.K, cfg.d, cfg.ffn, "bf16")
    try:
        y, idx, w = layer.forward_e4m3(dev(L["x"]), dev(L["W_g"]), *[dev(a) for a in q])
        layer.sync_status()
        y, idx, w = host(y), host(idx), host(w)
    finally:
        layer.close()
    o_idx, o_gate, o_logits = oracle.router(L["x"], L["W_g"], cfg.K)
    compare_routing(idx, w, o_idx, o_gate, o_logits, L["x"], L["W_g"], cfg.K)
    pick = stratified_sample(o_idx, cfg.n, 24)
    pick = pick[(idx[pick] == o_idx[pick]).all(axis=1)]
    y_ref = oracle.forward_e4m3(L["x"][pick], o_idx[pick], o_gate[pick], *q)
    err = rel_l2(y_as_f64(y)[pick], y_ref)
    assert err <= TOL_Y["bf16"], err


@pytest.mark.parametrize("name", ["prefill", "skew_prefill"])
def test_e4m3_full_size_prefill(name):
    """The prefill workloads (Mixtral layer shapes, 4,096 and 16,384 tokens,
    the second with most of them on one expert) with E4M3 experts, in the
    benchmark's launch configuration: routing on every token; y on a token
    sample with a row in every (expert, 128-row M-block) of both GEMMs, the
    ragged end of every segment included, against the oracle's E4M3 layer,
    in aggregate and per token."""
    import sparse_mixture_experts_24_b200 as m
    torch = require_cuda()
    cfg = mi.CONFIGS[name]
    L = mi.make_layer(cfg, seed=0)
    q = oracle_codes(L)
    layer = m.MoELayer(cfg.n, cfg.K, cfg.d, cfg.ffn, "bf16")
    try:
        qd = [dev(a) for a in q]
        y, idx, w = layer.forward_e4m3(dev(L["x"]), dev(L["W_g"]), *qd)
        layer.sync_status()
        y, idx, w = host(y), host(idx), host(w)
        del qd
    finally:
        layer.close()
    torch.cuda.empty_cache()
    o_idx, o_gate, o_logits = oracle.router(L["x"], L["W_g"], cfg.K)
    compare_routing(idx, w, o_idx, o_gate, o_logits, L["x"], L["W_g"], cfg.K)
    pick, nblk = block_covering_sample(o_idx, cfg.n, count=256)
    assert blocks_covered(pick, o_idx, cfg.n) == nblk
    pick = pick[(idx[pick] == o_idx[pick]).all(axis=1)]
    assert blocks_covered(pick, o_idx, cfg.n) >= nblk - 2
    y_ref = oracle.forward_e4m3(L["x"][pick], o_idx[pick], o_gate[pick], *q)
    yg = y_as_f64(y)[pick]
    assert np.isfinite(y_as_f64(y)).all()
    err = rel_l2(yg, y_ref)
    per_tok = np.linalg.norm(yg - y_ref, axis=1) / np.maximum(np.linalg.norm(y_ref, axis=1), 1e-30)
    print("\n%s E4M3 y rel-L2 on %d tokens (%d M-blocks): %.3e, worst token %.3e"
          % (name, pick.size, nblk, err, per_tok.max()))
    assert err <= TOL_Y["bf16"], err
    assert per_tok.max() <= PER_TOKEN_FACTOR * TOL_Y["bf16"], per_tok.max()


def test_e4m3_many_rows_sampled():
    """20,000 tokens over 16 experts, compared on a token sample."""
    import sparse_mixture_experts_24_b200 as m
    torch = require_cuda()
    name, T, d, F, n, K = "e4m3_many_rows", 20000, 256, 320, 16, 2
    cfg = mi.custom_config(name, T=T, d=d, ffn=F, n=n, K=K, dtype="bf16")
    L = mi.make_layer(cfg, seed=seed_of(name))
    q = oracle_codes(L)
    layer = m.MoELayer(n, K, d, F, "bf16")
    try:
        y, idx, w = layer.forward_e4m3(dev(L["x"]), dev(L["W_g"]), *[dev(a) for a in q])
        layer.sync_status()
        torch.cuda.synchronize()
        y, idx, w = host(y), host(idx), host(w)
    finally:
        layer.close()
    o_idx, o_gate, o_logits = oracle.router(L["x"], L["W_g"], K)
    compare_routing(idx, w, o_idx, o_gate, o_logits, L["x"], L["W_g"], K)
    pick = stratified_sample(o_idx, n, 300)
    pick = pick[(idx[pick] == o_idx[pick]).all(axis=1)]
    y_ref = oracle.forward_e4m3(L["x"][pick], o_idx[pick], o_gate[pick], *q)
    assert rel_l2(y_as_f64(y)[pick], y_ref) <= TOL_Y["bf16"]
