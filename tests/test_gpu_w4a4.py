"""4-bit weights and 4-bit activations on the block-scaled tensor cores vs the
fp64 oracle, through the C ABI (needs a B200).

The weight repacking is a pure permutation, checked byte for byte against a
numpy permutation of the same codes; the layer runs on the oracle's 4-bit
weights and is compared with the oracle's 4-bit weight-and-activation layer
under the oracle's routing (tokens whose GPU routing agrees)."""
import zlib

import numpy as np
import pytest

import moe_inputs as mi
import oracle
from gpu_helpers import (PER_TOKEN_FACTOR, TOL_Y, agreeing_tokens, block_covering_sample, blocks_covered,
                         compare_routing, dev, host, rel_l2, require_cuda, stratified_sample, y_as_f64)

pytestmark = pytest.mark.gpu


def seed_of(name: str) -> int:
    return zlib.crc32(name.encode()) % 1000


def numpy_pack(codes, bscale, pair=None):
    """The documented layout of moe_pack_weights_w4a4, written with numpy:
    the single matrix, or with pair = (codes, bscale) of w3 the gate/up pair
    whose packed column p is column 64 (p // 128) + p % 64 of w1 (p % 128 < 64)
    or of w3."""
    n, K, half = codes.shape
    N = 2 * half

    def nibbles(c):
        nib = np.empty((n, K, N), np.uint8)
        nib[:, :, 0::2], nib[:, :, 1::2] = c & 0xF, c >> 4
        return nib

    nib, bs = nibbles(codes), bscale
    if pair is not None:
        p = np.arange(2 * N)
        col = 64 * (p // 128) + p % 64
        from_w3 = (p % 128) >= 64
        nib = np.where(from_w3[None, None, :], nibbles(pair[0])[:, :, col], nib[:, :, col])
        bs = np.where(from_w3[None, None, :], pair[1][:, :, col], bscale[:, :, col])
        N = 2 * N
    kmaj = nib.transpose(0, 2, 1)                                   # [n][N][K]
    packed = (kmaj[:, :, 0::2] | (kmaj[:, :, 1::2] << 4)).astype(np.uint8)
    chunks = np.zeros((n, N // 128, K // 64, 512), np.uint8)
    c = np.arange(N)
    pos = 16 * (c % 32) + 4 * ((c % 128) // 32)
    for kb16 in range(K // 16):
        chunks[:, c // 128, kb16 // 4, pos + kb16 % 4] = bs[:, kb16, :]
    return packed, chunks


@pytest.mark.parametrize("shape", [(2, 64, 128), (3, 256, 384), (1, 512, 256)])
def test_pack_is_the_documented_permutation(shape):
    import sparse_mixture_experts_24_b200 as m
    torch = require_cuda()
    n, K, N = shape
    rng = np.random.default_rng(K + N)
    codes = rng.integers(0, 256, (n, K, N // 2), dtype=np.uint8)
    bscale = rng.integers(0, 0x7F, (n, K // 16, N), dtype=np.uint8)
    packed, chunks, _ = m.pack_weights_w4a4(dev(codes), dev(bscale), None)
    torch.cuda.synchronize()
    p_ref, c_ref = numpy_pack(codes, bscale)
    assert np.array_equal(host(packed), p_ref)
    assert np.array_equal(host(chunks), c_ref)


@pytest.mark.parametrize("shape", [(2, 64, 64), (3, 256, 192), (1, 128, 512)])
def test_pair_pack_is_the_documented_permutation(shape):
    import sparse_mixture_experts_24_b200 as m
    torch = require_cuda()
    n, K, N = shape
    rng = np.random.default_rng(7 * K + N)
    c1, c3 = (rng.integers(0, 256, (n, K, N // 2), dtype=np.uint8) for _ in range(2))
    b1, b3 = (rng.integers(0, 0x7F, (n, K // 16, N), dtype=np.uint8) for _ in range(2))
    packed, chunks, _, _ = m.pack_weights_w4a4(dev(c1), dev(b1), None, pair=(dev(c3), dev(b3), None))
    torch.cuda.synchronize()
    p_ref, c_ref = numpy_pack(c1, b1, pair=(c3, b3))
    assert np.array_equal(host(packed), p_ref)
    assert np.array_equal(host(chunks), c_ref)


def test_pack_rejects_bad_sizes():
    import sparse_mixture_experts_24_b200 as m
    torch = require_cuda()
    z = torch.zeros(1 << 16, dtype=torch.uint8, device="cuda")
    for rows, cols, pair in ((64, 64, False), (32, 128, False), (64, 96, True)):
        with pytest.raises(m.MoEError) as ei:
            m.moe_pack_weights_w4a4(1, rows, cols, z, z, z if pair else None, z if pair else None, z, z)
        assert ei.value.status == m.MOE_ERR_INVALID_ARG
    with pytest.raises(m.MoEError) as ei:                  # one pair pointer alone
        m.moe_pack_weights_w4a4(1, 64, 128, z, z, z, None, z, z)
    assert ei.value.status == m.MOE_ERR_INVALID_ARG


def prepared_weights(L):
    """Oracle 4-bit weights (logical layout) and their packed device form:
    the gate/up pair pack and w2."""
    import sparse_mixture_experts_24_b200 as m
    q = [oracle.quantize_weights_fp4(L[w]) for w in ("w1", "w3", "w2")]
    w13 = m.pack_weights_w4a4(*(dev(a) for a in q[0]), pair=tuple(dev(a) for a in q[1]))
    w2 = m.pack_weights_w4a4(*(dev(a) for a in q[2]))
    return q, (w13, w2)


FWD_CASES = [
    # name, T, d, ffn, n, K
    ("w4a4_small", 300, 256, 512, 8, 2),
    ("w4a4_tails", 77, 512, 256, 4, 1),
    ("w4a4_T1", 1, 256, 256, 8, 2),
    ("w4a4_n64", 700, 256, 256, 64, 4),
    ("w4a4_big_segments", 1500, 512, 768, 4, 2),
    ("w4a4_d2048_rows", 400, 2048, 256, 8, 2),   # 800 rows of 2,048: the warp-per-row quantiser
    ("w4a4_long_rows", 1300, 2560, 256, 8, 2),   # 2,600 rows of 2,560: 128-thread blocks per row
]


@pytest.mark.parametrize("tile", ["128x128", "128x32", "256x128", "256x32"])
@pytest.mark.parametrize("case", FWD_CASES, ids=[c[0] for c in FWD_CASES])
def test_w4a4_layer_matches_oracle(case, tile, monkeypatch):
    """Every tile shape on every case: 128 packed columns with two
    accumulators and 256 with one, each over 128-row and 32-row tiles."""
    import sparse_mixture_experts_24_b200 as m
    torch = require_cuda()
    cols, rows = tile.split("x")
    monkeypatch.setenv("MOE_W4A4_TILE", cols)
    monkeypatch.setenv("MOE_W4A4_ROWS", rows)
    name, T, d, F, n, K = case
    cfg = mi.custom_config(name, T=T, d=d, ffn=F, n=n, K=K, dtype="bf16")
    L = mi.make_layer(cfg, seed=seed_of(name))
    q, packed = prepared_weights(L)
    layer = m.MoELayer(n, K, d, F, "bf16")
    try:
        y, idx, w = layer.forward_w4a4(dev(L["x"]), dev(L["W_g"]), *packed)
        layer.sync_status()
        torch.cuda.synchronize()
        y, idx, w = host(y), host(idx), host(w)
    finally:
        layer.close()
    o_idx, o_gate, o_logits = oracle.router(L["x"], L["W_g"], K)
    compare_routing(idx, w, o_idx, o_gate, o_logits, L["x"], L["W_g"], K)
    agree = agreeing_tokens(idx, o_idx)
    y_ref = oracle.forward_w4a4(L["x"], o_idx, o_gate, *q)
    yg = y_as_f64(y)
    err = rel_l2(yg[agree], y_ref[agree])
    assert err <= TOL_Y["bf16"], err
    per_tok = np.linalg.norm(yg - y_ref, axis=1)[agree] / np.maximum(np.linalg.norm(y_ref, axis=1)[agree], 1e-30)
    assert per_tok.max() <= 5 * TOL_Y["bf16"], per_tok.max()
    # really 4-bit: away from the exact layer, inside the 4-bit band
    y_exact = oracle.forward_with_routing(L["x"], o_idx, o_gate, L["w1"], L["w3"], L["w2"])
    band = rel_l2(yg[agree], y_exact[agree])
    assert 0.03 < band < 0.4, band


@pytest.mark.parametrize("rows", ["128", "32"])
def test_w4a4_capacity_and_rejections(rows, monkeypatch):
    """Capacity dropping on both row-tile heights, and the argument checks."""
    import sparse_mixture_experts_24_b200 as m
    torch = require_cuda()
    monkeypatch.setenv("MOE_W4A4_ROWS", rows)
    name, T, d, F, n, K = "w4a4_capacity", 600, 256, 256, 8, 2
    cfg = mi.custom_config(name, T=T, d=d, ffn=F, n=n, K=K, dtype="bf16", skew=True)
    L = mi.make_layer(cfg, seed=seed_of(name))
    q, packed = prepared_weights(L)
    C = int(np.ceil(T * K / n))
    layer = m.MoELayer(n, K, d, F, "bf16")
    try:
        layer.set_capacity_factor(1.0)
        y, idx, w = layer.forward_w4a4(dev(L["x"]), dev(L["W_g"]), *packed)
        _, offsets, _, token_row = (host(a) for a in layer.dispatch(idx))
        layer.sync_status()
        y, idx = host(y), host(idx)
    finally:
        layer.close()
    o_idx, o_gate, _ = oracle.router(L["x"], L["W_g"], K)
    assert (idx == o_idx).all()
    _, o_off, _, o_tr = oracle.dispatch_capacity(o_idx, n, C)
    assert np.array_equal(offsets, o_off) and np.array_equal(token_row, o_tr)
    dropped = o_tr < 0
    assert dropped.any()
    y_ref = oracle.forward_w4a4(L["x"], o_idx, np.where(dropped, 0.0, o_gate), *q)
    assert rel_l2(y_as_f64(y), y_ref) <= TOL_Y["bf16"]
    # d or ffn not a multiple of 256, an fp32 handle
    for args in ((8, 2, 128, 256, "bf16"), (8, 2, 256, 256, "f32")):
        layer = m.MoELayer(*args)
        try:
            x = torch.zeros((4, args[2]), dtype=torch.bfloat16 if args[4] == "bf16" else torch.float32,
                            device="cuda")
            with pytest.raises(m.MoEError) as ei:
                layer.forward_w4a4(x, x, (x, x, x, x), (x, x, x))
            assert ei.value.status == m.MOE_ERR_UNSUPPORTED
        finally:
            layer.close()


def test_w4a4_full_size_decode():
    """The decode workload (Mixtral layer shapes) with 4-bit weights and
    activations on an expert-stratified token sample."""
    import sparse_mixture_experts_24_b200 as m
    torch = require_cuda()
    cfg = mi.CONFIGS["decode"]
    L = mi.make_layer(cfg, seed=0)
    q, packed = prepared_weights(L)
    layer = m.MoELayer(cfg.n, cfg.K, cfg.d, cfg.ffn, "bf16")
    try:
        y, idx, w = layer.forward_w4a4(dev(L["x"]), dev(L["W_g"]), *packed)
        layer.sync_status()
        torch.cuda.synchronize()
        y, idx, w = host(y), host(idx), host(w)
    finally:
        layer.close()
    o_idx, o_gate, o_logits = oracle.router(L["x"], L["W_g"], cfg.K)
    compare_routing(idx, w, o_idx, o_gate, o_logits, L["x"], L["W_g"], cfg.K)
    pick = stratified_sample(o_idx, cfg.n, 12)
    pick = pick[(idx[pick] == o_idx[pick]).all(axis=1)]
    y_ref = oracle.forward_w4a4(L["x"][pick], o_idx[pick], o_gate[pick], *q)
    assert rel_l2(y_as_f64(y)[pick], y_ref) <= TOL_Y["bf16"]


@pytest.mark.parametrize("name", ["prefill", "many_expert"])
def test_w4a4_full_size(name):
    """The prefill (Mixtral layer shapes, 4,096 tokens) and many-expert
    (128 experts) workloads with 4-bit weights and activations: routing on
    every token; y on a token sample with a row in every (expert, 128-row
    M-block), the ragged end of every segment included, against the oracle's
    4-bit layer, in aggregate and per token."""
    import sparse_mixture_experts_24_b200 as m
    torch = require_cuda()
    cfg = mi.CONFIGS[name]
    L = mi.make_layer(cfg, seed=0)
    q, packed = prepared_weights(L)
    layer = m.MoELayer(cfg.n, cfg.K, cfg.d, cfg.ffn, "bf16")
    try:
        y, idx, w = layer.forward_w4a4(dev(L["x"]), dev(L["W_g"]), *packed)
        layer.sync_status()
        torch.cuda.synchronize()
        y, idx, w = host(y), host(idx), host(w)
    finally:
        layer.close()
    del packed
    torch.cuda.empty_cache()
    o_idx, o_gate, o_logits = oracle.router(L["x"], L["W_g"], cfg.K)
    compare_routing(idx, w, o_idx, o_gate, o_logits, L["x"], L["W_g"], cfg.K)
    pick, nblk = block_covering_sample(o_idx, cfg.n, count=256)
    pick = pick[(idx[pick] == o_idx[pick]).all(axis=1)]
    assert blocks_covered(pick, o_idx, cfg.n) >= nblk - 2
    y_ref = oracle.forward_w4a4(L["x"][pick], o_idx[pick], o_gate[pick], *q)
    yg = y_as_f64(y)[pick]
    assert np.isfinite(y_as_f64(y)).all()
    err = rel_l2(yg, y_ref)
    per_tok = np.linalg.norm(yg - y_ref, axis=1) / np.maximum(np.linalg.norm(y_ref, axis=1), 1e-30)
    print("\n%s W4A4 y rel-L2 on %d tokens (%d M-blocks): %.3e, worst token %.3e"
          % (name, pick.size, nblk, err, per_tok.max()))
    assert err <= TOL_Y["bf16"], err
    assert per_tok.max() <= PER_TOKEN_FACTOR * TOL_Y["bf16"], per_tok.max()


def test_w4a4_many_rows_sampled():
    """20,000 tokens over 16 experts (hundreds of 128-row tiles, scale chunks
    far into the workspace), compared on a token sample."""
    import sparse_mixture_experts_24_b200 as m
    torch = require_cuda()
    name, T, d, F, n, K = "w4a4_many_rows", 20000, 256, 512, 16, 2
    cfg = mi.custom_config(name, T=T, d=d, ffn=F, n=n, K=K, dtype="bf16")
    L = mi.make_layer(cfg, seed=seed_of(name))
    q, packed = prepared_weights(L)
    layer = m.MoELayer(n, K, d, F, "bf16")
    try:
        y, idx, w = layer.forward_w4a4(dev(L["x"]), dev(L["W_g"]), *packed)
        layer.sync_status()
        torch.cuda.synchronize()
        y, idx, w = host(y), host(idx), host(w)
    finally:
        layer.close()
    o_idx, o_gate, o_logits = oracle.router(L["x"], L["W_g"], K)
    compare_routing(idx, w, o_idx, o_gate, o_logits, L["x"], L["W_g"], K)
    pick = stratified_sample(o_idx, n, 300)
    pick = pick[(idx[pick] == o_idx[pick]).all(axis=1)]
    y_ref = oracle.forward_w4a4(L["x"][pick], o_idx[pick], o_gate[pick], *q)
    assert rel_l2(y_as_f64(y)[pick], y_ref) <= TOL_Y["bf16"]
