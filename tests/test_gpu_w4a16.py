"""4-bit weights decoded into tensor memory, bf16 activations
(moe_pack_weights_w4a16 / moe_forward_w4a16) against the fp64 oracle, through
the C ABI (needs a B200).

The pack is decoded on the host by the rule moe.h documents (rotate, mask,
read the bf16 fields back) and compared bit for bit with the codes and block
scales of the oracle's quantiser; the layer runs on the oracle's codes and is
compared with the oracle's 4-bit layer (oracle.forward_fp4, the bf16 layer of
the dequantised weights) under the oracle's routing, in both token-block
heights; the hidden rows H are compared with numpy on the dequantised weights,
which locates a wrong column or row of a decoded weight tile."""
import zlib

import numpy as np
import pytest

import moe_inputs as mi
import oracle
from gpu_helpers import (PER_TOKEN_FACTOR, TOL_Y, agreeing_tokens, compare_routing, dev, host, read_workspace,
                         rel_l2, require_cuda, y_as_f64)

pytestmark = pytest.mark.gpu

P_MASK = 0x81C081C0


def seed_of(name: str) -> int:
    return zlib.crc32(name.encode()) % 1000


def rotr(w, s):
    w = w.astype(np.uint64)
    return (((w >> np.uint64(s)) | (w << np.uint64(32 - s))) & np.uint64(0xFFFFFFFF)).astype(np.uint32)


def bf16_fields_to_code(v, half):
    """The E2M1 code whose fields sit in bf16 half `half` of v (mantissa bit 6,
    exponent bits 7-8, sign bit 15 of the half)."""
    h = (v >> np.uint32(16 * half)) & np.uint32(0xFFFF)
    return ((h >> 6) & 1) | (((h >> 7) & 1) << 1) | (((h >> 8) & 1) << 2) | (((h >> 15) & 1) << 3)


def unpack_w4a16(packed, rows, cols, pair):
    """Host decode of a packed matrix -> (codes [n][rows][cols] per source
    matrix, block scales [n][rows/16][cols] per source matrix)."""
    n, tiles, steps, _ = packed.shape
    out_cols = 128
    codes = np.zeros((2 if pair else 1, n, rows, cols), np.uint8)
    scales = np.zeros((2 if pair else 1, n, rows // 16, cols), np.uint8)
    blk = packed.reshape(n, tiles, steps, 4608)
    words = blk[..., :4096].reshape(n, tiles, steps, 2, 128, 16).view(np.uint32)  # [.., half, col, 4]
    sc = blk[..., 4096:].reshape(n, tiles, steps, 128, 4)
    for p in range(out_cols):
        if pair:
            src, col = (0, None) if p < 64 else (1, None)
            cidx = np.arange(tiles) * 64 + (p & 63)
        else:
            src = 0
            cidx = np.arange(tiles) * 128 + p
        for half in range(2):
            for wi in range(4):
                w = words[:, :, :, half, p, wi]                       # [n][tiles][steps]
                pairs = [w & np.uint32(P_MASK), rotr(w, 4) & np.uint32(P_MASK), rotr(w, 10) & np.uint32(P_MASK),
                         (rotr(w, 6) & np.uint32(0x81808180)) | (rotr(w, 14) & np.uint32(0x00400040))]
                for i, v in enumerate(pairs):
                    r0 = half * 32 + wi * 8 + 2 * i
                    for hi in range(2):
                        c = bf16_fields_to_code(v, hi)                # [n][tiles][steps]
                        rows_k = np.arange(steps) * 64 + r0 + hi
                        codes[src][:, rows_k[None, :], cidx[:, None]] = np.transpose(c, (0, 1, 2))
        for g in range(4):
            rows_g = np.arange(steps) * 4 + g
            scales[src][:, rows_g[None, :], cidx[:, None]] = sc[:, :, :, p, g]
    return codes, scales


def nibbles(codes_packed):
    """[n][rows][cols/2] bytes (column 2j low nibble) -> [n][rows][cols] codes."""
    lo = codes_packed & 0xF
    hi = codes_packed >> 4
    out = np.empty(codes_packed.shape[:-1] + (2 * codes_packed.shape[-1],), np.uint8)
    out[..., 0::2] = lo
    out[..., 1::2] = hi
    return out


@pytest.mark.parametrize("rows,cols,pair", [(64, 128, False), (192, 256, False), (128, 64, True), (256, 192, True)])
def test_pack_layout_decodes_to_the_quantiser_codes(rows, cols, pair):
    import sparse_mixture_experts_24_b200 as m
    torch = require_cuda()
    rng = np.random.default_rng(rows + cols)
    n = 3
    w1 = (rng.standard_normal((n, rows, cols)) * rng.choice([1e-3, 1.0, 40.0], size=(n, 1, cols))).astype(np.float32)
    q1 = oracle.quantize_weights_fp4(w1)
    trip = tuple(dev(a) for a in q1)
    if pair:
        w3 = rng.standard_normal((n, rows, cols)).astype(np.float32)
        q3 = oracle.quantize_weights_fp4(w3)
        packed = m.pack_weights_w4a16(*trip, pair=tuple(dev(a) for a in q3))[0]
        srcs = [q1, q3]
    else:
        packed = m.pack_weights_w4a16(*trip)[0]
        srcs = [q1]
    torch.cuda.synchronize()
    codes, scales = unpack_w4a16(host(packed), rows, cols, pair)
    for s, q in enumerate(srcs):
        assert np.array_equal(codes[s], nibbles(q[0])), "codes of source %d differ" % s
        assert np.array_equal(scales[s], q[1]), "block scales of source %d differ" % s


def pack_gpu(q):
    import sparse_mixture_experts_24_b200 as m
    qd = [tuple(dev(a) for a in t) for t in q]
    w13 = m.pack_weights_w4a16(*qd[0], pair=qd[1])
    w2 = m.pack_weights_w4a16(*qd[2])
    return w13, w2


def run_w4a16(cfg, L, q, factor=0.0):
    import sparse_mixture_experts_24_b200 as m
    torch = require_cuda()
    w13, w2 = pack_gpu(q)
    layer = m.MoELayer(cfg.n, cfg.K, cfg.d, cfg.ffn, "bf16")
    try:
        if factor:
            layer.set_capacity_factor(factor)
        y, idx, w = layer.forward_w4a16(dev(L["x"]), dev(L["W_g"]), w13, w2)
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
    # name, T, d, ffn, n, K, token rows forced (None: the library's choice)
    ("w16_ragged", 300, 256, 320, 8, 2, None),
    ("w16_ragged_rows32", 300, 256, 320, 8, 2, 32),
    ("w16_tails", 77, 384, 192, 4, 1, None),
    ("w16_T1", 1, 256, 256, 8, 2, None),
    ("w16_decode_like", 32, 512, 448, 8, 2, None),
    ("w16_decode_like_rows128", 32, 512, 448, 8, 2, 128),
    ("w16_n64_k4", 700, 128, 64, 64, 4, None),
    ("w16_big_segments", 1500, 384, 512, 4, 2, None),
    ("w16_big_segments_rows32", 1500, 384, 512, 4, 2, 32),
]


@pytest.mark.parametrize("case", FWD_CASES, ids=[c[0] for c in FWD_CASES])
def test_w4a16_layer_matches_oracle(case, monkeypatch):
    name, T, d, F, n, K, rows = case
    if rows:
        monkeypatch.setenv("MOE_W4A16_ROWS", str(rows))
    cfg = mi.custom_config(name, T=T, d=d, ffn=F, n=n, K=K, dtype="bf16")
    L = mi.make_layer(cfg, seed=seed_of(name))
    q = [oracle.quantize_weights_fp4(L[w]) for w in ("w1", "w3", "w2")]
    deq = [oracle.dequantize_fp4(*t) for t in q]
    y, idx, w, H, offsets, row_token, _ = run_w4a16(cfg, L, q)
    o_idx, o_gate, o_logits = oracle.router(L["x"], L["W_g"], K)
    compare_routing(idx, w, o_idx, o_gate, o_logits, L["x"], L["W_g"], K)
    R = int(offsets[-1])
    seg = np.searchsorted(offsets, np.arange(R), side="right") - 1
    xr = mi.as_f32(L["x"]).astype(np.float64)[row_token[:R]]
    Hg = mi.as_f32(H[:R]).astype(np.float64)
    for e in np.unique(seg):
        sel = seg == e
        ref = silu(xr[sel] @ deq[0][e]) * (xr[sel] @ deq[1][e])
        err = np.linalg.norm(Hg[sel] - ref, axis=1) / np.maximum(np.linalg.norm(ref, axis=1), 1e-30)
        assert err.max() < 2e-2, (e, err.max(), int(np.argmax(err)))
    agree = agreeing_tokens(idx, o_idx)
    y_ref = oracle.forward_fp4(L["x"], o_idx, o_gate, *q)
    yg = y_as_f64(y)
    assert rel_l2(yg[agree], y_ref[agree]) <= TOL_Y["bf16"]
    per_tok = np.linalg.norm(yg - y_ref, axis=1)[agree] / np.maximum(np.linalg.norm(y_ref, axis=1)[agree], 1e-30)
    assert per_tok.max() <= PER_TOKEN_FACTOR * TOL_Y["bf16"], per_tok.max()


def test_w4a16_capacity_drops_like_bf16():
    name, T, d, F, n, K = "w16_capacity", 600, 128, 192, 8, 2
    cfg = mi.custom_config(name, T=T, d=d, ffn=F, n=n, K=K, dtype="bf16", skew=True)
    L = mi.make_layer(cfg, seed=seed_of(name))
    q = [oracle.quantize_weights_fp4(L[w]) for w in ("w1", "w3", "w2")]
    C = int(np.ceil(1.0 * T * K / n))
    y, idx, w, _, offsets, _, token_row = run_w4a16(cfg, L, q, factor=1.0)
    o_idx, o_gate, _ = oracle.router(L["x"], L["W_g"], K)
    assert (idx == o_idx).all(), "skewed case should route without near-ties"
    _, o_off, _, o_tr = oracle.dispatch_capacity(o_idx, n, C)
    assert np.array_equal(offsets, o_off) and np.array_equal(token_row, o_tr)
    dropped = o_tr < 0
    assert dropped.any()
    y_ref = oracle.forward_fp4(L["x"], o_idx, np.where(dropped, 0.0, o_gate), *q)
    assert rel_l2(y_as_f64(y), y_ref) <= TOL_Y["bf16"]


def test_w4a16_rejects_bad_handles_and_shapes():
    import sparse_mixture_experts_24_b200 as m
    torch = require_cuda()
    layer = m.MoELayer(8, 2, 128, 128, "f32")
    try:
        x = torch.zeros((4, 128), dtype=torch.float32, device="cuda")
        with pytest.raises(m.MoEError) as ei:
            layer.forward_w4a16(x, x, (x, x, x), (x, x))
        assert ei.value.status == m.MOE_ERR_UNSUPPORTED
    finally:
        layer.close()
    layer = m.MoELayer(8, 2, 192, 128, "bf16")          # d not a multiple of 128
    try:
        x = torch.zeros((4, 192), dtype=torch.bfloat16, device="cuda")
        with pytest.raises(m.MoEError) as ei:
            layer.forward_w4a16(x, x, (x, x, x), (x, x))
        assert ei.value.status == m.MOE_ERR_UNSUPPORTED
    finally:
        layer.close()
    buf = torch.zeros(1 << 16, dtype=torch.uint8, device="cuda")
    with pytest.raises(m.MoEError) as ei:                # cols not a multiple of 128 (single matrix)
        m.moe_pack_weights_w4a16(1, 64, 96, buf, buf, None, None, buf)
    assert ei.value.status == m.MOE_ERR_INVALID_ARG
    with pytest.raises(m.MoEError) as ei:                # rows not a multiple of 64
        m.moe_pack_weights_w4a16(1, 48, 128, buf, buf, None, None, buf)
    assert ei.value.status == m.MOE_ERR_INVALID_ARG
    with pytest.raises(m.MoEError) as ei:                # half a pair
        m.moe_pack_weights_w4a16(1, 64, 128, buf, buf, buf, None, buf)
    assert ei.value.status == m.MOE_ERR_INVALID_ARG
    torch.cuda.synchronize()


@pytest.mark.parametrize("name", ["decode", "many_expert"])
def test_w4a16_full_size(name):
    """Full-size workloads with the 4-bit weights packed for tensor memory:
    routing on every token, y on every token (decode) or a token sample that
    reaches every (expert, M-block) (many_expert) against the oracle's 4-bit
    layer."""
    import sparse_mixture_experts_24_b200 as m
    from gpu_helpers import block_covering_sample
    torch = require_cuda()
    cfg = mi.CONFIGS[name]
    L = mi.make_layer(cfg, seed=0)
    q = [oracle.quantize_weights_fp4(L[w]) for w in ("w1", "w3", "w2")]
    w13, w2 = pack_gpu(q)
    layer = m.MoELayer(cfg.n, cfg.K, cfg.d, cfg.ffn, "bf16")
    try:
        y, idx, w = layer.forward_w4a16(dev(L["x"]), dev(L["W_g"]), w13, w2)
        layer.sync_status()
        y, idx, w = host(y), host(idx), host(w)
    finally:
        layer.close()
    del w13, w2
    torch.cuda.empty_cache()
    o_idx, o_gate, o_logits = oracle.router(L["x"], L["W_g"], cfg.K)
    compare_routing(idx, w, o_idx, o_gate, o_logits, L["x"], L["W_g"], cfg.K)
    if cfg.T <= 64:
        pick = np.arange(cfg.T)
    else:
        pick, _ = block_covering_sample(o_idx, cfg.n, count=256, block=32)
    pick = pick[(idx[pick] == o_idx[pick]).all(axis=1)]
    y_ref = oracle.forward_fp4(L["x"][pick], o_idx[pick], o_gate[pick], *q)
    yg = y_as_f64(y)[pick]
    assert rel_l2(yg, y_ref) <= TOL_Y["bf16"]
    per_tok = np.linalg.norm(yg - y_ref, axis=1) / np.maximum(np.linalg.norm(y_ref, axis=1), 1e-30)
    assert per_tok.max() <= PER_TOKEN_FACTOR * TOL_Y["bf16"]
