"""Expert-choice routing on the GPU against the oracle, through the C ABI
(needs a B200): each expert's kept tokens bit-exact except where the
probability ranking has a near-tie at the capacity boundary; y within the
tolerance, under the GPU's own selection and against the oracle's."""
import zlib

import numpy as np
import pytest

import moe_inputs as mi
import oracle
from gpu_helpers import TOL_Y, dev, host, rel_l2, require_cuda, y_as_f64

pytestmark = pytest.mark.gpu

CASES = [
    # name, T, d, ffn, n, C, dtype
    ("ec_basic", 300, 128, 256, 8, 75, "bf16"),
    ("ec_n16", 1000, 256, 384, 16, 100, "bf16"),
    ("ec_full_capacity", 64, 128, 256, 8, 64, "bf16"),
    ("ec_many_experts", 600, 128, 128, 64, 20, "bf16"),
    ("ec_f32", 200, 64, 128, 8, 40, "f32"),
    ("ec_capacity_1", 17, 64, 64, 4, 1, "bf16"),
    ("ec_big_T", 5000, 64, 64, 8, 1250, "bf16"),
]


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_expert_choice_matches_oracle(case):
    import sparse_mixture_experts_24_b200 as m
    require_cuda()
    name, T, d, F, n, C, dt = case
    cfg = mi.custom_config(name, T=T, d=d, ffn=F, n=n, K=1, dtype=dt)
    L = mi.make_layer(cfg, seed=zlib.crc32(name.encode()) % 1000)
    layer = m.MoELayer(n, 1, d, F, dt)
    try:
        y, sel, gate = layer.forward_expert_choice(*[dev(L[k]) for k in ("x", "W_g", "w1", "w3", "w2")],
                                                   capacity=C)
        layer.sync_status()
        y, sel, gate = host(y), host(sel), host(gate)
    finally:
        layer.close()
    oy, osel, ogate = oracle.expert_choice(L["x"], L["W_g"], L["w1"], L["w3"], L["w2"], C)
    # probabilities from the oracle's router, for near-tie accounting
    _, _, logits = oracle.router(L["x"], L["W_g"], 1)
    P = np.exp(logits - logits.max(1, keepdims=True))
    P /= P.sum(1, keepdims=True)
    tol = 1e-5 * P.max() + 1e-7
    near = 0
    for e in range(n):
        assert np.all(np.diff(sel[e]) > 0), "tokens not ascending"
        if np.array_equal(sel[e], osel[e]):
            continue
        col = np.sort(P[:, e])[::-1]
        boundary = col[C - 1]
        assert C < T and abs(col[C - 1] - col[C]) < tol, "expert %d selection differs without a near-tie" % e
        sure = set(np.nonzero(P[:, e] > boundary + tol)[0].tolist())
        assert sure <= set(sel[e].tolist())
        near += 1
    # gates are the probabilities of the kept tokens
    assert np.allclose(gate, P[sel, np.arange(n)[:, None]], rtol=1e-5, atol=1e-7)
    # y against the oracle's expert-choice layer on every token that the same
    # experts kept on both sides (all tokens unless a near-tie moved one)
    same = np.ones(T, bool)
    for e in range(n):
        if not np.array_equal(sel[e], osel[e]):
            same[np.setxor1d(sel[e], osel[e])] = False
    assert near > 0 or same.all()
    assert rel_l2(y_as_f64(y)[same], oy[same]) <= TOL_Y[dt]
    kept = np.zeros(T, bool)
    kept[np.unique(sel)] = True
    assert np.all(y_as_f64(y)[~kept] == 0.0)


def test_expert_choice_rejects_bad_capacity():
    import sparse_mixture_experts_24_b200 as m
    torch = require_cuda()
    layer = m.MoELayer(4, 1, 64, 64, "bf16")
    try:
        x = torch.zeros((10, 64), dtype=torch.bfloat16, device="cuda")
        for c in (0, 11):
            with pytest.raises(m.MoEError) as ei:
                layer.forward_expert_choice(x, x, x, x, x, capacity=c)
            assert ei.value.status == m.MOE_ERR_INVALID_ARG
    finally:
        layer.close()
