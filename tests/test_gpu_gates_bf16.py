"""Gates rounded to bf16 (moe_set_gate_rounding) vs the oracle's cast of its
own gates, through the C ABI (needs a B200).

The routing code quoted on the neobadger page (Part 3) computes the softmax in
fp32 and casts the weights to the inputs' dtype.  With the option on, every
gate must be a bf16 value, equal to torch's bf16 cast of the same layer's fp32
gates, within one bf16 step of the oracle's cast of its fp64 gates (equal on
almost every token), and y must match the oracle's layer under those gates."""
import zlib

import numpy as np
import pytest

import moe_inputs as mi
import oracle
from gpu_helpers import TOL_Y, agreeing_tokens, dev, host, rel_l2, require_cuda, y_as_f64

pytestmark = pytest.mark.gpu

CASES = [
    # name, T, d, ffn, n, K   (the last two route on the tensor-core router)
    ("gates16_small", 300, 256, 384, 8, 2),
    ("gates16_k3_n16", 1000, 512, 640, 16, 3),
    ("gates16_tc_router", 600, 1024, 128, 40, 3),
    ("gates16_tc_router_T", 2048, 256, 256, 8, 2),
]


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_gates_rounded_to_bf16(case):
    import sparse_mixture_experts_24_b200 as m
    torch = require_cuda()
    name, T, d, F, n, K = case
    cfg = mi.custom_config(name, T=T, d=d, ffn=F, n=n, K=K, dtype="bf16")
    L = mi.make_layer(cfg, seed=zlib.crc32(name.encode()) % 1000)
    args = [dev(L[k]) for k in ("x", "W_g", "w1", "w3", "w2")]
    layer = m.MoELayer(n, K, d, F, "bf16")
    try:
        _, idx32, w32 = layer.forward(*args)
        layer.set_gate_rounding(True)
        y, idx, w = layer.forward(*args)
        layer.sync_status()
        torch.cuda.synchronize()
        assert torch.equal(idx, idx32)
        assert torch.equal(w, w32.to(torch.bfloat16).float()), "not the bf16 cast of the fp32 gates"
        y, idx, w = host(y), host(idx), host(w)
    finally:
        layer.close()
    assert np.all((w.view(np.uint32) & 0xFFFF) == 0), "a gate is not a bf16 value"
    o_idx, o_gate, _ = oracle.router(L["x"], L["W_g"], K)
    agree = agreeing_tokens(idx, o_idx)
    o16 = oracle.gates_to_bf16(o_gate)
    step = np.ldexp(1.0, np.floor(np.log2(o16[agree])).astype(int) - 7)   # bf16 spacing at each gate
    assert np.all(np.abs(w[agree] - o16[agree]) <= step), "more than one bf16 step from the oracle's cast"
    assert np.mean(w[agree] == o16[agree]) >= 0.98
    y_ref = oracle.forward_with_routing(L["x"], o_idx, o16, L["w1"], L["w3"], L["w2"])
    assert rel_l2(y_as_f64(y)[agree], y_ref[agree]) <= TOL_Y["bf16"]


def test_gate_rounding_argument_check():
    import sparse_mixture_experts_24_b200 as m
    require_cuda()
    layer = m.MoELayer(8, 2, 128, 128, "bf16")
    try:
        with pytest.raises(m.MoEError) as ei:
            m.moe_set_gate_rounding(layer.h, 2)
        assert ei.value.status == m.MOE_ERR_INVALID_ARG
    finally:
        layer.close()
