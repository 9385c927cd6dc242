"""The layer forward under CUDA graph capture (needs a B200).

After moe_reserve (and, for the E4M3 and 4-bit weight-and-activation paths,
a first call that sizes their workspace) a forward call enqueues kernels only -- no allocation, no host
synchronisation -- so it can be captured into a CUDA graph with its
programmatic dependent launches.  Replays must equal the eager call bit for
bit, also after the input buffer is refilled in place."""
import numpy as np
import pytest

import moe_inputs as mi
import oracle
from gpu_helpers import dev, host, require_cuda

pytestmark = pytest.mark.gpu


def _layer_call(m, layer, path, xd, rest, q):
    if path == "bf16":
        return layer.forward(xd, *rest)
    if path == "e4m3":
        return layer.forward_e4m3(xd, rest[0], *q)
    if path == "w4a4":
        return layer.forward_w4a4(xd, rest[0], *q)
    return layer.forward_fp4(xd, rest[0], *q)


@pytest.mark.parametrize("path", ["bf16", "e4m3", "fp4", "w4a4"])
def test_forward_replays_from_a_cuda_graph(path):
    import sparse_mixture_experts_24_b200 as m
    torch = require_cuda()
    # the 4-bit weight-and-activation path needs ffn a multiple of 256
    cfg = mi.custom_config("graph_" + path, T=200, d=256, ffn=512 if path == "w4a4" else 384, n=8, K=2,
                           dtype="bf16")
    L = mi.make_layer(cfg, seed=21)
    L2 = mi.make_layer(cfg, seed=22, only=("x",))
    layer = m.MoELayer(cfg.n, cfg.K, cfg.d, cfg.ffn, "bf16")
    try:
        layer.reserve(cfg.T)
        xd = dev(L["x"])
        rest = [dev(L[k]) for k in ("W_g", "w1", "w3", "w2")]
        q = None
        if path == "e4m3":
            q = [t for w in (L["w1"], L["w3"], L["w2"]) for t in oracle.quantize_weights_e4m3(w)]
            q = [dev(a) for a in q]
        elif path == "fp4":
            q = [tuple(dev(a) for a in oracle.quantize_weights_fp4(L[w])) for w in ("w1", "w3", "w2")]
        elif path == "w4a4":
            q4 = [oracle.quantize_weights_fp4(L[w]) for w in ("w1", "w3", "w2")]
            q = [m.pack_weights_w4a4(*(dev(a) for a in q4[0]), pair=tuple(dev(a) for a in q4[1])),
                 m.pack_weights_w4a4(*(dev(a) for a in q4[2]))]
        y0, i0, w0 = (t.clone() for t in _layer_call(m, layer, path, xd, rest, q))
        torch.cuda.synchronize()
        # outputs of the captured call live in these buffers
        y = torch.empty_like(y0)
        idx = torch.empty_like(i0)
        gw = torch.empty_like(w0)
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        g = torch.cuda.CUDAGraph()
        with torch.cuda.stream(s):
            with torch.cuda.graph(g, stream=s):
                if path == "bf16":
                    layer.forward(xd, *rest, y=y, topk_idx=idx, topk_w=gw)
                elif path == "e4m3":
                    layer.forward_e4m3(xd, rest[0], *q, y=y, topk_idx=idx, topk_w=gw)
                elif path == "w4a4":
                    layer.forward_w4a4(xd, rest[0], *q, y=y, topk_idx=idx, topk_w=gw)
                else:
                    layer.forward_fp4(xd, rest[0], *q, y=y, topk_idx=idx, topk_w=gw)
        torch.cuda.synchronize()
        for _ in range(3):
            g.replay()
            torch.cuda.synchronize()
            assert torch.equal(y, y0) and torch.equal(idx, i0) and torch.equal(gw, w0)
        # refill x in place: the replay computes the new batch
        xd.copy_(dev(L2["x"]))
        g.replay()
        torch.cuda.synchronize()
        y1, i1, w1 = _layer_call(m, layer, path, xd, rest, q)
        torch.cuda.synchronize()
        assert torch.equal(y, y1) and torch.equal(idx, i1) and torch.equal(gw, w1)
        assert not torch.equal(y, y0)
        layer.sync_status()
        del g
    finally:
        layer.close()
