"""Expert parallelism on one GPU (ranks emulated phase by phase, every rank's
buffers in this GPU's memory), through the C ABI (needs a B200).

Each rank's y must equal, bit for bit, the single-GPU layer run with that
rank's routing (moe_forward_with_routing: same kernels, same order), and must
match the fp64 oracle under the oracle's routing on the tokens whose routing
agrees.  Also: the plan's rejections (counts that disagree with the routing,
a receive buffer too small) and the argument checks."""
import zlib

import numpy as np
import pytest

import moe_inputs as mi
import oracle
from gpu_helpers import TOL_Y, agreeing_tokens, compare_routing, dev, host, rel_l2, require_cuda, y_as_f64

pytestmark = pytest.mark.gpu


def seed_of(name: str) -> int:
    return zlib.crc32(name.encode()) % 1000


CASES = [
    # name, tokens per rank, d, ffn, n, K
    ("ep_w2_ragged", (300, 77), 256, 384, 8, 2),
    ("ep_w4_empty_rank", (1, 0, 250, 513), 128, 192, 16, 3),
    ("ep_w8_one_expert_each", (64, 64, 1, 200, 17, 5, 90, 33), 128, 128, 8, 2),
    ("ep_w1", (400,), 256, 256, 8, 2),
    ("ep_w2_k1", (129, 255), 192, 320, 4, 1),
    ("ep_w4_many_experts", (700, 300, 512, 1000), 128, 256, 64, 4),
    ("ep_w16_most_ranks", (40, 0, 17, 90, 33, 1, 64, 8, 120, 5, 77, 2, 50, 30, 11, 60), 128, 128, 32, 2),
]


def split_weights(L, world, n):
    nl = n // world
    w = [dev(L[k]) for k in ("w1", "w3", "w2")]
    return w, [tuple(t[q * nl:(q + 1) * nl] for t in w) for q in range(world)]


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_ep_equals_single_gpu_and_oracle(case):
    import sparse_mixture_experts_24_b200 as m
    from sparse_mixture_experts_24_b200.ep import emulate_ranks
    torch = require_cuda()
    name, Ts, d, F, n, K = case
    world = len(Ts)
    cfg = mi.custom_config(name, T=sum(Ts), d=d, ffn=F, n=n, K=K, dtype="bf16")
    L = mi.make_layer(cfg, seed=seed_of(name))
    x_all, Wg = dev(L["x"]), dev(L["W_g"])
    bounds = np.cumsum((0,) + Ts)
    xs = [x_all[bounds[r]:bounds[r + 1]].contiguous() for r in range(world)]
    w_full, w_local = split_weights(L, world, n)
    ys, idxs, gates = emulate_ranks(xs, Wg, w_local, n, K)
    torch.cuda.synchronize()
    single = m.MoELayer(n, K, d, F, "bf16")
    try:
        for r in range(world):
            T = Ts[r]
            if T == 0:
                assert ys[r].shape[0] == 0
                continue
            y_ref = single.forward_with_routing(xs[r], idxs[r], gates[r], *w_full)
            single.sync_status()
            assert torch.equal(ys[r].view(torch.int16), y_ref.view(torch.int16)), "rank %d differs from one GPU" % r
            xr = L["x"][bounds[r]:bounds[r + 1]]
            idx, w = host(idxs[r]), host(gates[r])
            o_idx, o_gate, o_logits = oracle.router(xr, L["W_g"], K)
            compare_routing(idx, w, o_idx, o_gate, o_logits, xr, L["W_g"], K)
            agree = agreeing_tokens(idx, o_idx)
            y_or = oracle.forward_with_routing(xr, o_idx, o_gate, L["w1"], L["w3"], L["w2"])
            err = rel_l2(y_as_f64(host(ys[r]))[agree], y_or[agree])
            assert err <= TOL_Y["bf16"], (r, err)
    finally:
        single.close()


def ep_setup(name, Ts, d, F, n, K):
    cfg = mi.custom_config(name, T=sum(Ts), d=d, ffn=F, n=n, K=K, dtype="bf16")
    L = mi.make_layer(cfg, seed=seed_of(name))
    x_all, Wg = dev(L["x"]), dev(L["W_g"])
    bounds = np.cumsum((0,) + Ts)
    xs = [x_all[bounds[r]:bounds[r + 1]].contiguous() for r in range(len(Ts))]
    return xs, Wg, split_weights(L, len(Ts), n)[1]


def test_ep_plan_rejects_bad_counts_and_small_buffers():
    """counts_all whose own row disagrees with the routing, and a receive
    buffer smaller than what an owner receives: moe_sync_status reports
    MOE_ERR_INVALID_ARG and nothing is stored (row_pos all -1)."""
    import sparse_mixture_experts_24_b200 as m
    from sparse_mixture_experts_24_b200.ep import _Rank
    torch = require_cuda()
    n, K, d, F = 8, 2, 128, 128
    xs, Wg, w_local = ep_setup("ep_reject", (200, 100), d, F, n, K)
    ranks = [_Rank(n, K, d, F) for _ in range(2)]
    try:
        counts_all = torch.stack([rk.route(x, Wg, None) for rk, x in zip(ranks, xs)])
        need = int(host(counts_all).sum())
        for bad_counts, recv_rows in ((True, need), (False, 10)):
            ca = counts_all.clone()
            if bad_counts:
                ca[0, 0] += 1
            recv = [torch.full((recv_rows, d), 7.0, dtype=torch.bfloat16, device="cuda") for _ in range(2)]
            rk = ranks[0]
            rk.dispatch(2, 0, xs[0], ca, recv, recv_rows, None)
            with pytest.raises(m.MoEError) as ei:
                rk.layer.sync_status()
            assert ei.value.status == m.MOE_ERR_INVALID_ARG
            assert (host(rk.row_pos) == -1).all()
            assert all(bool((r == 7.0).all()) for r in recv), "a rejected plan stored rows"
        # the experts step under a rejected plan computes nothing either
        out = torch.full((10, d), 3.0, dtype=torch.bfloat16, device="cuda")
        recv = torch.zeros((10, d), dtype=torch.bfloat16, device="cuda")
        ranks[1].experts(2, 1, counts_all, recv, 10, *w_local[1], out, None)
        with pytest.raises(m.MoEError):
            ranks[1].layer.sync_status()
        assert bool((out == 3.0).all())
    finally:
        for rk in ranks:
            rk.close()


def test_ep_argument_checks():
    import sparse_mixture_experts_24_b200 as m
    torch = require_cuda()
    layer = m.MoELayer(8, 2, 128, 128, "bf16")
    z = torch.zeros((64, 128), dtype=torch.bfloat16, device="cuda")
    i = torch.zeros((32, 2), dtype=torch.int32, device="cuda")
    try:
        for world, rank in ((3, 0), (17, 0), (2, 2), (0, 0)):
            with pytest.raises(m.MoEError) as ei:
                m.moe_ep_dispatch(layer.h, world, rank, 32, z, i, i, [z] * max(world, 1), 64, i)
            assert ei.value.status == m.MOE_ERR_INVALID_ARG
        with pytest.raises(m.MoEError) as ei:                       # a null peer pointer
            m.moe_ep_combine(layer.h, 2, 32, i, i, i, [z, None], z)
        assert ei.value.status == m.MOE_ERR_INVALID_ARG
        layer.set_capacity_factor(1.0)                               # EP is dropless
        with pytest.raises(m.MoEError) as ei:
            m.moe_ep_experts(layer.h, 2, 0, i, z, 64, z, z, z, z)
        assert ei.value.status == m.MOE_ERR_UNSUPPORTED
    finally:
        layer.close()
    f32 = m.MoELayer(8, 2, 128, 128, "f32")
    try:
        with pytest.raises(m.MoEError) as ei:
            m.moe_ep_combine(f32.h, 2, 32, i, i, i, [z, z], z)
        assert ei.value.status == m.MOE_ERR_UNSUPPORTED
    finally:
        f32.close()
