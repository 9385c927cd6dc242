"""ExpertParallelMoE with its real library side: two processes on the one GPU
a test box has, each a rank with its own handle and CUDA IPC buffers
(moe_ep_buffer_alloc / moe_ep_buffer_open across the processes), a gloo
process group for the counts and the barriers (needs a B200).

No kernel of one rank waits on another rank's kernel: the ranks are ordered
only by the host-side barriers (gloo all-reduce after each rank's stream has
drained), so the two processes' kernels may run in any interleaving.  Each
rank's y must equal, bit for bit, the single-process layer under that rank's
routing, over three consecutive steps, the last on a side stream that is not
torch's current stream."""
import os
import socket

import numpy as np
import pytest

import moe_inputs as mi

pytestmark = pytest.mark.gpu


def free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def rank_main(rank, world, port, Ts, dims):
    import datetime

    import torch
    import torch.distributed as dist

    import sparse_mixture_experts_24_b200 as m
    from sparse_mixture_experts_24_b200.ep import ExpertParallelMoE
    torch.cuda.set_device(0)
    os.environ["MASTER_ADDR"], os.environ["MASTER_PORT"] = "127.0.0.1", str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=120))
    try:
        d, F, n, K = dims
        cfg = mi.custom_config("ep_ipc", T=sum(Ts), d=d, ffn=F, n=n, K=K, dtype="bf16")
        L = mi.make_layer(cfg, seed=5)

        def dev(a):
            t = torch.from_numpy(np.ascontiguousarray(a))
            if a.dtype == np.uint16:
                t = t.view(torch.int16).view(torch.bfloat16)
            return t.cuda()

        lo = sum(Ts[:rank])
        x = dev(L["x"][lo:lo + Ts[rank]])
        Wg = dev(L["W_g"])
        w = [dev(L[k]) for k in ("w1", "w3", "w2")]
        nl = n // world
        wl = [t[rank * nl:(rank + 1) * nl] for t in w]
        layer = ExpertParallelMoE(n, K, d, F, recv_rows=sum(Ts) * K)
        single = m.MoELayer(n, K, d, F, "bf16")
        try:
            side = torch.cuda.Stream()
            for step in range(3):
                if step < 2:
                    y, idx, gate = layer.forward(x, Wg, *wl)
                else:
                    # a stream that is not torch's current one: the step's
                    # barriers must still order this rank's peer stores
                    side.wait_stream(torch.cuda.current_stream())
                    y, idx, gate = layer.forward(x, Wg, *wl, stream=side)
                    torch.cuda.current_stream().wait_stream(side)
                layer._rank.layer.sync_status()
                y_ref = single.forward_with_routing(x, idx, gate, *w)
                single.sync_status()
                assert torch.equal(y.view(torch.int16), y_ref.view(torch.int16)), (rank, step)
        finally:
            single.close()
            layer.close()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("Ts,dims", [((100, 37), (256, 256, 8, 2)), ((64, 1, 200), (128, 192, 6, 3))],
                         ids=["w2", "w3"])
def test_expert_parallel_two_processes_one_gpu(Ts, dims):
    import torch.multiprocessing as mp
    mp.spawn(rank_main, args=(len(Ts), free_port(), Ts, dims), nprocs=len(Ts), join=True)
