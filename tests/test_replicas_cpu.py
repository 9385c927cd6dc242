"""The N > 1 host logic of bench.py on CPU: two gloo ranks (replicas only, no
collective on the data path; the timings are max-reduced over ranks)."""
import os
import socket

import numpy as np
import torch.distributed as dist
import torch.multiprocessing as mp

import moe_inputs as mi


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, out):
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        local_ms = [3.0, 5.0][rank]
        ms = bench.max_over_ranks(local_ms, dist, "cpu")
        cfg = mi.custom_config(T=16, d=64, ffn=64, n=4, K=2, dtype="bf16")
        x = mi.make_layer(cfg, seed=bench.replica_seed(rank), only=("x",))["x"]
        out[rank] = (ms, bench.tokens_per_s(cfg.T, world, ms), int(x.astype(np.int64).sum()))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_replicas_max_reduce_and_distinct_batches():
    world = 2
    port = _free_port()
    with mp.get_context("spawn").Manager() as mgr:
        out = mgr.dict()
        mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    assert res[0][0] == res[1][0] == 5.0          # slowest rank sets the time
    assert res[0][1] == res[1][1] == 16 * 2 / 5e-3  # whole-job tokens/s
    assert res[0][2] != res[1][2]                   # each replica has its own batch
