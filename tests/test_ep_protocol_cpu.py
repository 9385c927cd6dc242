"""The expert-parallel exchange protocol on 2 and 4 gloo ranks on the CPU.

ExpertParallelMoE (the product's host side: peer-buffer handle exchange,
counts all-gather, the barriers and the order of the steps) runs unchanged;
only its library side is replaced by a stand-in that does what include/moe.h
documents for moe_ep_dispatch / moe_ep_experts / moe_ep_combine, in fp64
numpy over buffers in shared memory (the stand-in for peer memory), with the
expert SwiGLU from the oracle.  Each rank's y must equal the oracle's layer on
that rank's tokens, in two consecutive steps (buffer reuse).  No GPU."""
import os
import socket

import numpy as np
import pytest

import moe_inputs as mi
import oracle


class FakeRank:
    def __init__(self, n, K, d, ffn):
        self.n, self.K = n, K

    def route(self, x, W_g, stream):
        import torch
        if x.shape[0] == 0:
            idx, gate = np.zeros((0, self.K), np.int32), np.zeros((0, self.K))
        else:
            idx, gate, _ = oracle.router(x.numpy(), W_g, self.K)
        self.idx, self.gate = idx, gate
        return torch.from_numpy(np.bincount(idx.ravel(), minlength=self.n).astype(np.int32))

    def dispatch(self, world, rank, x, counts_all, recv_ptrs, recv_rows, stream):
        ca = counts_all.numpy()
        nl = self.n // world
        tot = ca.sum(axis=0)
        seg = np.zeros(self.n, np.int64)               # start of expert e in its owner's buffer
        for e in range(self.n):
            first = (e // nl) * nl
            seg[e] = tot[first:e].sum()
        base = seg + ca[:rank].sum(axis=0)
        xs = x.numpy()
        T = xs.shape[0]
        seen = np.zeros(self.n, np.int64)
        self.row_pos = np.full((T, self.K), -1, np.int64)
        for t in range(T):                              # token order inside an expert
            for k in range(self.K):
                e = self.idx[t, k]
                pos = base[e] + seen[e]
                seen[e] += 1
                assert pos < recv_rows
                recv_ptrs[e // nl][pos] = xs[t]
                self.row_pos[t, k] = pos

    def experts(self, world, rank, counts_all, recv, recv_rows, w1, w3, w2, out, stream):
        ca = counts_all.numpy()
        nl = self.n // world
        tot = ca.sum(axis=0)[rank * nl:(rank + 1) * nl]
        off = np.concatenate(([0], np.cumsum(tot)))
        for i in range(nl):
            rows = recv[off[i]:off[i + 1]]
            if len(rows):
                one = np.zeros((len(rows), 1), np.int32)
                out[off[i]:off[i + 1]] = oracle.forward_with_routing(rows, one, np.ones((len(rows), 1)),
                                                                     w1[i:i + 1], w3[i:i + 1], w2[i:i + 1])

    def combine(self, world, out_ptrs, y, stream):
        nl = self.n // world
        yy = np.zeros(tuple(y.shape))
        for t in range(yy.shape[0]):
            for k in range(self.K):
                e = self.idx[t, k]
                yy[t] += self.gate[t, k] * out_ptrs[e // nl][self.row_pos[t, k]]
        y.copy_(__import__("torch").from_numpy(yy))

    def close(self):
        pass


class FakeOps:
    """Buffers in POSIX shared memory; a handle is the segment's name."""

    def __init__(self, recv_rows, d):
        import torch
        self.device = torch.device("cpu")
        self.shape = (recv_rows, d)
        self.segments = {}

    def new_rank(self, n, K, d, ffn):
        return FakeRank(n, K, d, ffn)

    def _view(self, shm):
        return np.ndarray(self.shape, np.float64, buffer=shm.buf)

    def alloc(self, nbytes):
        from multiprocessing import shared_memory
        shm = shared_memory.SharedMemory(create=True, size=int(np.prod(self.shape)) * 8)
        a = self._view(shm)
        a[:] = np.nan                                   # any row read before it is written shows up
        self.segments[id(a)] = (shm, True)
        return a, shm.name

    def open(self, name):
        from multiprocessing import shared_memory
        shm = shared_memory.SharedMemory(name=name)
        a = self._view(shm)
        self.segments[id(a)] = (shm, False)
        return a

    def close(self, ptr, opened):
        shm, own = self.segments.pop(id(ptr))
        del ptr
        shm.close()
        if own:
            shm.unlink()

    def synchronize(self):
        pass


def free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def rank_main(rank, world, port, Ts, dims):
    import torch
    import torch.distributed as dist
    from sparse_mixture_experts_24_b200.ep import ExpertParallelMoE
    os.environ["MASTER_ADDR"], os.environ["MASTER_PORT"] = "127.0.0.1", str(port)
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        d, F, n, K = dims
        cfg = mi.custom_config("ep_protocol", T=sum(Ts), d=d, ffn=F, n=n, K=K, dtype="bf16")
        L = mi.make_layer(cfg, seed=11)
        lo = sum(Ts[:rank])
        x = mi.as_f32(L["x"][lo:lo + Ts[rank]]).astype(np.float64)
        nl = n // world
        wl = [mi.as_f32(L[k][rank * nl:(rank + 1) * nl]).astype(np.float64) for k in ("w1", "w3", "w2")]
        recv_rows = sum(Ts) * K
        layer = ExpertParallelMoE(n, K, d, F, recv_rows, ops=FakeOps(recv_rows, d))
        try:
            y_ref = (oracle.moe_forward(x, L["W_g"], L["w1"], L["w3"], L["w2"], K)[0] if len(x)
                     else np.zeros((0, d)))
            for step in range(2):
                xt = torch.from_numpy(x.copy())
                y, _, _ = layer.forward(xt, L["W_g"], *wl)
                assert y.shape == y_ref.shape
                if len(x):
                    err = np.abs(y.numpy() - y_ref).max() / np.abs(y_ref).max()
                    assert err < 1e-12, (rank, step, err)
        finally:
            layer.close()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("Ts,dims", [((40, 13), (64, 64, 8, 2)), ((7, 0, 30, 21), (64, 128, 8, 3))],
                         ids=["w2", "w4_empty_rank"])
def test_ep_protocol_matches_oracle(Ts, dims):
    import torch.multiprocessing as mp
    mp.spawn(rank_main, args=(len(Ts), free_port(), Ts, dims), nprocs=len(Ts), join=True)
