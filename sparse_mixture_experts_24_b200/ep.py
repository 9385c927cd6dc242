"""Expert parallelism: the n experts split over W ranks, each rank routing its
own tokens (rank q holds experts [q n/W, (q+1) n/W)).

One layer step on rank r, every arithmetic step in the library's kernels:

    moe_route, moe_dispatch          routing and this rank's counts [n]
    counts_all [W][n]                every rank's counts (all-gather)
    moe_ep_dispatch                  x rows stored into the owners' receive buffers
    barrier
    moe_ep_experts                   grouped SwiGLU of the local experts
    barrier
    moe_ep_combine                   expert outputs loaded from the owners' buffers

ExpertParallelMoE runs one rank per process (torch.distributed for the counts
and the barriers -- NCCL with a GPU per rank; peer buffers mapped by CUDA IPC).
emulate_ranks runs W ranks in one process on one GPU, phase by phase, with
every rank's buffers in that GPU's memory -- the same kernels and layouts.
"""
from . import (MoELayer, moe_dispatch, moe_ep_buffer_alloc, moe_ep_buffer_close, moe_ep_buffer_open,
               moe_ep_combine, moe_ep_dispatch, moe_ep_experts)


class _Rank:
    """A rank's handle and per-step tensors."""

    def __init__(self, n, K, d, ffn):
        self.layer = MoELayer(n, K, d, ffn, "bf16")
        self.counts = self.idx = self.gate = self.row_pos = None

    def route(self, x, W_g, stream):
        import torch
        T = x.shape[0]
        self.counts = torch.zeros(self.layer.n, dtype=torch.int32, device=x.device)
        if T == 0:
            self.idx = torch.empty((0, self.layer.K), dtype=torch.int32, device=x.device)
            self.gate = torch.empty((0, self.layer.K), dtype=torch.float32, device=x.device)
            return self.counts
        self.idx, self.gate = self.layer.route(x, W_g, stream=stream)
        moe_dispatch(self.layer.h, T, self.idx, counts=self.counts, stream=stream)
        return self.counts

    def dispatch(self, world, rank, x, counts_all, recv_ptrs, recv_rows, stream):
        import torch
        T = x.shape[0]
        self.row_pos = torch.empty((T, self.layer.K), dtype=torch.int32, device=x.device)
        moe_ep_dispatch(self.layer.h, world, rank, T, x, self.idx, counts_all, recv_ptrs, recv_rows,
                        self.row_pos, stream)

    def experts(self, world, rank, counts_all, recv_ptr, recv_rows, w1, w3, w2, out_ptr, stream):
        moe_ep_experts(self.layer.h, world, rank, counts_all, recv_ptr, recv_rows, w1, w3, w2, out_ptr, stream)

    def combine(self, world, out_ptrs, y, stream):
        moe_ep_combine(self.layer.h, world, y.shape[0], self.idx, self.gate, self.row_pos, out_ptrs, y, stream)

    def close(self):
        self.layer.close()


class EmulatedExpertParallel:
    """W ranks on the current GPU with persistent handles and buffers: every
    phase runs for all ranks before the next phase starts (the order the
    barriers impose across GPUs), each rank's buffers in this GPU's memory.
    recv_rows: rows of each receive buffer (W * T_max * K always suffices)."""

    def __init__(self, n, K, d, ffn, world, recv_rows):
        import torch
        self.n, self.K, self.d, self.world, self.recv_rows = n, K, d, world, recv_rows
        self.ranks = [_Rank(n, K, d, ffn) for _ in range(world)]
        dev = torch.device("cuda", torch.cuda.current_device())
        self.recv = [torch.empty((recv_rows, d), dtype=torch.bfloat16, device=dev) for _ in range(world)]
        self.out = [torch.empty((recv_rows, d), dtype=torch.bfloat16, device=dev) for _ in range(world)]

    def forward(self, xs, W_g, weights, ys=None, stream=None, mark=None):
        """xs: W bf16 token blocks [T_r][d]; weights: W (w1, w3, w2) triples of
        each rank's local experts.  -> (ys, idxs, gates), one entry per rank.
        mark(i), if given, is called after phase i (0 routing and counts,
        1 dispatch, 2 experts, 3 combine) -- e.g. to record CUDA events."""
        import torch
        W = self.world
        mark = mark or (lambda i: None)
        counts_all = torch.stack([rk.route(x, W_g, stream) for rk, x in zip(self.ranks, xs)])
        mark(0)
        for r, (rk, x) in enumerate(zip(self.ranks, xs)):
            rk.dispatch(W, r, x, counts_all, self.recv, self.recv_rows, stream)
        mark(1)
        for q, rk in enumerate(self.ranks):
            rk.experts(W, q, counts_all, self.recv[q], self.recv_rows, *weights[q], self.out[q], stream)
        mark(2)
        if ys is None:
            ys = [torch.empty_like(x) for x in xs]
        for rk, y in zip(self.ranks, ys):
            rk.combine(W, self.out, y, stream)
        mark(3)
        return ys, [rk.idx for rk in self.ranks], [rk.gate for rk in self.ranks]

    def launch_count(self):
        from . import moe_launch_count
        return sum(moe_launch_count(rk.layer.h) for rk in self.ranks)

    def sync_status(self, stream=None):
        for rk in self.ranks:
            rk.layer.sync_status(stream)

    def close(self):
        for rk in self.ranks:
            rk.close()
        self.ranks = []


def emulate_ranks(xs, W_g, weights, n, K, recv_rows=None, stream=None):
    """One expert-parallel step of W = len(xs) ranks on the current GPU (see
    EmulatedExpertParallel).  -> (ys, idxs, gates)."""
    world = len(xs)
    d = xs[0].shape[1]
    ffn = weights[0][0].shape[2]
    if recv_rows is None:
        recv_rows = max(1, sum(int(x.shape[0]) for x in xs) * K)
    ep = EmulatedExpertParallel(n, K, d, ffn, world, recv_rows)
    try:
        out = ep.forward(xs, W_g, weights, stream=stream)
        ep.sync_status(stream)
        return out
    finally:
        ep.close()


def _current_stream(stream):
    """Context that makes `stream` torch's current stream (no-op for None)."""
    import contextlib
    if stream is None:
        return contextlib.nullcontext()
    import torch
    if isinstance(stream, int):
        stream = torch.cuda.ExternalStream(stream)
    return torch.cuda.stream(stream)


class _CudaOps:
    """The library's side of ExpertParallelMoE: handles and IPC buffers."""

    def __init__(self):
        import torch
        self.device = torch.device("cuda", torch.cuda.current_device())

    def new_rank(self, n, K, d, ffn):
        return _Rank(n, K, d, ffn)

    def alloc(self, nbytes):
        return moe_ep_buffer_alloc(nbytes)

    def open(self, handle):
        return moe_ep_buffer_open(handle)

    def close(self, ptr, opened):
        moe_ep_buffer_close(ptr, opened)

    def synchronize(self):
        import torch
        torch.cuda.synchronize(self.device)


class ExpertParallelMoE:
    """This process's rank of an expert-parallel layer (one GPU per process,
    torch.distributed initialised with the NCCL backend).  recv_rows: rows of
    every receive buffer, at least the most rows any rank's experts receive
    in one step (W * T_max * K always suffices).  `ops` replaces the library
    side (handles, buffers) for tests of the exchange protocol."""

    def __init__(self, n, K, d, ffn, recv_rows, group=None, ops=None):
        import torch
        import torch.distributed as dist
        self.ops = ops if ops is not None else _CudaOps()
        self.dist, self.group = dist, group
        self.world = dist.get_world_size(group)
        self.rank = dist.get_rank(group)
        if n % self.world:
            raise ValueError("n = %d experts do not split over %d ranks" % (n, self.world))
        self.n, self.K, self.d, self.recv_rows = n, K, d, recv_rows
        self._rank = self.ops.new_rank(n, K, d, ffn)
        nbytes = recv_rows * d * 2
        self._own, handles = [], []
        for _ in range(2):  # receive buffer, output buffer
            p, hd = self.ops.alloc(nbytes)
            self._own.append(p)
            handles.append(hd)
        table = [None] * self.world
        dist.all_gather_object(table, handles, group=group)
        self._opened = []
        self.recv_ptrs, self.out_ptrs = [], []
        for q in range(self.world):
            if q == self.rank:
                ptrs = self._own
            else:
                ptrs = [self.ops.open(hd) for hd in table[q]]
                self._opened += ptrs
            self.recv_ptrs.append(ptrs[0])
            self.out_ptrs.append(ptrs[1])
        self._one = torch.ones(1, dtype=torch.int32, device=self.ops.device)

    def _barrier(self):
        # an all-reduce on the current stream: every rank's earlier kernels
        # (and their peer stores) are done before any rank goes past it
        self.dist.all_reduce(self._one, group=self.group)

    def forward(self, x, W_g, w1, w3, w2, y=None, stream=None):
        """x [T][d] bf16 of this rank; w1, w3 [n/W][d][ffn], w2 [n/W][ffn][d]:
        this rank's experts.  -> (y, topk_idx, topk_w).

        stream (a torch.cuda.Stream or a raw cudaStream_t as an int): the
        whole step, its all-gather and barriers included, is ordered on it.
        The barriers are collectives on torch's current stream, so the step
        makes `stream` current while it runs; otherwise a barrier could pass
        before this rank's peer stores on `stream` are done."""
        with _current_stream(stream):
            return self._forward(x, W_g, w1, w3, w2, y, stream)

    def _forward(self, x, W_g, w1, w3, w2, y, stream):
        import torch
        rk = self._rank
        counts = rk.route(x, W_g, stream)
        rows = [torch.empty_like(counts) for _ in range(self.world)]
        self.dist.all_gather(rows, counts, group=self.group)
        counts_all = torch.stack(rows)
        rk.dispatch(self.world, self.rank, x, counts_all, self.recv_ptrs, self.recv_rows, stream)
        self._barrier()
        rk.experts(self.world, self.rank, counts_all, self.recv_ptrs[self.rank], self.recv_rows, w1, w3, w2,
                   self.out_ptrs[self.rank], stream)
        self._barrier()
        if y is None:
            y = torch.empty_like(x)
        rk.combine(self.world, self.out_ptrs, y, stream)
        return y, rk.idx, rk.gate

    def close(self):
        # no rank may still read this rank's buffers, and no rank may still
        # hold a mapping of them when they are freed
        self._barrier()
        self.ops.synchronize()
        for p in self._opened:
            self.ops.close(p, True)
        self._barrier()
        self.ops.synchronize()
        for p in self._own:
            self.ops.close(p, False)
        self._opened, self._own = [], []
        self._rank.close()
