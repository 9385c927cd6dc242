"""moe_dispatch_noalloc: the dispatch for callers that cannot allocate device
memory (their memory belongs to a framework allocator or a fixed memory plan,
or they cannot take cudaMalloc's device-wide synchronisation).  It keeps its
scratch in a fixed array inside the library instead of a cudaMalloc'd
workspace.  Checked through the C ABI against the regular moe_dispatch,
bit-exact (integer outputs), on two calls in a row so that the second call
cannot lean on a clean scratch array; and sizes over the array's limit must be
refused.  This file is collected last on purpose."""
import numpy as np
import pytest

from gpu_helpers import dev, host, require_cuda

pytestmark = pytest.mark.gpu


def _regular(T, n, K, idx_d):
    import sparse_mixture_experts_24_b200 as m
    layer = m.MoELayer(n, K, 64, 64, "bf16")
    try:
        out = layer.dispatch(idx_d)
        layer.sync_status()
        return [host(t) for t in out]
    finally:
        layer.close()


def _noalloc(T, n, K, idx_d):
    import sparse_mixture_experts_24_b200 as m
    torch = require_cuda()
    counts = torch.full((n,), -7, dtype=torch.int32, device="cuda")
    offsets = torch.full((n + 1,), -7, dtype=torch.int32, device="cuda")
    row_token = torch.full((T * K,), -7, dtype=torch.int32, device="cuda")
    token_row = torch.full((T, K), -7, dtype=torch.int32, device="cuda")
    m.moe_dispatch_noalloc(T, n, K, idx_d, counts, offsets, row_token, token_row)
    torch.cuda.synchronize()
    return [host(t) for t in (counts, offsets, row_token, token_row)]


def test_noalloc_dispatch_matches_moe_dispatch_twice_in_a_row():
    torch = require_cuda()
    # Both calls have more than 4,096 pairs, so both take the three-kernel
    # path that reads the scratch array.  The first sits exactly at the
    # 65,536-pair limit (256 pair blocks x 256 experts: every word of the
    # per-block counts); the second is smaller, with another n, and runs over
    # what the first left behind.
    cases = [(8192, 256, 8), (2100, 8, 2)]
    for T, n, K in cases:
        rng = np.random.default_rng(T + n)
        idx = np.stack([rng.permutation(n)[:K] for _ in range(T)]).astype(np.int32)
        idx_d = dev(idx)
        want = _regular(T, n, K, idx_d)
        got = _noalloc(T, n, K, idx_d)
        for name, a, b in zip(("counts", "offsets", "row_token", "token_row"), got, want):
            assert np.array_equal(a, b), "%s differs for T=%d n=%d K=%d" % (name, T, n, K)
    torch.cuda.synchronize()


@pytest.mark.parametrize("T,K", [(65537, 1), (32769, 2), (2 ** 61, 4)])
def test_noalloc_dispatch_refuses_sizes_over_its_limit(T, K):
    """One pair over the limit is refused, and so is a T whose product with K
    would overflow 64 bits; nothing is launched."""
    import sparse_mixture_experts_24_b200 as m
    torch = require_cuda()
    rows = min(T, 65537)
    idx = torch.zeros((rows, K), dtype=torch.int32, device="cuda")
    buf = torch.zeros(rows * K + 1, dtype=torch.int32, device="cuda")
    with pytest.raises(m.MoEError) as ei:
        m.moe_dispatch_noalloc(T, 8, K, idx, buf, buf, buf, buf)
    assert ei.value.status == m.MOE_ERR_INVALID_ARG
    assert "65536" in str(ei.value)
    torch.cuda.synchronize()
