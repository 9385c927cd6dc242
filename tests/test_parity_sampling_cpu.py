"""The full-size GPU parity tests' token sample (CPU only): it must put a row
in every (expert, 128-row M-block) of the grouped GEMMs, include the last
row of every expert's segment, and reach the requested size."""
import numpy as np
import pytest

import oracle
from gpu_helpers import GEMM_ROW_BLOCK, block_covering_sample, blocks_covered


@pytest.mark.parametrize("T,n,K,skew", [(8192, 128, 2, False), (4096, 8, 2, False), (16384, 8, 2, True),
                                        (700, 256, 8, False), (300, 3, 1, False)])
def test_sample_reaches_every_m_block(T, n, K, skew):
    rng = np.random.default_rng(T + n)
    idx = np.stack([rng.permutation(n)[:K] for _ in range(T)]).astype(np.int32)
    if skew:
        idx[:, 0] = 0
        idx[:, 1] = 1 + rng.integers(0, n - 1, T)
    sample, nblk = block_covering_sample(idx, n, count=512)
    counts, offsets, row_token, token_row = oracle.dispatch(idx, n)
    assert nblk == int(sum((c + GEMM_ROW_BLOCK - 1) // GEMM_ROW_BLOCK for c in counts))
    assert blocks_covered(sample, idx, n) == nblk
    assert sample.size >= min(512, T) and np.unique(sample).size == sample.size
    last_rows = offsets[1:][counts > 0] - 1
    assert set(row_token[last_rows].tolist()) <= set(sample.tolist())
