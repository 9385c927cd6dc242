"""Helpers shared by the GPU parity tests: device copies of the seeded inputs,
routing comparison with near-tie accounting, and the reference y."""
from __future__ import annotations

import numpy as np

import moe_inputs as mi
import oracle

NEAR_TIE = 1e-4          # gap below which two logits count as a near-tie
TOL_Y = {"f32": 1e-5, "bf16": 2e-2}   # relative L2 bars on y
PER_TOKEN_FACTOR = 5                   # per-token relative L2 bar = 5 x the aggregate one
GEMM_ROW_BLOCK = 128                   # rows per M-block of the bf16 grouped GEMMs (MMA M)


def require_cuda():
    import torch
    if not torch.cuda.is_available():
        raise RuntimeError("GPU test collected on a machine without CUDA")
    return torch


def dev(a: np.ndarray):
    """numpy -> CUDA tensor; uint16 bf16 bit patterns become torch.bfloat16."""
    torch = require_cuda()
    t = torch.from_numpy(np.ascontiguousarray(a))
    if a.dtype == np.uint16:
        t = t.view(torch.int16).view(torch.bfloat16)
    return t.cuda()


def host(t) -> np.ndarray:
    """CUDA tensor -> numpy (bf16 -> uint16 bit patterns)."""
    import torch
    t = t.detach().cpu()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    return t.numpy()


class DevArray:
    """Borrowed view of device memory for torch.as_tensor (CUDA array interface)."""

    def __init__(self, ptr, shape, typestr):
        self.__cuda_array_interface__ = {"shape": tuple(shape), "typestr": typestr,
                                         "data": (int(ptr), False), "version": 3, "strides": None}


def read_workspace(layer, name: str, rows: int, cols: int, dtype) -> np.ndarray:
    """Copy rows x cols of a handle's workspace buffer to a numpy array of
    `dtype` (uint8, uint16 for bf16 bits, float32)."""
    import sparse_mixture_experts_24_b200 as m
    torch = require_cuda()
    ptr, cap = m.moe_workspace_view(layer.h, name)
    assert cap >= rows
    typestr = {np.dtype(np.uint8): "|u1", np.dtype(np.uint16): "<i2", np.dtype(np.float32): "<f4"}[np.dtype(dtype)]
    torch.cuda.synchronize()
    t = torch.as_tensor(DevArray(ptr, (rows, cols), typestr), device="cuda").clone()
    torch.cuda.synchronize()
    return t.cpu().numpy().view(dtype)


def y_as_f64(y: np.ndarray) -> np.ndarray:
    return mi.as_f32(y).astype(np.float64)


def rel_l2(a, b) -> float:
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


def compare_routing(gpu_idx, gpu_w, o_idx, o_gate, o_logits, x, Wg, K):
    """Routing indices bit-exact except near-ties; gates within a bound derived
    from the fp32 dot-product error.  Returns a report dict."""
    T, n = o_logits.shape
    order = np.argsort(-o_logits, axis=1, kind="stable")
    srt = np.take_along_axis(o_logits, order, axis=1)
    m = min(K + 1, n)
    gaps = np.diff(-srt[:, :m], axis=1) if m > 1 else np.zeros((T, 0))
    near = (gaps < NEAR_TIE).any(axis=1) if gaps.size else np.zeros(T, bool)
    same_order = (gpu_idx == o_idx).all(axis=1)
    same_set = (np.sort(gpu_idx, 1) == np.sort(o_idx, 1)).all(axis=1)
    bad = ~same_order & ~near
    assert not bad.any(), "routing differs on %d tokens that are not near-ties (first %s)" % (
        bad.sum(), np.nonzero(bad)[0][:5])
    # gates: |dg| <= 0.5 * |d(L_i - L_j)|; fp32 dot error <= d * 2^-24 * sum |x||w|
    xf = mi.as_f32(x).astype(np.float64)
    d = xf.shape[1]
    absdot = np.abs(xf) @ np.abs(Wg.astype(np.float64))
    bound_L = d * 2.0 ** -24 * absdot.max(axis=1) + 1e-7
    tol = bound_L + 1e-6
    ok_tok = same_order
    err = np.abs(gpu_w.astype(np.float64) - o_gate)[ok_tok].max(axis=1) if ok_tok.any() else np.zeros(0)
    assert (err <= tol[ok_tok]).all(), "gate error %.3g above bound" % float((err - tol[ok_tok]).max())
    assert np.allclose(gpu_w.sum(1), 1.0, atol=1e-5)
    return {"near_ties": int(near.sum()), "set_differs": int((~same_set).sum()),
            "order_differs": int((~same_order & same_set).sum()), "max_gate_err": float(err.max()) if err.size else 0.0}


def agreeing_tokens(gpu_idx, o_idx) -> np.ndarray:
    """Tokens whose GPU routing equals the oracle's (order included); the
    others are near-ties that compare_routing has already accounted for."""
    agree = (gpu_idx == o_idx).all(axis=1)
    assert agree.mean() >= 0.99, "routing agrees on only %.3f of the tokens" % agree.mean()
    return agree


def stratified_sample(idx: np.ndarray, n: int, count: int, seed: int = 0) -> np.ndarray:
    """Token sample that includes at least one token of every used expert."""
    rng = np.random.default_rng(seed)
    T = idx.shape[0]
    pick = []
    for e in range(n):
        toks = np.nonzero((idx == e).any(axis=1))[0]
        if toks.size:
            pick.append(int(rng.choice(toks)))
    rest = rng.permutation(T)
    for t in rest:
        if len(set(pick)) >= min(count, T):
            break
        pick.append(int(t))
    return np.array(sorted(set(pick)), np.int64)


def near_tie_mask(o_logits, K):
    """Tokens with an adjacent gap below NEAR_TIE among the oracle's top K+1
    logits (the definition compare_routing counts)."""
    T, n = o_logits.shape
    srt = -np.sort(-o_logits, axis=1)
    m = min(K + 1, n)
    if m < 2:
        return np.zeros(T, bool)
    return (np.diff(-srt[:, :m], axis=1) < NEAR_TIE).any(axis=1)


def block_covering_sample(o_idx, n, count=512, block=GEMM_ROW_BLOCK, seed=0):
    """Tokens such that every (expert, M-block) of the grouped GEMMs holds at
    least one sampled row.  The GEMMs cut each expert's segment of the
    dispatch (oracle.dispatch of the oracle's routing: experts ascending,
    tokens ascending) into `block`-row M-blocks from the segment start; one
    random row of every block is taken, and the segment's last row (the
    ragged end of its last block), then random tokens up to `count`.
    -> (tokens sorted, number of M-blocks)."""
    counts, offsets, row_token, _ = oracle.dispatch(o_idx, n)
    rng = np.random.default_rng(seed)
    pick = set()
    blocks = 0
    for e in range(n):
        lo, hi = int(offsets[e]), int(offsets[e + 1])
        for b0 in range(lo, hi, block):
            pick.add(int(row_token[rng.integers(b0, min(b0 + block, hi))]))
            blocks += 1
        if hi > lo:
            pick.add(int(row_token[hi - 1]))
    T = o_idx.shape[0]
    for t in rng.permutation(T):
        if len(pick) >= min(count, T):
            break
        pick.add(int(t))
    return np.array(sorted(pick), np.int64), blocks


def blocks_covered(tokens, o_idx, n, block=GEMM_ROW_BLOCK):
    """Number of distinct (expert, M-block) pairs the rows of `tokens` fall in."""
    counts, offsets, _, token_row = oracle.dispatch(o_idx, n)
    seg = np.repeat(np.arange(n), counts)             # expert of each row
    rows = token_row[tokens].ravel()
    e = seg[rows]
    return len(set(zip(e.tolist(), ((rows - offsets[e]) // block).tolist())))


def y_check_with_alternatives(y_gpu, gpu_idx, o_logits, o_idx, o_gate, tokens, L, K, tol):
    """y of the sampled tokens against the oracle's layer.  A token whose
    routing agrees with the oracle's is compared with the oracle's y; a
    near-tie token with the closest of the oracle's own alternative routings
    (oracle.routing_alternatives: every ordering of its top logits closer
    than NEAR_TIE, with the oracle's gates for each), and its GPU routing
    must be one of those alternatives.  No GPU value is an oracle input.
    Returns (aggregate rel-L2, worst per-token rel-L2, number of near-tie
    tokens checked)."""
    tokens = np.asarray(tokens, np.int64)
    agree = (gpu_idx[tokens] == o_idx[tokens]).all(axis=1)
    ref = np.zeros((tokens.size, L["x"].shape[1]))
    ta = tokens[agree]
    if ta.size:
        ref[agree] = oracle.forward_with_routing(L["x"][ta], o_idx[ta], o_gate[ta], L["w1"], L["w3"], L["w2"])
    yg = y_as_f64(y_gpu[tokens])
    tied = np.nonzero(~agree)[0]
    for j in tied:
        t = int(tokens[j])
        alts = oracle.routing_alternatives(o_logits[t], K, NEAR_TIE)
        assert tuple(gpu_idx[t]) in {tuple(int(e) for e in i) for i, _ in alts}, \
            "token %d: GPU routing %s is no near-tie alternative of the oracle's" % (t, gpu_idx[t])
        ai = np.stack([i for i, _ in alts])
        ag = np.stack([g for _, g in alts])
        xs = np.repeat(L["x"][t:t + 1], len(alts), axis=0)
        ys = oracle.forward_with_routing(xs, ai, ag, L["w1"], L["w3"], L["w2"])
        errs = np.linalg.norm(ys - yg[j], axis=1)
        ref[j] = ys[int(np.argmin(errs))]
    per_tok = np.linalg.norm(yg - ref, axis=1) / np.maximum(np.linalg.norm(ref, axis=1), 1e-30)
    return rel_l2(yg, ref), float(per_tok.max()), int(tied.size)
