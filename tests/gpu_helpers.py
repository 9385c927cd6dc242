"""Helpers shared by the GPU parity tests: device copies of the seeded inputs,
routing comparison with near-tie accounting, and the reference y."""
from __future__ import annotations

import numpy as np

import moe_inputs as mi
import oracle

NEAR_TIE = 1e-4          # gap below which two logits count as a near-tie
TOL_Y = {"f32": 1e-5, "bf16": 2e-2}   # relative L2 bars on y


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
