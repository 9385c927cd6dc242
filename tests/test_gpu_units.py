"""Per-kernel checks of the bf16 tensor-core GEMMs through the workspace view
(needs a B200): H after GEMM1 and O after GEMM2 against numpy fp64 on the same
bf16 inputs, row by row, so a wrong descriptor or epilogue mapping shows up as
the exact rows / columns it breaks."""
import numpy as np
import pytest

import moe_inputs as mi
from gpu_helpers import dev, host, require_cuda

pytestmark = pytest.mark.gpu


def silu(z):
    return z / (1.0 + np.exp(-z))


class _DevArray:
    """Borrowed view of device memory for torch.as_tensor (CUDA array interface)."""

    def __init__(self, ptr, shape, typestr):
        self.__cuda_array_interface__ = {"shape": tuple(shape), "typestr": typestr,
                                         "data": (int(ptr), False), "version": 3, "strides": None}


def read_ws(layer, name, rows, cols, torch_dtype):
    """Copy rows x cols of workspace buffer `name` ("H" or "O") to a new tensor."""
    import sparse_mixture_experts_24_b200 as m
    torch = require_cuda()
    ptr, cap = m.moe_workspace_view(layer.h, name)
    assert cap >= rows
    typestr = "<i2" if torch_dtype == torch.bfloat16 else "<f4"
    t = torch.as_tensor(_DevArray(ptr, (rows, cols), typestr), device="cuda").clone()
    torch.cuda.synchronize()
    return t.view(torch.bfloat16) if torch_dtype == torch.bfloat16 else t


@pytest.mark.parametrize("path", ["single", "single_fused_gather", "single_separate_gather", "single_banded", "pair",
                                  "dual", "dual_banded"])
@pytest.mark.parametrize("T,d,F,n,K", [(200, 128, 256, 4, 2), (333, 256, 384, 8, 2), (129, 320, 192, 3, 1),
                                       (700, 192, 320, 2, 1), (1500, 256, 512, 3, 2)])
def test_gemm1_and_gemm2_rows(T, d, F, n, K, path, monkeypatch):
    """path: single-SM tiles (128 rows; the library's choice of gather), the
    same with GEMM1 gathering its x rows itself, or with the x rows gathered
    into Xp by their own kernel, the same with
    bands of a row block or two in the tile order (64 KB of A rows), CTA-pair tiles (256 rows,
    cta_group::2), or two row blocks per single-SM tile (x rows gathered into
    Xp by their own kernel; with and without bands of a pair or two)."""
    monkeypatch.setenv("MOE_GEMM_PATH", path.split("_")[0] if path.startswith(("pair", "dual")) else "single")
    if path.startswith("dual"):
        monkeypatch.setenv("MOE_GATHER", "separate")
    if path == "dual_banded":
        monkeypatch.setenv("MOE_GEMM1_BAND_KB", "128")
        monkeypatch.setenv("MOE_GEMM2_BAND_KB", "128")
    if path == "single_separate_gather":
        monkeypatch.setenv("MOE_GATHER", "separate")
    if path == "single_fused_gather":
        monkeypatch.setenv("MOE_GATHER", "fused")
    if path == "single_banded":
        monkeypatch.setenv("MOE_GEMM1_BAND_KB", "64")
        monkeypatch.setenv("MOE_GEMM2_BAND_KB", "64")
    import sparse_mixture_experts_24_b200 as m
    torch = require_cuda()
    cfg = mi.custom_config("units", T=T, d=d, ffn=F, n=n, K=K, dtype="bf16")
    L = mi.make_layer(cfg, seed=5)
    layer = m.MoELayer(n, K, d, F, "bf16")
    try:
        y, idx, w = layer.forward(*[dev(L[k]) for k in ("x", "W_g", "w1", "w3", "w2")])
        layer.sync_status()
        idx = host(idx)
        counts, offsets, row_token, token_row = (host(t) for t in layer.dispatch(dev(idx)))
        R = T * K
        H = host(read_ws(layer, "H", R, F, torch.bfloat16))
        O = host(read_ws(layer, "O", R, d, torch.bfloat16))
    finally:
        layer.close()
    x = mi.as_f32(L["x"]).astype(np.float64)
    w1 = mi.as_f32(L["w1"]).astype(np.float64)
    w3 = mi.as_f32(L["w3"]).astype(np.float64)
    w2 = mi.as_f32(L["w2"]).astype(np.float64)
    Hf = mi.as_f32(H).astype(np.float64)
    Of = mi.as_f32(O).astype(np.float64)
    bad_h, bad_o = [], []
    for e in range(n):
        rows = np.arange(offsets[e], offsets[e + 1])
        if rows.size == 0:
            continue
        xe = x[row_token[rows]]
        h_ref = silu(xe @ w1[e]) * (xe @ w3[e])
        o_ref = Hf[rows] @ w2[e]          # GEMM2 checked on the GPU's own H
        eh = np.abs(Hf[rows] - h_ref) > 1e-2 * (np.abs(h_ref) + 0.05)
        eo = np.abs(Of[rows] - o_ref) > 1e-2 * (np.abs(o_ref) + 0.05)
        if eh.any():
            r, c = np.nonzero(eh)
            bad_h.append((e, int(eh.sum()), rows[r[:3]].tolist(), c[:8].tolist()))
        if eo.any():
            r, c = np.nonzero(eo)
            bad_o.append((e, int(eo.sum()), rows[r[:3]].tolist(), c[:8].tolist()))
    assert not bad_h, "GEMM1 mismatches (expert, count, rows, cols): %s" % bad_h
    assert not bad_o, "GEMM2 mismatches (expert, count, rows, cols): %s" % bad_o
