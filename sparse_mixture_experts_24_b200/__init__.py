"""B200 (sm_100a) sparse mixture-of-experts layer forward: thin ctypes binding.

The functions here carry the names of the C ABI in include/moe.h and only
marshal arguments (torch tensors or raw device pointers) into that library;
every step of the layer runs in its CUDA kernels.  Importing this package
fails with ImportError when libmoe_b200.so has not been built
(`python sparse_mixture_experts_24_b200/build.py`): there is no fallback.

The layer: y = sum_i Softmax(TopK(x . W_g))_i * SwiGLU_i(x) with
SwiGLU_i(x) = (silu(x . w1_i) * (x . w3_i)) . w2_i ("Mixtral of Experts",
section 2.1; Part 3, Steps 1-4 of "Mixture of Experts: Why Mixtral Only Wakes
Up Two Specialists").
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmoe_b200.so")

MOE_F32 = 0
MOE_BF16 = 1

MOE_OK = 0
MOE_ERR_INVALID_ARG = 1
MOE_ERR_UNSUPPORTED = 2
MOE_ERR_ALLOC = 3
MOE_ERR_CUDA = 4
MOE_ERR_TIMEOUT = 5

STATUS_NAMES = {0: "MOE_OK", 1: "MOE_ERR_INVALID_ARG", 2: "MOE_ERR_UNSUPPORTED",
                3: "MOE_ERR_ALLOC", 4: "MOE_ERR_CUDA", 5: "MOE_ERR_TIMEOUT"}


class MoEError(RuntimeError):
    def __init__(self, status: int, where: str, message: str):
        super().__init__("%s: %s (%s)" % (where, message, STATUS_NAMES.get(status, status)))
        self.status = status


if not os.path.exists(LIB_PATH):
    raise ImportError("libmoe_b200.so is not built; run `python sparse_mixture_experts_24_b200/build.py`")

_vp, _i64, _int = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int
lib = ctypes.CDLL(LIB_PATH)
lib.moe_create.argtypes = [_int, _int, _int, _int, _int, ctypes.POINTER(_vp)]
lib.moe_reserve.argtypes = [_vp, _i64]
lib.moe_forward.argtypes = [_vp, _i64, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp]
lib.moe_route.argtypes = [_vp, _i64, _vp, _vp, _vp, _vp, _vp]
lib.moe_dispatch.argtypes = [_vp, _i64, _vp, _vp, _vp, _vp, _vp, _vp]
lib.moe_forward_with_routing.argtypes = [_vp, _i64, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp]
lib.moe_workspace_view.argtypes = [_vp, ctypes.c_char_p, ctypes.POINTER(_vp), ctypes.POINTER(_i64)]
lib.moe_sync_status.argtypes = [_vp, _vp]
lib.moe_destroy.argtypes = [_vp]
lib.moe_trace_begin.argtypes = [_vp, _int]
lib.moe_forward_expert_choice.argtypes = [_vp, _i64, _i64, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp,
                                          _vp]
lib.moe_selftest_timeout.argtypes = [_vp, _int, _vp]
lib.moe_launch_count.argtypes = [_vp, ctypes.POINTER(_i64)]
lib.moe_set_capacity_factor.argtypes = [_vp, ctypes.c_double]
lib.moe_set_gate_rounding.argtypes = [_vp, _int]
lib.moe_router_stats.argtypes = [_vp, _i64, _vp, _vp, _vp, ctypes.c_float, _vp, _vp, _vp, _vp]
lib.moe_dispatch_noalloc.argtypes = [_i64, _int, _int, _vp, _vp, _vp, _vp, _vp, _vp]
lib.moe_trace_end.argtypes = [_vp, ctypes.POINTER(ctypes.c_double), _int, ctypes.POINTER(_int)]
lib.moe_quantize_weights_e4m3.argtypes = [_int, _int, _int, _vp, _int, _vp, _vp, _vp]
lib.moe_forward_e4m3.argtypes = [_vp, _i64, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp]
lib.moe_quantize_weights_fp4.argtypes = [_int, _int, _int, _vp, _int, _vp, _vp, _vp, _vp]
lib.moe_forward_fp4.argtypes = [_vp, _i64, _vp, _vp] + [_vp] * 9 + [_vp, _vp, _vp, _vp]
lib.moe_pack_weights_w4a4.argtypes = [_int, _int, _int, _vp, _vp, _vp, _vp, _vp, _vp, _vp]
lib.moe_forward_w4a4.argtypes = [_vp, _i64, _vp, _vp] + [_vp] * 7 + [_vp, _vp, _vp, _vp]
lib.moe_pack_weights_w4a16.argtypes = [_int, _int, _int, _vp, _vp, _vp, _vp, _vp, _vp]
lib.moe_forward_w4a16.argtypes = [_vp, _i64, _vp, _vp] + [_vp] * 5 + [_vp, _vp, _vp, _vp]
lib.moe_ep_dispatch.argtypes = [_vp, _int, _int, _i64, _vp, _vp, _vp, _vp, _i64, _vp, _vp]
lib.moe_ep_experts.argtypes = [_vp, _int, _int, _vp, _vp, _i64, _vp, _vp, _vp, _vp, _vp]
lib.moe_ep_combine.argtypes = [_vp, _int, _i64, _vp, _vp, _vp, _vp, _vp, _vp]
lib.moe_ep_buffer_alloc.argtypes = [_i64, ctypes.POINTER(_vp), _vp]
lib.moe_ep_buffer_open.argtypes = [_vp, ctypes.POINTER(_vp)]
lib.moe_ep_buffer_close.argtypes = [_vp, _int]
lib.moe_last_error.restype = ctypes.c_char_p
lib.moe_version.restype = ctypes.c_char_p
for _f in ("moe_create", "moe_reserve", "moe_forward", "moe_route", "moe_dispatch",
           "moe_forward_with_routing", "moe_workspace_view", "moe_sync_status", "moe_destroy",
           "moe_trace_begin", "moe_trace_end", "moe_dispatch_noalloc", "moe_set_capacity_factor",
           "moe_router_stats", "moe_launch_count", "moe_selftest_timeout",
           "moe_forward_expert_choice", "moe_quantize_weights_e4m3", "moe_forward_e4m3",
           "moe_quantize_weights_fp4", "moe_forward_fp4", "moe_pack_weights_w4a4", "moe_forward_w4a4",
           "moe_pack_weights_w4a16", "moe_forward_w4a16", "moe_ep_dispatch", "moe_ep_experts", "moe_ep_combine", "moe_ep_buffer_alloc", "moe_ep_buffer_open",
           "moe_ep_buffer_close", "moe_set_gate_rounding"):
    getattr(lib, _f).restype = _int

EXPORTED = ("moe_create", "moe_reserve", "moe_forward", "moe_route", "moe_dispatch",
            "moe_forward_with_routing", "moe_workspace_view", "moe_sync_status", "moe_destroy",
            "moe_last_error", "moe_version", "moe_trace_begin", "moe_trace_end",
            "moe_dispatch_noalloc", "moe_set_capacity_factor", "moe_router_stats",
            "moe_launch_count", "moe_selftest_timeout", "moe_forward_expert_choice",
            "moe_quantize_weights_e4m3", "moe_forward_e4m3", "moe_quantize_weights_fp4", "moe_forward_fp4",
            "moe_pack_weights_w4a4", "moe_forward_w4a4", "moe_pack_weights_w4a16", "moe_forward_w4a16",
            "moe_ep_dispatch", "moe_ep_experts", "moe_ep_combine",
            "moe_ep_buffer_alloc", "moe_ep_buffer_open", "moe_ep_buffer_close", "moe_set_gate_rounding")

TRACE_STAGES = ("router", "dispatch", "gather", "gemm1", "gemm2", "combine")


def _ptr(a):
    """Device (or host) address of a tensor, an int address, or None -> NULL."""
    if a is None:
        return None
    if isinstance(a, int):
        return a
    return a.data_ptr()


def _stream(s):
    if s is None:
        try:
            import torch
            if torch.cuda.is_available() and torch.cuda.is_initialized():
                return torch.cuda.current_stream().cuda_stream
        except ImportError:
            pass
        return None
    if isinstance(s, int):
        return s
    return s.cuda_stream


def _check(rc: int, where: str) -> None:
    if rc != MOE_OK:
        raise MoEError(rc, where, moe_last_error())


def moe_last_error() -> str:
    return lib.moe_last_error().decode()


def moe_version() -> str:
    return lib.moe_version().decode()


def moe_create(n: int, K: int, d: int, ffn: int, dtype: int) -> int:
    h = _vp()
    _check(lib.moe_create(n, K, d, ffn, dtype, ctypes.byref(h)), "moe_create")
    return h.value


def moe_reserve(h: int, T_max: int) -> None:
    _check(lib.moe_reserve(h, T_max), "moe_reserve")


def moe_forward(h, T, x, W_g, w1, w3, w2, y, topk_idx, topk_w, stream=None) -> None:
    _check(lib.moe_forward(h, T, _ptr(x), _ptr(W_g), _ptr(w1), _ptr(w3), _ptr(w2), _ptr(y),
                           _ptr(topk_idx), _ptr(topk_w), _stream(stream)), "moe_forward")


def moe_route(h, T, x, W_g, topk_idx, topk_w, stream=None) -> None:
    _check(lib.moe_route(h, T, _ptr(x), _ptr(W_g), _ptr(topk_idx), _ptr(topk_w), _stream(stream)),
           "moe_route")


def moe_dispatch(h, T, topk_idx, counts=None, offsets=None, row_token=None, token_row=None,
                 stream=None) -> None:
    _check(lib.moe_dispatch(h, T, _ptr(topk_idx), _ptr(counts), _ptr(offsets), _ptr(row_token),
                            _ptr(token_row), _stream(stream)), "moe_dispatch")


def moe_forward_with_routing(h, T, x, topk_idx, topk_w, w1, w3, w2, y, stream=None) -> None:
    _check(lib.moe_forward_with_routing(h, T, _ptr(x), _ptr(topk_idx), _ptr(topk_w), _ptr(w1),
                                        _ptr(w3), _ptr(w2), _ptr(y), _stream(stream)),
           "moe_forward_with_routing")


def moe_workspace_view(h, name: str):
    p, rows = _vp(), _i64()
    _check(lib.moe_workspace_view(h, name.encode(), ctypes.byref(p), ctypes.byref(rows)),
           "moe_workspace_view")
    return p.value, rows.value


def moe_sync_status(h, stream=None) -> None:
    _check(lib.moe_sync_status(h, _stream(stream)), "moe_sync_status")


def moe_dispatch_noalloc(T, n, K, topk_idx, counts, offsets, row_token, token_row,
                         stream=None) -> None:
    """Dispatch without a handle and without allocating device memory (scratch
    in a fixed array inside the library; T * K <= 65,536)."""
    _check(lib.moe_dispatch_noalloc(T, n, K, _ptr(topk_idx), _ptr(counts), _ptr(offsets),
                                    _ptr(row_token), _ptr(token_row), _stream(stream)),
           "moe_dispatch_noalloc")


def moe_set_capacity_factor(h, factor: float) -> None:
    _check(lib.moe_set_capacity_factor(h, float(factor)), "moe_set_capacity_factor")


def moe_router_stats(h, T, x, W_g, topk_idx, alpha, f, P, aux, stream=None) -> None:
    _check(lib.moe_router_stats(h, T, _ptr(x), _ptr(W_g), _ptr(topk_idx), float(alpha), _ptr(f),
                                _ptr(P), _ptr(aux), _stream(stream)), "moe_router_stats")


def moe_trace_begin(h, max_calls: int) -> None:
    _check(lib.moe_trace_begin(h, max_calls), "moe_trace_begin")


def moe_trace_end(h):
    """-> (dict stage -> summed ms, number of traced calls)"""
    ms = (ctypes.c_double * len(TRACE_STAGES))()
    calls = _int()
    _check(lib.moe_trace_end(h, ms, len(TRACE_STAGES), ctypes.byref(calls)), "moe_trace_end")
    return dict(zip(TRACE_STAGES, list(ms))), calls.value


def moe_forward_expert_choice(h, T, capacity, x, W_g, w1, w3, w2, y, sel_token, sel_gate,
                              stream=None) -> None:
    _check(lib.moe_forward_expert_choice(h, T, capacity, _ptr(x), _ptr(W_g), _ptr(w1), _ptr(w3),
                                         _ptr(w2), _ptr(y), _ptr(sel_token), _ptr(sel_gate),
                                         _stream(stream)), "moe_forward_expert_choice")


def moe_selftest_timeout(h, budget_us: int = 1000, stream=None) -> None:
    _check(lib.moe_selftest_timeout(h, budget_us, _stream(stream)), "moe_selftest_timeout")


def moe_launch_count(h) -> int:
    c = _i64()
    _check(lib.moe_launch_count(h, ctypes.byref(c)), "moe_launch_count")
    return c.value


def moe_quantize_weights_e4m3(n, rows, cols, w, dtype, codes, scales, stream=None) -> None:
    _check(lib.moe_quantize_weights_e4m3(n, rows, cols, _ptr(w), dtype, _ptr(codes), _ptr(scales),
                                         _stream(stream)), "moe_quantize_weights_e4m3")


def moe_forward_e4m3(h, T, x, W_g, w1_q, w1_s, w3_q, w3_s, w2_q, w2_s, y, topk_idx, topk_w,
                     stream=None) -> None:
    _check(lib.moe_forward_e4m3(h, T, _ptr(x), _ptr(W_g), _ptr(w1_q), _ptr(w1_s), _ptr(w3_q), _ptr(w3_s),
                                _ptr(w2_q), _ptr(w2_s), _ptr(y), _ptr(topk_idx), _ptr(topk_w),
                                _stream(stream)), "moe_forward_e4m3")


def quantize_weights_e4m3(w, stream=None):
    """w [n][rows][cols] (torch bf16 or fp32, CUDA) -> (codes uint8 [n][rows][cols],
    scales fp32 [n][cols]), one scale per output column."""
    import torch
    n, rows, cols = w.shape
    codes = torch.empty((n, rows, cols), dtype=torch.uint8, device=w.device)
    scales = torch.empty((n, cols), dtype=torch.float32, device=w.device)
    moe_quantize_weights_e4m3(n, rows, cols, w, MOE_BF16 if w.dtype == torch.bfloat16 else MOE_F32,
                              codes, scales, stream)
    return codes, scales


def moe_quantize_weights_fp4(n, rows, cols, w, dtype, codes, block_scales, matrix_scales, stream=None) -> None:
    _check(lib.moe_quantize_weights_fp4(n, rows, cols, _ptr(w), dtype, _ptr(codes), _ptr(block_scales),
                                        _ptr(matrix_scales), _stream(stream)), "moe_quantize_weights_fp4")


def moe_forward_fp4(h, T, x, W_g, w1_c, w1_b, w1_t, w3_c, w3_b, w3_t, w2_c, w2_b, w2_t, y, topk_idx, topk_w,
                    stream=None) -> None:
    _check(lib.moe_forward_fp4(h, T, _ptr(x), _ptr(W_g), _ptr(w1_c), _ptr(w1_b), _ptr(w1_t), _ptr(w3_c),
                               _ptr(w3_b), _ptr(w3_t), _ptr(w2_c), _ptr(w2_b), _ptr(w2_t), _ptr(y), _ptr(topk_idx),
                               _ptr(topk_w), _stream(stream)), "moe_forward_fp4")


def quantize_weights_fp4(w, stream=None):
    """w [n][rows][cols] (torch bf16 or fp32, CUDA) -> (codes uint8 [n][rows][cols/2],
    block scales uint8 [n][rows/16][cols] (E4M3 codes), matrix scales fp32 [n])."""
    import torch
    n, rows, cols = w.shape
    codes = torch.empty((n, rows, cols // 2), dtype=torch.uint8, device=w.device)
    bscale = torch.empty((n, rows // 16, cols), dtype=torch.uint8, device=w.device)
    tscale = torch.empty(n, dtype=torch.float32, device=w.device)
    moe_quantize_weights_fp4(n, rows, cols, w, MOE_BF16 if w.dtype == torch.bfloat16 else MOE_F32, codes, bscale,
                             tscale, stream)
    return codes, bscale, tscale


def moe_pack_weights_w4a4(n, rows, cols, codes, block_scales, pair_codes, pair_block_scales, packed, chunks,
                          stream=None) -> None:
    _check(lib.moe_pack_weights_w4a4(n, rows, cols, _ptr(codes), _ptr(block_scales), _ptr(pair_codes),
                                     _ptr(pair_block_scales), _ptr(packed), _ptr(chunks), _stream(stream)),
           "moe_pack_weights_w4a4")


def moe_forward_w4a4(h, T, x, W_g, w13_p, w13_c, w1_t, w3_t, w2_p, w2_c, w2_t, y, topk_idx, topk_w,
                     stream=None) -> None:
    _check(lib.moe_forward_w4a4(h, T, _ptr(x), _ptr(W_g), _ptr(w13_p), _ptr(w13_c), _ptr(w1_t), _ptr(w3_t),
                                _ptr(w2_p), _ptr(w2_c), _ptr(w2_t), _ptr(y), _ptr(topk_idx), _ptr(topk_w),
                                _stream(stream)), "moe_forward_w4a4")


def pack_weights_w4a4(codes, block_scales, matrix_scales, pair=None, stream=None):
    """(codes [n][rows][cols/2], block scales [n][rows/16][cols], matrix scales [n])
    of quantize_weights_fp4 (torch CUDA tensors) -> (packed codes [n][cols][rows/2],
    scale chunks [n][cols/128][rows/64][512], matrix scales).  With pair = w3's
    triple (codes being w1's): the gate/up pair pack of 2*cols packed columns,
    returned as (packed, chunks, w1 matrix scales, w3 matrix scales)."""
    import torch
    n, rows, half = codes.shape
    cols = 2 * half
    out_cols = 2 * cols if pair is not None else cols
    packed = torch.empty((n, out_cols, rows // 2), dtype=torch.uint8, device=codes.device)
    chunks = torch.empty((n, out_cols // 128, rows // 64, 512), dtype=torch.uint8, device=codes.device)
    pc, pb = (pair[0], pair[1]) if pair is not None else (None, None)
    moe_pack_weights_w4a4(n, rows, cols, codes, block_scales, pc, pb, packed, chunks, stream)
    if pair is not None:
        return packed, chunks, matrix_scales, pair[2]
    return packed, chunks, matrix_scales


def moe_pack_weights_w4a16(n, rows, cols, codes, block_scales, pair_codes, pair_block_scales, packed,
                           stream=None) -> None:
    _check(lib.moe_pack_weights_w4a16(n, rows, cols, _ptr(codes), _ptr(block_scales), _ptr(pair_codes),
                                      _ptr(pair_block_scales), _ptr(packed), _stream(stream)),
           "moe_pack_weights_w4a16")


def moe_forward_w4a16(h, T, x, W_g, w13_p, w1_t, w3_t, w2_p, w2_t, y, topk_idx, topk_w, stream=None) -> None:
    _check(lib.moe_forward_w4a16(h, T, _ptr(x), _ptr(W_g), _ptr(w13_p), _ptr(w1_t), _ptr(w3_t), _ptr(w2_p),
                                 _ptr(w2_t), _ptr(y), _ptr(topk_idx), _ptr(topk_w), _stream(stream)),
           "moe_forward_w4a16")


def pack_weights_w4a16(codes, block_scales, matrix_scales, pair=None, stream=None):
    """(codes [n][rows][cols/2], block scales [n][rows/16][cols], matrix scales [n])
    of quantize_weights_fp4 (torch CUDA tensors) -> (packed [n][cols/128][rows/64][4608],
    matrix scales).  With pair = w3's triple (codes being w1's): the gate/up pair
    pack [n][cols/64][rows/64][4608], returned as (packed, w1 matrix scales,
    w3 matrix scales)."""
    import torch
    n, rows, half = codes.shape
    cols = 2 * half
    tiles = cols // 64 if pair is not None else cols // 128
    packed = torch.empty((n, tiles, rows // 64, 4608), dtype=torch.uint8, device=codes.device)
    pc, pb = (pair[0], pair[1]) if pair is not None else (None, None)
    moe_pack_weights_w4a16(n, rows, cols, codes, block_scales, pc, pb, packed, stream)
    if pair is not None:
        return packed, matrix_scales, pair[2]
    return packed, matrix_scales


def _ptr_table(ptrs):
    """Host array of device addresses (tensors, ints) for the peer tables."""
    return (ctypes.c_void_p * len(ptrs))(*[_ptr(p) for p in ptrs])


def moe_ep_dispatch(h, world, rank, T, x, topk_idx, counts_all, recv_buffers, recv_rows, row_pos,
                    stream=None) -> None:
    _check(lib.moe_ep_dispatch(h, world, rank, T, _ptr(x), _ptr(topk_idx), _ptr(counts_all),
                               _ptr_table(recv_buffers), recv_rows, _ptr(row_pos), _stream(stream)),
           "moe_ep_dispatch")


def moe_ep_experts(h, world, rank, counts_all, recv, recv_rows, w1, w3, w2, out, stream=None) -> None:
    _check(lib.moe_ep_experts(h, world, rank, _ptr(counts_all), _ptr(recv), recv_rows, _ptr(w1), _ptr(w3),
                              _ptr(w2), _ptr(out), _stream(stream)), "moe_ep_experts")


def moe_ep_combine(h, world, T, topk_idx, topk_w, row_pos, out_buffers, y, stream=None) -> None:
    _check(lib.moe_ep_combine(h, world, T, _ptr(topk_idx), _ptr(topk_w), _ptr(row_pos),
                              _ptr_table(out_buffers), _ptr(y), _stream(stream)), "moe_ep_combine")


def moe_ep_buffer_alloc(nbytes: int, with_ipc_handle: bool = True):
    """-> (device address, 64-byte IPC handle or None)."""
    p = ctypes.c_void_p()
    hd = ctypes.create_string_buffer(64) if with_ipc_handle else None
    _check(lib.moe_ep_buffer_alloc(nbytes, ctypes.byref(p), hd), "moe_ep_buffer_alloc")
    return p.value, (hd.raw if hd is not None else None)


def moe_ep_buffer_open(handle: bytes) -> int:
    p = ctypes.c_void_p()
    buf = ctypes.create_string_buffer(bytes(handle), 64)
    _check(lib.moe_ep_buffer_open(buf, ctypes.byref(p)), "moe_ep_buffer_open")
    return p.value


def moe_ep_buffer_close(ptr: int, opened: bool) -> None:
    _check(lib.moe_ep_buffer_close(ptr, 1 if opened else 0), "moe_ep_buffer_close")


def moe_set_gate_rounding(h, bf16: int) -> None:
    _check(lib.moe_set_gate_rounding(h, bf16), "moe_set_gate_rounding")


def moe_destroy(h) -> None:
    _check(lib.moe_destroy(h), "moe_destroy")


class MoELayer:
    """Owns one handle; allocates outputs with torch and calls the C ABI.

    Tensors are torch CUDA tensors; bf16 layers take torch.bfloat16 x and
    weights, fp32 layers torch.float32; W_g is always torch.float32 [d][n].
    """

    def __init__(self, n: int, K: int, d: int, ffn: int, dtype: str = "bf16"):
        self.n, self.K, self.d, self.ffn = n, K, d, ffn
        self.dtype = dtype
        self.h = moe_create(n, K, d, ffn, MOE_BF16 if dtype == "bf16" else MOE_F32)

    def reserve(self, T_max: int) -> None:
        moe_reserve(self.h, T_max)

    def forward(self, x, W_g, w1, w3, w2, y=None, topk_idx=None, topk_w=None, stream=None):
        import torch
        T = x.shape[0]
        if y is None:
            y = torch.empty_like(x)
        if topk_idx is None:
            topk_idx = torch.empty((T, self.K), dtype=torch.int32, device=x.device)
        if topk_w is None:
            topk_w = torch.empty((T, self.K), dtype=torch.float32, device=x.device)
        moe_forward(self.h, T, x, W_g, w1, w3, w2, y, topk_idx, topk_w, stream)
        return y, topk_idx, topk_w

    def route(self, x, W_g, stream=None):
        import torch
        T = x.shape[0]
        idx = torch.empty((T, self.K), dtype=torch.int32, device=x.device)
        w = torch.empty((T, self.K), dtype=torch.float32, device=x.device)
        moe_route(self.h, T, x, W_g, idx, w, stream)
        return idx, w

    def forward_with_routing(self, x, topk_idx, topk_w, w1, w3, w2, y=None, stream=None):
        import torch
        if y is None:
            y = torch.empty_like(x)
        moe_forward_with_routing(self.h, x.shape[0], x, topk_idx, topk_w, w1, w3, w2, y, stream)
        return y

    def dispatch(self, topk_idx, stream=None):
        import torch
        T = topk_idx.shape[0]
        dev = topk_idx.device
        counts = torch.empty(self.n, dtype=torch.int32, device=dev)
        offsets = torch.empty(self.n + 1, dtype=torch.int32, device=dev)
        row_token = torch.empty(max(1, T * self.K), dtype=torch.int32, device=dev)
        token_row = torch.empty((max(1, T), self.K), dtype=torch.int32, device=dev)
        moe_dispatch(self.h, T, topk_idx, counts, offsets, row_token, token_row, stream)
        return counts, offsets, row_token[:T * self.K], token_row[:T]

    def forward_expert_choice(self, x, W_g, w1, w3, w2, capacity: int, stream=None):
        """-> y, sel_token [n][capacity], sel_gate [n][capacity]"""
        import torch
        T = x.shape[0]
        y = torch.empty_like(x)
        sel = torch.empty((self.n, capacity), dtype=torch.int32, device=x.device)
        gate = torch.empty((self.n, capacity), dtype=torch.float32, device=x.device)
        moe_forward_expert_choice(self.h, T, capacity, x, W_g, w1, w3, w2, y, sel, gate, stream)
        return y, sel, gate

    def forward_e4m3(self, x, W_g, w1_q, w1_s, w3_q, w3_s, w2_q, w2_s, y=None, topk_idx=None,
                     topk_w=None, stream=None):
        """The layer with E4M3 experts (codes and scales of quantize_weights_e4m3)."""
        import torch
        T = x.shape[0]
        if y is None:
            y = torch.empty_like(x)
        if topk_idx is None:
            topk_idx = torch.empty((T, self.K), dtype=torch.int32, device=x.device)
        if topk_w is None:
            topk_w = torch.empty((T, self.K), dtype=torch.float32, device=x.device)
        moe_forward_e4m3(self.h, T, x, W_g, w1_q, w1_s, w3_q, w3_s, w2_q, w2_s, y, topk_idx, topk_w, stream)
        return y, topk_idx, topk_w

    def forward_fp4(self, x, W_g, w1, w3, w2, y=None, topk_idx=None, topk_w=None, stream=None):
        """The layer with 4-bit experts; w1, w3, w2 are (codes, block scales,
        matrix scales) triples from quantize_weights_fp4."""
        import torch
        T = x.shape[0]
        if y is None:
            y = torch.empty_like(x)
        if topk_idx is None:
            topk_idx = torch.empty((T, self.K), dtype=torch.int32, device=x.device)
        if topk_w is None:
            topk_w = torch.empty((T, self.K), dtype=torch.float32, device=x.device)
        moe_forward_fp4(self.h, T, x, W_g, *w1, *w3, *w2, y, topk_idx, topk_w, stream)
        return y, topk_idx, topk_w

    def forward_w4a4(self, x, W_g, w13, w2, y=None, topk_idx=None, topk_w=None, stream=None):
        """The layer with 4-bit weights and activations; w13 is the gate/up pair
        pack (packed, chunks, w1 scales, w3 scales) and w2 the (packed, chunks,
        matrix scales) triple, both from pack_weights_w4a4."""
        import torch
        T = x.shape[0]
        if y is None:
            y = torch.empty_like(x)
        if topk_idx is None:
            topk_idx = torch.empty((T, self.K), dtype=torch.int32, device=x.device)
        if topk_w is None:
            topk_w = torch.empty((T, self.K), dtype=torch.float32, device=x.device)
        moe_forward_w4a4(self.h, T, x, W_g, *w13, *w2, y, topk_idx, topk_w, stream)
        return y, topk_idx, topk_w

    def forward_w4a16(self, x, W_g, w13, w2, y=None, topk_idx=None, topk_w=None, stream=None):
        """The layer with 4-bit weights decoded into tensor memory and bf16
        activations; w13 is the gate/up pair pack (packed, w1 scales, w3 scales)
        and w2 the (packed, matrix scales) pair, both from pack_weights_w4a16."""
        import torch
        T = x.shape[0]
        if y is None:
            y = torch.empty_like(x)
        if topk_idx is None:
            topk_idx = torch.empty((T, self.K), dtype=torch.int32, device=x.device)
        if topk_w is None:
            topk_w = torch.empty((T, self.K), dtype=torch.float32, device=x.device)
        moe_forward_w4a16(self.h, T, x, W_g, *w13, *w2, y, topk_idx, topk_w, stream)
        return y, topk_idx, topk_w

    def set_capacity_factor(self, factor: float) -> None:
        moe_set_capacity_factor(self.h, factor)

    def set_gate_rounding(self, bf16: bool) -> None:
        moe_set_gate_rounding(self.h, 1 if bf16 else 0)

    def router_stats(self, x, W_g, topk_idx, alpha=0.01, stream=None):
        """-> f [n], P [n], aux [1] (device float32 tensors)."""
        import torch
        f = torch.empty(self.n, dtype=torch.float32, device=x.device)
        P = torch.empty(self.n, dtype=torch.float32, device=x.device)
        aux = torch.empty(1, dtype=torch.float32, device=x.device)
        moe_router_stats(self.h, x.shape[0], x, W_g, topk_idx, alpha, f, P, aux, stream)
        return f, P, aux

    def sync_status(self, stream=None) -> None:
        moe_sync_status(self.h, stream)

    def close(self) -> None:
        if self.h:
            moe_destroy(self.h)
            self.h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
