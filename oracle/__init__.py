"""fp64 CPU oracle for the sparse MoE layer forward (ctypes wrapper over moe_oracle.c).

TEST INFRASTRUCTURE ONLY: the tests, the smoke check and the benchmark's CPU
baseline leg may import this package; the product package never does.  It
shares no code with the CUDA library.

Functions (all inputs numpy arrays; x and weights may be float32, float64 or
bf16 bit patterns stored as uint16, and are widened exactly to double):

  router(x, W_g, K)                     -> idx [T,K] int32, gate [T,K] f64, logits [T,n] f64
  gates_to_bf16(gate)                   -> the gates cast to bf16 as the quoted routing code
                                           does (fp64 -> fp32 -> bf16, nearest even), as f64
  routing_alternatives(logits_row, K, gap) -> the top-K routings (and their softmax gates)
                                           a ranking that can misorder logits closer
                                           than gap may produce, the oracle's own first
  expert(x_row, w1, w3, w2, e)          -> [d] f64, one SwiGLU expert on one token
  forward_with_routing(x, idx, gate, w1, w3, w2) -> y [T,d] f64
  moe_forward(x, W_g, w1, w3, w2, K)    -> y, idx, gate
  dispatch(idx, n)                      -> counts, offsets, row_token, token_row
  dispatch_capacity(idx, n, C)          -> the same with at most C pairs per expert
  router_stats(x, W_g, idx, alpha)      -> f [n], P [n], aux (load-balancing statistics)
  expert_choice(x, W_g, w1, w3, w2, C)  -> y, sel_token [n][C], sel_gate [n][C]
  silu(z)                               -> z * sigmoid(z) in double

Sources: the layer equation of "Mixtral of Experts" section 2.1 (flash-card
page learn.ifs.name/d/jiang2024) and Part 3, Steps 1-4, of "Mixture of
Experts: Why Mixtral Only Wakes Up Two Specialists" (neobadger.com).
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "moe_oracle.c")
_LIB = os.path.join(_HERE, "libmoe_oracle.so")

_F32, _BF16, _F64 = 0, 1, 2


def compile_source(src: str, out: str) -> str:
    """gcc -O2 (no fast-math: IEEE double semantics), OpenMP over tokens."""
    tmp = out + ".tmp%d" % os.getpid()
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared",
                           "-Wall", "-Wextra", "-o", tmp, src, "-lm"])
    os.replace(tmp, out)
    return out


def build(force: bool = False) -> str:
    """Compile moe_oracle.c in place (libmoe_oracle.so beside it)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        compile_source(_SRC, _LIB)
    return _LIB


def _bind(L):
    vp, i64, i32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int
    L.oracle_router.argtypes = [i64, i32, i32, i32, vp, i32, vp, i32, vp, vp, vp]
    L.oracle_gates_to_bf16.argtypes = [i64, vp, vp]
    L.oracle_expert.argtypes = [i32, i32, i32, i32, vp, i32, vp, vp, vp, i32, vp]
    L.oracle_forward_with_routing.argtypes = [i64, i32, i32, i32, i32, vp, i32, vp, vp,
                                              vp, vp, vp, i32, vp]
    L.oracle_moe_forward.argtypes = [i64, i32, i32, i32, i32, vp, i32, vp, i32,
                                     vp, vp, vp, i32, vp, vp, vp]
    L.oracle_dispatch.argtypes = [i64, i32, i32, vp, vp, vp, vp, vp]
    L.oracle_router_stats.argtypes = [i64, i32, i32, i32, vp, i32, vp, i32, vp, ctypes.c_double,
                                      vp, vp, vp]
    L.oracle_dispatch_capacity.argtypes = [i64, i32, i32, vp, i64, vp, vp, vp, vp]
    L.oracle_e4m3_decode.argtypes = [ctypes.c_int]
    L.oracle_e4m3_decode.restype = ctypes.c_double
    L.oracle_e4m3_encode.argtypes = [ctypes.c_double]
    L.oracle_e4m3_encode.restype = ctypes.c_int
    L.oracle_quantize_weights_e4m3.argtypes = [i32, i32, i32, vp, i32, vp, vp]
    L.oracle_forward_e4m3.argtypes = [i64, i32, i32, i32, i32, vp, i32, vp, vp, vp, vp, vp, vp, vp,
                                      vp, vp]
    L.oracle_expert_choice.argtypes = [i64, i32, i32, i32, i64, vp, i32, vp, i32, vp, vp, vp, i32,
                                       vp, vp, vp]
    L.oracle_e2m1_decode.argtypes = [ctypes.c_int]
    L.oracle_e2m1_decode.restype = ctypes.c_double
    L.oracle_e2m1_encode.argtypes = [ctypes.c_double]
    L.oracle_e2m1_encode.restype = ctypes.c_int
    L.oracle_quantize_weights_fp4.argtypes = [i32, i32, i32, vp, i32, vp, vp, vp]
    L.oracle_dequantize_fp4.argtypes = [i32, i32, i32, vp, vp, vp, vp]
    L.oracle_forward_fp4.argtypes = [i64, i32, i32, i32, i32, vp, i32, vp, vp] + [vp] * 9 + [vp]
    L.oracle_quantize_rows_fp4.argtypes = [i64, i32, vp, i32, vp, vp, vp]
    L.oracle_forward_w4a4.argtypes = [i64, i32, i32, i32, i32, vp, i32, vp, vp] + [vp] * 9 + [vp]
    L.oracle_silu.argtypes = [ctypes.c_double]
    L.oracle_silu.restype = ctypes.c_double
    L.oracle_num_threads.restype = ctypes.c_int
    L.oracle_set_num_threads.argtypes = [ctypes.c_int]
    for f in ("oracle_router", "oracle_expert", "oracle_forward_with_routing",
              "oracle_moe_forward", "oracle_dispatch", "oracle_router_stats",
              "oracle_dispatch_capacity", "oracle_expert_choice", "oracle_quantize_weights_e4m3",
              "oracle_forward_e4m3", "oracle_quantize_weights_fp4", "oracle_dequantize_fp4",
              "oracle_forward_fp4", "oracle_quantize_rows_fp4", "oracle_forward_w4a4"):
        getattr(L, f).restype = ctypes.c_int
    return L


def _dt(a: np.ndarray) -> int:
    if a.dtype == np.float32:
        return _F32
    if a.dtype == np.uint16:
        return _BF16
    if a.dtype == np.float64:
        return _F64
    raise TypeError("oracle inputs must be float32, float64 or bf16 bits (uint16), got %s" % a.dtype)


def _p(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _c(a):
    a = np.asarray(a)
    if a.dtype not in (np.float32, np.float64, np.uint16):
        a = a.astype(np.float64)
    return np.ascontiguousarray(a)


def _check(rc: int, what: str) -> None:
    if rc != 0:
        raise ValueError("oracle %s rejected its arguments" % what)


class Oracle:
    """The oracle's entry points bound to one compiled copy of moe_oracle.c."""

    def __init__(self, path: str):
        self.path = path
        self.L = _bind(ctypes.CDLL(path))

    def num_threads(self) -> int:
        return int(self.L.oracle_num_threads())

    def set_num_threads(self, n: int) -> None:
        self.L.oracle_set_num_threads(int(n))

    def silu(self, z: float) -> float:
        return float(self.L.oracle_silu(float(z)))

    def router(self, x, W_g, K: int):
        x, W_g = _c(x), _c(W_g)
        T, d = x.shape
        d2, n = W_g.shape
        assert d == d2
        idx = np.empty((T, K), np.int32)
        gate = np.empty((T, K), np.float64)
        logits = np.empty((T, n), np.float64)
        _check(self.L.oracle_router(T, d, n, K, _p(x), _dt(x), _p(W_g), _dt(W_g),
                                    _p(idx), _p(gate), _p(logits)), "router")
        return idx, gate, logits

    def gates_to_bf16(self, gate):
        gate = np.ascontiguousarray(gate, dtype=np.float64)
        out = np.empty_like(gate)
        _check(self.L.oracle_gates_to_bf16(gate.size, _p(gate), _p(out)), "gates_to_bf16")
        return out

    def expert(self, x_row, w1, w3, w2, e: int):
        x_row, w1, w3, w2 = _c(x_row), _c(w1), _c(w3), _c(w2)
        n, d, F = w1.shape
        assert w3.shape == (n, d, F) and w2.shape == (n, F, d) and x_row.shape == (d,)
        assert w1.dtype == w3.dtype == w2.dtype
        out = np.empty(d, np.float64)
        _check(self.L.oracle_expert(d, F, n, e, _p(x_row), _dt(x_row), _p(w1), _p(w3), _p(w2),
                                    _dt(w1), _p(out)), "expert")
        return out

    def forward_with_routing(self, x, idx, gate, w1, w3, w2):
        x, w1, w3, w2 = _c(x), _c(w1), _c(w3), _c(w2)
        idx = np.ascontiguousarray(idx, dtype=np.int32)
        gate = np.ascontiguousarray(gate, dtype=np.float64)
        T, d = x.shape
        n, d2, F = w1.shape
        K = idx.shape[1]
        assert d == d2 and idx.shape == (T, K) and gate.shape == (T, K)
        assert w1.dtype == w3.dtype == w2.dtype
        y = np.empty((T, d), np.float64)
        _check(self.L.oracle_forward_with_routing(T, d, F, n, K, _p(x), _dt(x), _p(idx), _p(gate),
                                                  _p(w1), _p(w3), _p(w2), _dt(w1), _p(y)),
               "forward_with_routing")
        return y

    def moe_forward(self, x, W_g, w1, w3, w2, K: int):
        x, W_g, w1, w3, w2 = _c(x), _c(W_g), _c(w1), _c(w3), _c(w2)
        T, d = x.shape
        n, d2, F = w1.shape
        assert d == d2 and W_g.shape == (d, n)
        assert w1.dtype == w3.dtype == w2.dtype
        y = np.empty((T, d), np.float64)
        idx = np.empty((T, K), np.int32)
        gate = np.empty((T, K), np.float64)
        _check(self.L.oracle_moe_forward(T, d, F, n, K, _p(x), _dt(x), _p(W_g), _dt(W_g),
                                         _p(w1), _p(w3), _p(w2), _dt(w1), _p(y), _p(idx), _p(gate)),
               "moe_forward")
        return y, idx, gate

    def dispatch(self, idx, n: int):
        idx = np.ascontiguousarray(idx, dtype=np.int32)
        T, K = idx.shape
        counts = np.empty(n, np.int64)
        offsets = np.empty(n + 1, np.int64)
        row_token = np.empty(T * K, np.int64)
        token_row = np.empty(T * K, np.int64)
        _check(self.L.oracle_dispatch(T, n, K, _p(idx), _p(counts), _p(offsets), _p(row_token),
                                      _p(token_row)), "dispatch")
        return counts, offsets, row_token, token_row.reshape(T, K)


    def router_stats(self, x, W_g, idx, alpha: float):
        """-> f [n], P [n], aux (the load-balancing statistics of the routing idx)."""
        x, W_g = _c(x), _c(W_g)
        idx = np.ascontiguousarray(idx, dtype=np.int32)
        T, d = x.shape
        n = W_g.shape[1]
        K = idx.shape[1]
        f = np.empty(n, np.float64)
        P = np.empty(n, np.float64)
        aux = np.empty(1, np.float64)
        _check(self.L.oracle_router_stats(T, d, n, K, _p(x), _dt(x), _p(W_g), _dt(W_g), _p(idx),
                                          float(alpha), _p(f), _p(P), _p(aux)), "router_stats")
        return f, P, float(aux[0])

    def dispatch_capacity(self, idx, n: int, capacity: int):
        idx = np.ascontiguousarray(idx, dtype=np.int32)
        T, K = idx.shape
        counts = np.empty(n, np.int64)
        offsets = np.empty(n + 1, np.int64)
        row_token = np.full(max(1, T * K), -1, np.int64)
        token_row = np.empty(max(1, T * K), np.int64)
        _check(self.L.oracle_dispatch_capacity(T, n, K, _p(idx), int(capacity), _p(counts),
                                               _p(offsets), _p(row_token), _p(token_row)),
               "dispatch_capacity")
        return counts, offsets, row_token[:T * K], token_row[:T * K].reshape(T, K)


    def expert_choice(self, x, W_g, w1, w3, w2, C: int):
        """-> y [T,d], sel_token [n,C] (ascending tokens), sel_gate [n,C]."""
        x, W_g, w1, w3, w2 = _c(x), _c(W_g), _c(w1), _c(w3), _c(w2)
        T, d = x.shape
        n, d2, F = w1.shape
        assert d == d2 and W_g.shape == (d, n)
        y = np.empty((T, d), np.float64)
        sel = np.empty((n, C), np.int64)
        gate = np.empty((n, C), np.float64)
        _check(self.L.oracle_expert_choice(T, d, F, n, int(C), _p(x), _dt(x), _p(W_g), _dt(W_g),
                                           _p(w1), _p(w3), _p(w2), _dt(w1), _p(y), _p(sel), _p(gate)),
               "expert_choice")
        return y, sel, gate


    def e4m3_decode(self, code: int) -> float:
        return float(self.L.oracle_e4m3_decode(int(code)))

    def e4m3_encode(self, v: float) -> int:
        return int(self.L.oracle_e4m3_encode(float(v)))

    def quantize_weights_e4m3(self, w):
        """w [n][rows][cols] -> codes uint8 [n][rows][cols], scales fp32 [n][cols]."""
        w = _c(w)
        n, rows, cols = w.shape
        codes = np.empty((n, rows, cols), np.uint8)
        scales = np.empty((n, cols), np.float32)
        _check(self.L.oracle_quantize_weights_e4m3(n, rows, cols, _p(w), _dt(w), _p(codes), _p(scales)),
               "quantize_weights_e4m3")
        return codes, scales

    def e2m1_decode(self, code: int) -> float:
        return float(self.L.oracle_e2m1_decode(int(code)))

    def e2m1_encode(self, v: float) -> int:
        return int(self.L.oracle_e2m1_encode(float(v)))

    def quantize_weights_fp4(self, w):
        """w [n][rows][cols] -> codes uint8 [n][rows][cols/2] (column 2j in the low
        nibble of byte j), block scales uint8 E4M3 codes [n][rows/16][cols],
        tensor scales fp32 [n]."""
        w = _c(w)
        n, rows, cols = w.shape
        codes = np.empty((n, rows, cols // 2), np.uint8)
        bscale = np.empty((n, rows // 16, cols), np.uint8)
        tscale = np.empty(n, np.float32)
        _check(self.L.oracle_quantize_weights_fp4(n, rows, cols, _p(w), _dt(w), _p(codes), _p(bscale),
                                                  _p(tscale)), "quantize_weights_fp4")
        return codes, bscale, tscale

    def dequantize_fp4(self, codes, bscale, tscale):
        codes = np.ascontiguousarray(codes, dtype=np.uint8)
        bscale = np.ascontiguousarray(bscale, dtype=np.uint8)
        tscale = np.ascontiguousarray(tscale, dtype=np.float32)
        n, rows, half = codes.shape
        w = np.empty((n, rows, 2 * half), np.float64)
        _check(self.L.oracle_dequantize_fp4(n, rows, 2 * half, _p(codes), _p(bscale), _p(tscale), _p(w)),
               "dequantize_fp4")
        return w

    def forward_fp4(self, x, idx, gate, w1, w3, w2):
        """The layer of the dequantised 4-bit weights; w1, w3, w2 are (codes,
        block scales, matrix scales) triples of quantize_weights_fp4."""
        x = _c(x)
        idx = np.ascontiguousarray(idx, dtype=np.int32)
        gate = np.ascontiguousarray(gate, dtype=np.float64)
        T, d = x.shape
        n, d2, half = w1[0].shape
        F = 2 * half
        K = idx.shape[1]
        parts = []
        for c, b, t in (w1, w3, w2):
            parts += [np.ascontiguousarray(c, dtype=np.uint8), np.ascontiguousarray(b, dtype=np.uint8),
                      np.ascontiguousarray(t, dtype=np.float32)]
        y = np.empty((T, d), np.float64)
        _check(self.L.oracle_forward_fp4(T, d, F, n, K, _p(x), _dt(x), _p(idx), _p(gate), *[_p(a) for a in parts],
                                         _p(y)), "forward_fp4")
        return y

    def quantize_rows_fp4(self, x):
        """x [T][d] -> codes uint8 [T][d/2] (element 2j in the low nibble of
        byte j), block scales uint8 E4M3 codes [T][d/16], row scales fp32 [T]."""
        x = _c(x)
        T, d = x.shape
        codes = np.empty((T, d // 2), np.uint8)
        bscale = np.empty((T, d // 16), np.uint8)
        rscale = np.empty(T, np.float32)
        _check(self.L.oracle_quantize_rows_fp4(T, d, _p(x), _dt(x), _p(codes), _p(bscale), _p(rscale)),
               "quantize_rows_fp4")
        return codes, bscale, rscale

    def forward_w4a4(self, x, idx, gate, w1, w3, w2):
        """The layer with 4-bit weights (triples of quantize_weights_fp4) and
        4-bit activations (x rows and hidden rows quantised per row)."""
        x = _c(x)
        idx = np.ascontiguousarray(idx, dtype=np.int32)
        gate = np.ascontiguousarray(gate, dtype=np.float64)
        T, d = x.shape
        n, d2, half = w1[0].shape
        F = 2 * half
        K = idx.shape[1]
        parts = []
        for c, b, t in (w1, w3, w2):
            parts += [np.ascontiguousarray(c, dtype=np.uint8), np.ascontiguousarray(b, dtype=np.uint8),
                      np.ascontiguousarray(t, dtype=np.float32)]
        y = np.empty((T, d), np.float64)
        _check(self.L.oracle_forward_w4a4(T, d, F, n, K, _p(x), _dt(x), _p(idx), _p(gate), *[_p(a) for a in parts],
                                          _p(y)), "forward_w4a4")
        return y

    def forward_e4m3(self, x, idx, gate, q1, s1, q3, s3, q2, s2):
        x = _c(x)
        idx = np.ascontiguousarray(idx, dtype=np.int32)
        gate = np.ascontiguousarray(gate, dtype=np.float64)
        q1, q3, q2 = (np.ascontiguousarray(a, dtype=np.uint8) for a in (q1, q3, q2))
        s1, s3, s2 = (np.ascontiguousarray(a, dtype=np.float32) for a in (s1, s3, s2))
        T, d = x.shape
        n, d2, F = q1.shape
        K = idx.shape[1]
        y = np.empty((T, d), np.float64)
        _check(self.L.oracle_forward_e4m3(T, d, F, n, K, _p(x), _dt(x), _p(idx), _p(gate), _p(q1), _p(s1),
                                          _p(q3), _p(s3), _p(q2), _p(s2), _p(y)), "forward_e4m3")
        return y


_default = None


def default() -> Oracle:
    global _default
    if _default is None:
        _default = Oracle(build())
    return _default


def num_threads() -> int:
    return default().num_threads()


def set_num_threads(n: int) -> None:
    default().set_num_threads(n)


def silu(z: float) -> float:
    return default().silu(z)


def router(x, W_g, K: int):
    return default().router(x, W_g, K)


def gates_to_bf16(gate):
    return default().gates_to_bf16(gate)


def routing_alternatives(logits_row, K: int, gap: float, limit: int = 720):
    """Every top-K routing of one token that moving each logit by less than
    about `gap` can produce, the oracle's own routing first.

    Experts are ranked by (logit descending, index ascending), as the router
    ranks them.  Neighbours in that ranking whose logits differ by less than
    `gap` form a run; the experts of a run can come out of a lower-precision
    ranking in any order.  The alternatives are all routings in which the
    positions [0, K) that a run covers are filled by an ordered choice of
    that run's experts.  The gates of each are the softmax over its K chosen
    logits, listed with their experts: the gate rule of the layer equation
    ("Mixtral of Experts" section 2.1, softmax over the Top-K logits; Part 3,
    Step 3 of "Mixture of Experts: Why Mixtral Only Wakes Up Two
    Specialists").  -> list of (idx [K] int32, gate [K] float64)."""
    import itertools
    L = np.asarray(logits_row, np.float64)
    n = L.size
    order = sorted(range(n), key=lambda e: (-L[e], e))
    runs = []                      # (first position, last position) of each run
    a = 0
    for p in range(1, n + 1):
        if p == n or L[order[p - 1]] - L[order[p]] >= gap:
            runs.append((a, p - 1))
            a = p
    choices = []                   # per run meeting [0, K): its possible fillings
    for a, b in runs:
        if a >= K:
            break
        members = order[a:b + 1]
        m = min(b, K - 1) - a + 1
        choices.append(list(itertools.permutations(members, m)))
    out = []
    for combo in itertools.product(*choices):
        sel = [e for part in combo for e in part]
        z = L[sel]
        g = np.exp(z - z.max())
        out.append((np.array(sel, np.int32), g / g.sum()))
        if len(out) >= limit:
            break
    return out


def expert(x_row, w1, w3, w2, e: int):
    return default().expert(x_row, w1, w3, w2, e)


def forward_with_routing(x, idx, gate, w1, w3, w2):
    return default().forward_with_routing(x, idx, gate, w1, w3, w2)


def moe_forward(x, W_g, w1, w3, w2, K: int):
    return default().moe_forward(x, W_g, w1, w3, w2, K)


def dispatch(idx, n: int):
    return default().dispatch(idx, n)


def router_stats(x, W_g, idx, alpha: float):
    return default().router_stats(x, W_g, idx, alpha)


def dispatch_capacity(idx, n: int, capacity: int):
    return default().dispatch_capacity(idx, n, capacity)


def expert_choice(x, W_g, w1, w3, w2, C: int):
    return default().expert_choice(x, W_g, w1, w3, w2, C)


def e4m3_decode(code: int) -> float:
    return default().e4m3_decode(code)


def e4m3_encode(v: float) -> int:
    return default().e4m3_encode(v)


def quantize_weights_e4m3(w):
    return default().quantize_weights_e4m3(w)


def forward_e4m3(x, idx, gate, q1, s1, q3, s3, q2, s2):
    return default().forward_e4m3(x, idx, gate, q1, s1, q3, s3, q2, s2)


def e2m1_decode(code: int) -> float:
    return default().e2m1_decode(code)


def e2m1_encode(v: float) -> int:
    return default().e2m1_encode(v)


def quantize_weights_fp4(w):
    return default().quantize_weights_fp4(w)


def dequantize_fp4(codes, bscale, tscale):
    return default().dequantize_fp4(codes, bscale, tscale)


def forward_fp4(x, idx, gate, w1, w3, w2):
    return default().forward_fp4(x, idx, gate, w1, w3, w2)


def quantize_rows_fp4(x):
    return default().quantize_rows_fp4(x)


def forward_w4a4(x, idx, gate, w1, w3, w2):
    return default().forward_w4a4(x, idx, gate, w1, w3, w2)
