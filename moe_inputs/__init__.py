"""Seeded synthetic inputs for the sparse MoE layer (shared by the oracle tests,
the CUDA parity tests and the benchmark).

This module only draws and stores numbers.  It holds none of the layer's
arithmetic: no router, no top-K, no softmax, no expert FFN.

Recipe (all configs):
  * every tensor is drawn as float32 N(0, std^2) from its own PCG64 streams,
    one stream per (seed, tensor id, chunk of CHUNK elements), spawned with
    numpy's SeedSequence; chunks are independent, so they are drawn in
    parallel and the result does not depend on the thread count;
  * tensor ids: x = 0, W_g = 1, w1 = 2, w3 = 3, w2 = 4;
  * std: x 1; W_g and w1, w3 1/sqrt(d) (fan-in d); w2 1/sqrt(ffn) (fan-in ffn);
  * for bf16 configs x, w1, w3, w2 are rounded to bf16 (round to nearest even)
    and stored as uint16 bit patterns; W_g is always float32 (fp32 router);
  * the skewed config adds a constant input channel x[:, d-1] = 1 and gives
    expert 0 a logit offset of +2 sigma_L and expert n-1 one of -2 sigma_L
    through W_g[d-1, :], where sigma_L = 1 is the logit standard deviation
    that x ~ N(0,1), W_g ~ N(0,1/d) give.

Layouts (row-major): x[T][d], W_g[d][n], w1[n][d][ffn], w3[n][d][ffn],
w2[n][ffn][d].
"""
from __future__ import annotations

import dataclasses
import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np

CHUNK = 1 << 22  # elements per independent random stream

TENSOR_IDS = {"x": 0, "W_g": 1, "w1": 2, "w3": 3, "w2": 4}


@dataclasses.dataclass(frozen=True)
class LayerConfig:
    name: str
    T: int          # tokens
    d: int          # model dim
    ffn: int        # expert hidden dim
    n: int          # experts
    K: int          # experts per token
    dtype: str      # "f32" or "bf16": dtype of x, w1, w3, w2 and y
    skew: bool = False

    @property
    def R(self) -> int:
        return self.T * self.K

    def active_flops(self) -> float:
        """6*T*K*d*ffn for the experts plus 2*T*d*n for the router."""
        return 6.0 * self.T * self.K * self.d * self.ffn + 2.0 * self.T * self.d * self.n

    def expert_bytes(self) -> int:
        """Bytes of one expert's three weight matrices."""
        return 3 * self.d * self.ffn * (4 if self.dtype == "f32" else 2)


# The five workloads: a tiny fp32 case, Mixtral-shape decode / prefill /
# skewed prefill, and a many-expert layer.
CONFIGS = {
    "tiny_fp32": LayerConfig("tiny_fp32", T=64, d=128, ffn=256, n=8, K=2, dtype="f32"),
    "decode": LayerConfig("decode", T=32, d=4096, ffn=14336, n=8, K=2, dtype="bf16"),
    "prefill": LayerConfig("prefill", T=4096, d=4096, ffn=14336, n=8, K=2, dtype="bf16"),
    "skew_prefill": LayerConfig("skew_prefill", T=16384, d=4096, ffn=14336, n=8, K=2,
                                dtype="bf16", skew=True),
    "many_expert": LayerConfig("many_expert", T=8192, d=2048, ffn=768, n=128, K=2, dtype="bf16"),
}


def _threads() -> int:
    return max(1, min(16, os.cpu_count() or 1))


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round float32 to bf16 (nearest, ties to even); return the uint16 bit patterns."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)
    r = (u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)
    return r.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Widen bf16 bit patterns to float32 exactly."""
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def _draw(seed: int, tensor: str, shape, std: float, to_bf16: bool) -> np.ndarray:
    total = int(np.prod(shape))
    out = np.empty(total, dtype=np.uint16 if to_bf16 else np.float32)
    nchunk = (total + CHUNK - 1) // CHUNK
    tid = TENSOR_IDS[tensor]

    def one(c: int) -> None:
        lo, hi = c * CHUNK, min(total, (c + 1) * CHUNK)
        g = np.random.Generator(np.random.PCG64(np.random.SeedSequence(seed, spawn_key=(tid, c))))
        v = g.standard_normal(hi - lo, dtype=np.float32)
        if std != 1.0:
            v *= np.float32(std)
        out[lo:hi] = f32_to_bf16_bits(v) if to_bf16 else v

    if nchunk == 1:
        one(0)
    else:
        with ThreadPoolExecutor(_threads()) as ex:
            list(ex.map(one, range(nchunk)))
    return out.reshape(shape)


def make_layer(cfg: LayerConfig, seed: int = 0, only=None) -> dict:
    """Draw x, W_g, w1, w3, w2 for `cfg`.  `only` limits which tensors are drawn."""
    bf = cfg.dtype == "bf16"
    T, d, F, n = cfg.T, cfg.d, cfg.ffn, cfg.n
    want = set(only) if only is not None else set(TENSOR_IDS)
    out = {}
    if "x" in want:
        x = _draw(seed, "x", (T, d), 1.0, False)
        if cfg.skew:
            x[:, d - 1] = 1.0
        out["x"] = f32_to_bf16_bits(x) if bf else x
    if "W_g" in want:
        wg = _draw(seed, "W_g", (d, n), 1.0 / np.sqrt(d), False)
        if cfg.skew:
            sigma_l = 1.0
            wg[d - 1, :] = 0.0
            wg[d - 1, 0] = 2.0 * sigma_l
            wg[d - 1, n - 1] = -2.0 * sigma_l
        out["W_g"] = wg
    if "w1" in want:
        out["w1"] = _draw(seed, "w1", (n, d, F), 1.0 / np.sqrt(d), bf)
    if "w3" in want:
        out["w3"] = _draw(seed, "w3", (n, d, F), 1.0 / np.sqrt(d), bf)
    if "w2" in want:
        out["w2"] = _draw(seed, "w2", (n, F, d), 1.0 / np.sqrt(F), bf)
    return out


def custom_config(name="custom", T=64, d=128, ffn=256, n=8, K=2, dtype="bf16", skew=False) -> LayerConfig:
    return LayerConfig(name, T=T, d=d, ffn=ffn, n=n, K=K, dtype=dtype, skew=skew)


def as_f32(a: np.ndarray) -> np.ndarray:
    """float32 view of a stored tensor (bf16 bits widened exactly)."""
    return bf16_bits_to_f32(a) if a.dtype == np.uint16 else np.asarray(a, dtype=np.float32)
