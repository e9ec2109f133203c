"""Seeded synthetic workloads shared by the tests, the smoke check and the benchmark.

This module holds the input recipe only: it draws q, k, v (and dO, decode states)
from numpy generators and rounds them to the mode's dtype.  It contains none of
SLAY's arithmetic (no phi, no quadrature, no contraction) and imports neither the
CUDA library nor the oracle.

Recipe (per workload): q, k, v iid N(0, 1) in fp64; the vision-shaped workload adds
0.5 * mu_b to q and k, with mu_b ~ N(0, I_D) drawn once per batch element and shared
by q and k, all heads and all tokens (correlated angles); then q and k are scaled to
unit L2 norm per row, as the workloads prescribe, and every tensor is rounded to the
mode's dtype (bf16 by round-to-nearest-even).  Each tensor has its own numpy stream
seeded by (data_seed, tensor id), so adding a tensor never shifts another one.
"""
from dataclasses import dataclass, field
from typing import Tuple

import numpy as np

SKETCH_SEED = 1234
EPS = 1e-6

_STREAM = {"q": 0, "k": 1, "v": 2, "dout": 3, "mu": 4, "S": 5, "z": 6,
           "scale_q": 7, "scale_k": 8, "dphi": 9}


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    L: int
    D: int = 64
    Dv: int = 64
    R: int = 4
    m: int = 64
    dtype: str = "bf16"          # "f32" or "bf16": input/output dtype of the path
    causal: bool = True
    correlated: bool = False
    data_seed: int = 0
    sketch_seed: int = SKETCH_SEED
    eps: float = EPS
    modes: Tuple[str, ...] = field(default=("causal",))

    @property
    def F(self) -> int:
        return self.R * self.m

    @property
    def tokens(self) -> int:
        return self.B * self.L


# The five workloads of the benchmark plan, by what they are.
TINY = Workload("tiny_B1H1L256_F32_fp32", B=1, H=1, L=256, R=2, m=16, dtype="f32",
                data_seed=0, modes=("causal", "bidir"))
CAUSAL_2K = Workload("causal_B4H8L2048_F256_bf16", B=4, H=8, L=2048, R=4, m=64,
                     data_seed=1, modes=("causal",))
CAUSAL_16K = Workload("causal_B1H16L16384_F256_bf16", B=1, H=16, L=16384, R=4, m=64,
                      data_seed=2, modes=("causal",))
BIDIR_VISION = Workload("bidir_B32H12L1024_F256_bf16_corr", B=32, H=12, L=1024, R=4, m=64,
                        causal=False, correlated=True, data_seed=3, modes=("bidir",))
FWDBWD_8K = Workload("fwdbwd_B2H16L8192_F512_bf16", B=2, H=16, L=8192, R=8, m=64,
                     data_seed=4, modes=("causal", "bwd"))
# Decode: batch 256 x 16 heads, one new token each, state S [F, Dv] fp32 per (b, h).
DECODE = Workload("decode_Bt256H16_F512_bf16", B=256, H=16, L=1, R=8, m=64,
                  data_seed=5, modes=("decode",))

ALL = [TINY, CAUSAL_2K, CAUSAL_16K, BIDIR_VISION, FWDBWD_8K, DECODE]


def _rng(seed: int, tensor: str) -> np.random.Generator:
    return np.random.default_rng([int(seed), _STREAM[tensor]])


def round_bf16(x: np.ndarray) -> np.ndarray:
    """fp32 values rounded to the nearest bf16 (ties to even), returned as fp32."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    b = x.view(np.uint32).astype(np.uint64)
    b = (b + 0x7FFF + ((b >> 16) & 1)) & 0xFFFF0000
    return b.astype(np.uint32).view(np.float32)


def to_dtype(x: np.ndarray, dtype: str) -> np.ndarray:
    """Round to the mode's dtype; the result is fp32 holding exactly representable values."""
    x32 = np.asarray(x, dtype=np.float32)
    if dtype == "f32":
        return np.ascontiguousarray(x32)
    if dtype == "bf16":
        return round_bf16(x32)
    raise ValueError(dtype)


def _unit_rows(x: np.ndarray) -> np.ndarray:
    n = np.sqrt(np.sum(x * x, axis=-1, keepdims=True))
    return x / np.maximum(n, 1e-300)


def gen_qkv(w: Workload, B=None, H=None, L=None):
    """q, k [B,H,L,D] (unit rows) and v [B,H,L,Dv], fp32 arrays in w.dtype's values."""
    B = w.B if B is None else B
    H = w.H if H is None else H
    L = w.L if L is None else L
    q = _rng(w.data_seed, "q").standard_normal((B, H, L, w.D))
    k = _rng(w.data_seed, "k").standard_normal((B, H, L, w.D))
    v = _rng(w.data_seed, "v").standard_normal((B, H, L, w.Dv))
    if w.correlated:
        mu = _rng(w.data_seed, "mu").standard_normal((B, 1, 1, w.D))
        q = q + 0.5 * mu
        k = k + 0.5 * mu
    q = _unit_rows(q)
    k = _unit_rows(k)
    return to_dtype(q, w.dtype), to_dtype(k, w.dtype), to_dtype(v, w.dtype)


def gen_dout(w: Workload, B=None, H=None, L=None):
    B = w.B if B is None else B
    H = w.H if H is None else H
    L = w.L if L is None else L
    g = _rng(w.data_seed, "dout").standard_normal((B, H, L, w.Dv))
    return to_dtype(g, w.dtype)


def gen_dphi(w: Workload, n: int):
    """An upstream gradient for n rows of features: [n, F] iid N(0, 1), in w.dtype's values."""
    g = _rng(w.data_seed, "dphi").standard_normal((n, w.F))
    return to_dtype(g, w.dtype)


def gen_decode(w: Workload, Bt=None, H=None):
    """One new token per (b,h): q,k [Bt,H,D], v [Bt,H,Dv] in w.dtype's values, and a
    state S [Bt,H,F,Dv] ~ N(0,1), z [Bt,H,F] ~ 1 + U(0,1), both fp32."""
    Bt = w.B if Bt is None else Bt
    H = w.H if H is None else H
    q = _rng(w.data_seed, "q").standard_normal((Bt, H, w.D))
    k = _rng(w.data_seed, "k").standard_normal((Bt, H, w.D))
    v = _rng(w.data_seed, "v").standard_normal((Bt, H, w.Dv))
    q = _unit_rows(q)
    k = _unit_rows(k)
    S = _rng(w.data_seed, "S").standard_normal((Bt, H, w.F, w.Dv), dtype=np.float32)
    z = (1.0 + _rng(w.data_seed, "z").random((Bt, H, w.F), dtype=np.float32)).astype(np.float32)
    return (to_dtype(q, w.dtype), to_dtype(k, w.dtype), to_dtype(v, w.dtype),
            np.ascontiguousarray(S), np.ascontiguousarray(z))


def row_scales(w: Workload, shape, tensor: str, extremes=(6.0, -6.0, 10.0, -10.0)):
    """Per-row factors 10^e for a tensor whose rows are indexed by `shape` (all but the
    last axis): e ~ U(-3, 3), and the first len(extremes) rows of a seeded permutation get
    e = extremes[i] exactly (rows far from unit length, inside the range the library
    states it supports)."""
    rng = _rng(w.data_seed, "scale_" + tensor)
    e = rng.uniform(-3.0, 3.0, size=shape)
    flat = e.reshape(-1)
    pick = rng.permutation(flat.size)[:len(extremes)]
    for i, r in enumerate(pick):
        flat[r] = extremes[i]
    return np.power(10.0, e)


def scale_rows(w: Workload, x: np.ndarray, tensor: str, extremes=(6.0, -6.0, 10.0, -10.0)):
    """x with every row multiplied by row_scales(...), rounded to w.dtype: the same values
    feed the library and the oracle, so only the library's normalisation is exercised."""
    f = row_scales(w, x.shape[:-1], tensor, extremes)
    return to_dtype(np.asarray(x, np.float64) * f[..., None], w.dtype)


def tile_border_rows(L: int, tile: int = 128):
    """Sorted row indices: the first and the last row of every `tile`-row block (every
    segment the tensor-core kernels cut a sequence into starts and ends on such rows)."""
    s = set()
    for t0 in range(0, L, tile):
        s.add(t0)
        s.add(min(t0 + tile, L) - 1)
    return np.array(sorted(s), dtype=np.int64)


def sample_rows(L: int, n: int, seed: int = 7, chunk: int = 64):
    """Sorted row indices: the ends, chunk and tile borders, and n random rows."""
    rng = np.random.default_rng([seed, L])
    fixed = {0, 1, L - 1, L - 2}
    for c in (chunk - 1, chunk, 2 * chunk - 1, 2 * chunk, L // 2, L // 2 - 1):
        if 0 <= c < L:
            fixed.add(c)
    extra = rng.choice(L, size=min(n, L), replace=False)
    return np.array(sorted(fixed | set(int(x) for x in extra)), dtype=np.int64)
