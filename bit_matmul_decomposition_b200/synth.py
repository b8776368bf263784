"""Seeded synthetic inputs for the LLM.int8() decomposed linear layer.

This module holds random draws and fp16 casts only -- none of the method's arithmetic --
so that the CUDA path and the CPU oracle can be fed identical bytes.

Recipe (shared by every workload):
  * numpy ``Generator(PCG64)``; one child seed per tensor from ``SeedSequence(seed)``
    (child 0: hidden states X, child 1: weight W, child 2: bias, child 3: outlier layout);
  * N(mu, sigma) is drawn in fp32 and cast to fp16 with round-to-nearest-even;
  * "+-U[a,b]" means magnitude U[a,b] with an independent random sign per entry;
  * fixed outlier columns are drawn without replacement from [0, K) and overwritten in
    every row (the systematic outlier features of the LLM.int8() summary: the same
    feature dims in every token);
  * random outlier entries (the non-systematic ones) are placed uniformly over the
    whole [T, K] matrix.

The workload shapes follow the pages' setting: OPT-6.7B / OPT-175B / BLOOM-176B layer
shapes, whose real weights are not available, stand in for the evaluated models.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional, Sequence

import numpy as np


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    T: int
    K: int
    N: int
    seed: int
    threshold: float = 6.0
    fixed_cols: Optional[Sequence[int]] = None   # explicit outlier columns
    n_fixed: int = 0                             # else: this many drawn columns
    fixed_mag: tuple = (8.0, 60.0)
    random_frac: float = 0.0                     # fraction of all entries made outliers
    random_mag: tuple = (6.0, 10.0)
    x_sigma: float = 1.0
    w_sigma: float = 0.02
    b_sigma: float = 0.02
    bias: bool = True

    def describe(self) -> dict:
        d = dict(workload=self.name, T=self.T, K=self.K, N=self.N, seed=self.seed,
                 threshold=self.threshold)
        if self.fixed_cols is not None:
            d["outlier_cols"] = list(self.fixed_cols)
        else:
            d["fixed_outlier_cols"] = self.n_fixed
        if self.random_frac:
            d["random_outlier_frac"] = self.random_frac
        return d


def tiny() -> Workload:
    """[16 tokens, K=64] x [64, 64]; columns 3 and 41 carry +-U[8,20] outliers; seed 0."""
    return Workload("tiny_16x64x64", 16, 64, 64, seed=0, fixed_cols=(3, 41),
                    fixed_mag=(8.0, 20.0))


def opt_ffn_up_prefill() -> Workload:
    """OPT-6.7B FFN up-projection prefill: X [2048, 4096], W [16384, 4096], 6 fixed cols."""
    return Workload("opt6.7b_ffn_up_prefill_2048x4096x16384", 2048, 4096, 16384, seed=1,
                    n_fixed=6)


def bloom_ffn_decode(T: int) -> Workload:
    """BLOOM-176B FFN decode: X [T, 14336], W [57344, 14336], 8 fixed cols; T in {1,8,16}."""
    return Workload("bloom176b_ffn_decode_%dx14336x57344" % T, T, 14336, 57344, seed=2,
                    n_fixed=8)


def bloom_qkv_prefill() -> Workload:
    """BLOOM-176B fused QKV prefill: X [4096, 14336], W [43008, 14336], 8 fixed cols
    plus 0.01% of all entries set to +-U[6,10]."""
    return Workload("bloom176b_qkv_prefill_4096x14336x43008", 4096, 14336, 43008, seed=3,
                    n_fixed=8, random_frac=1e-4)


def opt175b_sweep(n_cols: int, threshold: float) -> Workload:
    """OPT-175B outlier-density sweep: X [8192, 12288], W [49152, 12288];
    n_cols in {0, 8, 64, 256} planted columns; threshold in {6, +inf}."""
    tag = "inf" if math.isinf(threshold) else ("%g" % threshold)
    return Workload("opt175b_sweep_8192x12288x49152_cols%d_thr%s" % (n_cols, tag), 8192,
                    12288, 49152, seed=4, n_fixed=n_cols, threshold=threshold)


def _children(seed: int):
    return [np.random.Generator(np.random.PCG64(s))
            for s in np.random.SeedSequence(seed).spawn(4)]


def _normal_fp16(rng, shape, sigma, chunk_rows=2048) -> np.ndarray:
    out = np.empty(shape, np.float16)
    if len(shape) == 1:
        out[:] = (rng.standard_normal(shape[0], dtype=np.float32) * np.float32(sigma))
        return out
    rows = shape[0]
    for r0 in range(0, rows, chunk_rows):
        r1 = min(rows, r0 + chunk_rows)
        blk = rng.standard_normal((r1 - r0,) + tuple(shape[1:]), dtype=np.float32)
        if sigma != 1.0:
            blk *= np.float32(sigma)
        out[r0:r1] = blk
    return out


def _signed_uniform(rng, n, lo, hi) -> np.ndarray:
    mag = rng.uniform(lo, hi, size=n).astype(np.float32)
    sign = np.where(rng.integers(0, 2, size=n) == 0, -1.0, 1.0).astype(np.float32)
    return (mag * sign).astype(np.float16)


def outlier_columns(w: Workload) -> np.ndarray:
    """The planted fixed outlier columns of a workload (sorted)."""
    if w.fixed_cols is not None:
        return np.array(sorted(w.fixed_cols), np.int64)
    if w.n_fixed == 0:
        return np.zeros(0, np.int64)
    rng = _children(w.seed)[3]
    return np.sort(rng.choice(w.K, size=w.n_fixed, replace=False)).astype(np.int64)


def make_x(w: Workload, T: Optional[int] = None) -> np.ndarray:
    """Hidden states X [T, K] fp16 (T defaults to the workload's)."""
    T = w.T if T is None else T
    rng = _children(w.seed)[0]
    X = _normal_fp16(rng, (T, w.K), w.x_sigma)
    cols = outlier_columns(w)
    if cols.size:
        vals = _signed_uniform(rng, T * cols.size, *w.fixed_mag).reshape(T, cols.size)
        X[:, cols] = vals
    if w.random_frac > 0:
        n = int(round(w.random_frac * T * w.K))
        flat = rng.choice(T * w.K, size=n, replace=False)
        X.reshape(-1)[flat] = _signed_uniform(rng, n, *w.random_mag)
    return X


def make_w(w: Workload) -> np.ndarray:
    """Weight W [N, K] fp16 in the nn.Linear [out, in] layout."""
    return _normal_fp16(_children(w.seed)[1], (w.N, w.K), w.w_sigma)


def make_bias(w: Workload) -> Optional[np.ndarray]:
    if not w.bias:
        return None
    return _normal_fp16(_children(w.seed)[2], (w.N,), w.b_sigma)


def random_fp16(shape, seed: int, sigma: float = 1.0) -> np.ndarray:
    """Plain N(0, sigma) fp16 tensor for ad-hoc shapes (ragged and edge cases)."""
    return _normal_fp16(np.random.Generator(np.random.PCG64(seed)), tuple(shape), sigma)


def random_int8(shape, seed: int, lo: int = -127, hi: int = 127) -> np.ndarray:
    """Uniform int8 codes in [lo, hi] for integer-matmul cases."""
    rng = np.random.Generator(np.random.PCG64(seed))
    return rng.integers(lo, hi + 1, size=tuple(shape), dtype=np.int64).astype(np.int8)


def plant_columns(X: np.ndarray, cols, seed: int, mag=(8.0, 60.0)) -> np.ndarray:
    """Return a copy of X with the given columns overwritten by +-U[mag] in every row."""
    X = X.copy()
    cols = np.asarray(list(cols), np.int64)
    if cols.size:
        rng = np.random.Generator(np.random.PCG64(seed))
        X[:, cols] = _signed_uniform(rng, X.shape[0] * cols.size, *mag).reshape(
            X.shape[0], cols.size)
    return X
