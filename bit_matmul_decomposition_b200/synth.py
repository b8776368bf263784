"""Seeded synthetic inputs for the LLM.int8() decomposed linear layer.

This module holds random draws and fp16 casts only -- none of the method's arithmetic --
so that the CUDA path and the CPU oracle can be fed identical bytes.

Recipe (shared by every workload):
  * numpy ``Generator(PCG64)``; one child seed per tensor from ``SeedSequence(seed)``
    (child 0: hidden states X, child 1: weight W, child 2: bias, child 3: outlier layout);
    the weight is drawn in blocks of W_BLOCK rows, block i from the seed sequence with
    spawn key (1, i), so that any range of output channels (one GPU's shard of the layer)
    can be drawn on its own and equals the same rows of the whole weight;
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

import concurrent.futures
import dataclasses
import math
import os
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
                 threshold="inf" if math.isinf(self.threshold) else self.threshold)
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


W_BLOCK = 2048   # rows of the weight drawn from one generator


def _w_block_rng(seed: int, blk: int):
    return np.random.Generator(np.random.PCG64(
        np.random.SeedSequence(entropy=seed, spawn_key=(1, blk))))


def make_w(w: Workload, rows: Optional[tuple] = None) -> np.ndarray:
    """Weight W [N, K] fp16 in the nn.Linear [out, in] layout, or only its rows
    [rows[0], rows[1]) (bit for bit the same rows of the whole weight)."""
    r0, r1 = (0, w.N) if rows is None else (int(rows[0]), int(rows[1]))
    if not 0 <= r0 <= r1 <= w.N:
        raise ValueError("rows %r outside [0, %d]" % (rows, w.N))
    out = np.empty((r1 - r0, w.K), np.float16)

    def draw(blk):
        b0, b1 = blk * W_BLOCK, min(w.N, (blk + 1) * W_BLOCK)
        lo, hi = max(b0, r0), min(b1, r1)
        if lo == b0 and hi == b1:   # a whole block: straight into the output
            out[lo - r0:hi - r0] = _normal_fp16(_w_block_rng(w.seed, blk), (b1 - b0, w.K),
                                                w.w_sigma, chunk_rows=W_BLOCK)
        else:
            full = _normal_fp16(_w_block_rng(w.seed, blk), (b1 - b0, w.K), w.w_sigma,
                                chunk_rows=W_BLOCK)
            out[lo - r0:hi - r0] = full[lo - b0:hi - b0]

    blocks = range(r0 // W_BLOCK, (r1 + W_BLOCK - 1) // W_BLOCK)
    if len(blocks) <= 1:
        for blk in blocks:
            draw(blk)
    else:   # blocks are independent streams: draw them on several threads
        with concurrent.futures.ThreadPoolExecutor(min(len(blocks), os.cpu_count() or 1)) as ex:
            list(ex.map(draw, blocks))
    return out


def make_bias(w: Workload, rows: Optional[tuple] = None) -> Optional[np.ndarray]:
    """Bias [N] fp16 (or its entries [rows[0], rows[1])), None for a layer without."""
    if not w.bias:
        return None
    b = _normal_fp16(_children(w.seed)[2], (w.N,), w.b_sigma)
    return b if rows is None else b[int(rows[0]):int(rows[1])].copy()


def shard_rows(N: int, rank: int, world: int) -> tuple:
    """Output channels [r0, r1) of rank `rank` when an N-wide layer is split over `world`
    GPUs by output channel: contiguous blocks, sizes differing by at most one."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError("rank %d of %d" % (rank, world))
    return (N * rank) // world, (N * (rank + 1)) // world


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
