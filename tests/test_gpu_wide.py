"""The 256 x 512 tile GEMM (chosen for K >= 8192 when there are at least four tiles per
co-resident cluster pair) against the oracle, at sizes that select it and leave ragged
edges on every dimension: T = 3996 (the last 256-row tile has 156 rows), N = 9928 (the
last 512-column tile has 200 columns, so its second 256-column half is empty), K = 8192.

Each case compares every row and column of the four corner output tiles and a seeded
sample of rows x columns with the oracle (each output depends only on its own row of X
and its own output channel, so a sample is exact), per row within
    max|C - C_ref| <= 2^-9 * max_row|C_ref| + 1e-3,
and the whole output bit for bit with a second call (deterministic).  Outlier sets: none
(threshold +inf), 8 systematic columns, 80 columns (two 64-column chunks of fp16 MMAs),
and threshold 0 (every column in the fp16 product: 128 chunks).
"""
import math

import numpy as np
import pytest
import torch

from bit_matmul_decomposition_b200 import abi, synth
from oracle import oracle as O
from tests.gpu_util import check_output, dev, gpu_forward, gpu_quantize_weight, host, sync_ok

pytestmark = pytest.mark.gpu

T, K, N = 3996, 8192, 9928


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    abi.load()
    yield
    torch.cuda.empty_cache()


@pytest.fixture(scope="module")
def weights():
    w = synth.Workload("wide", T, K, N, seed=31)
    W, b = synth.make_w(w), synth.make_bias(w)
    CB, SCB = gpu_quantize_weight(dev(W))
    sync_ok()
    CBr, SCBr = O.quantize_weight(W)
    assert np.array_equal(host(CB), CBr)
    return CB, SCB, CBr, SCBr, b


def _edges(n, tile):
    return list(range(min(n, tile))) + list(range(max(0, n - tile), n))


def _sample(n, extra, count, seed):
    rng = np.random.Generator(np.random.PCG64(seed))
    s = set(int(i) for i in extra if 0 <= i < n)
    s.update(int(i) for i in rng.choice(n, size=min(n, count), replace=False))
    return np.array(sorted(s), np.int64)


def test_forward_kernel_query_names_the_wide_tiles():
    assert abi.i8_forward_kernel(T, N, K) == "i8_gemm_wide_kernel"
    assert abi.i8_forward_kernel(T, N, 4096) == "i8_gemm_tcgen05_kernel"   # K below 8192
    assert abi.i8_forward_kernel(300, 1000, K) == "i8_gemm_tcgen05_kernel"  # too few tiles
    assert abi.i8_forward_kernel(16, N, K) == "decode_kernel"


@pytest.mark.parametrize("n_cols,thr", [(0, math.inf), (8, 6.0), (80, 6.0), (0, 0.0)])
def test_wide_tiles_match_the_oracle(weights, n_cols, thr):
    CB, SCB, CBr, SCBr, b = weights
    w = synth.Workload("wide", T, K, N, seed=32 + n_cols, n_fixed=n_cols, threshold=thr)
    X = synth.make_x(w)
    X_d, b_d = dev(X), dev(b)
    C = gpu_forward(X_d, CB, SCB, b_d, thr)
    C2 = gpu_forward(X_d, CB, SCB, b_d, thr)
    sync_ok()
    assert torch.equal(C.view(torch.int16), C2.view(torch.int16))
    rows = _sample(T, _edges(T, 256), 24, seed=n_cols + 1)
    cols = _sample(N, _edges(N, 512) + [9727, 9728], 512, seed=n_cols + 2)
    Cs = host(C[torch.from_numpy(rows).cuda()][:, torch.from_numpy(cols).cuda()])
    r = O.linear_forward(X, CBr[cols], SCBr[cols], b[cols], thr, rows=rows)
    if thr == 6.0:
        assert r["n_o"] >= n_cols
    check_output(Cs, r["C"])
