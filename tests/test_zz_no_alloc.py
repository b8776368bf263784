"""i8_linear_forward_noalloc: the forward for callers that cannot allocate device memory
(a plugin whose host application owns every device allocation and lends it no scratch, or
a serving loop that must not call cudaMalloc/cudaFree because those can synchronise the
device).  It takes no workspace and uses the library's fixed 32 MiB device array instead.

The check: through the C ABI, two calls in a row of the no-allocation entry point give
bit for bit the output of i8_linear_forward with a caller workspace (the same kernels on
the same inputs), and that output is within the tests' fp16 tolerance of the oracle, on
the decode path and on the tcgen05 GEMM path; prefill, decode and prefill calls in turn
share the array without one call's leftovers reaching the next one's output; a size whose
workspace would exceed 32 MiB is refused before anything runs.  This file sorts last so
that a run which stops at the first failure has already run every other test; it also
passes alone.
"""
import ctypes
import math

import numpy as np
import pytest
import torch

from bit_matmul_decomposition_b200 import abi, synth
from oracle import oracle as O

pytestmark = pytest.mark.gpu

LIMIT = 32 << 20


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    abi.load()
    yield
    torch.cuda.synchronize()


def _f16(a):
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.float16).cuda()


def _bits(C):
    return C.cpu().view(torch.int16).numpy()


def _within_tolerance(C, C_ref):
    """Per row: max|C - C_ref| <= 2^-9 max|C_ref| + 1e-3, C_ref the oracle's fp64 output."""
    C = C.float().cpu().numpy().astype(np.float64)
    err = np.abs(C - C_ref).max(axis=1)
    allowed = 2.0 ** -9 * np.abs(C_ref).max(axis=1) + 1e-3
    return bool(np.isfinite(C).all() and (err <= allowed).all())


def _layer(T, K, N, cols, thr):
    w = synth.Workload("noalloc", T, K, N, seed=T + N,
                       fixed_cols=tuple(cols) if cols else None)
    X, W, b = synth.make_x(w), synth.make_w(w), synth.make_bias(w)
    CB = torch.empty((N, K), dtype=torch.int8, device="cuda")
    SCB = torch.empty((N,), dtype=torch.float32, device="cuda")
    abi.i8_quantize_weight(_f16(W), CB, SCB)
    CBr, SCBr = O.quantize_weight(W)
    C_or = O.linear_forward(X, CBr, SCBr, b, thr)["C"]
    return _f16(X), CB, SCB, _f16(b), C_or


def _noalloc_call(lib, X, CB, SCB, b, thr, C):
    T, K = X.shape
    N = CB.shape[0]
    return lib.i8_linear_forward_noalloc(
        X.data_ptr(), T, K, CB.data_ptr(), SCB.data_ptr(),
        None if b is None else b.data_ptr(), N, ctypes.c_float(thr), C.data_ptr(),
        torch.cuda.current_stream().cuda_stream)


@pytest.mark.parametrize("T,K,N,cols,thr", [
    (16, 1024, 2048, (5, 700), 6.0),        # decode GEMV path
    (256, 1024, 1024, (3, 64, 900), 6.0),   # tcgen05 GEMM path with outliers
    (200, 512, 700, (), math.inf),          # GEMM path, no outliers
])
def test_noalloc_matches_workspace_forward(T, K, N, cols, thr):
    lib = abi.load()
    assert lib.i8_linear_workspace_size(T, N, K) <= LIMIT
    X, CB, SCB, b, C_or = _layer(T, K, N, cols, thr)
    ws = torch.empty((lib.i8_linear_workspace_size(T, N, K),), dtype=torch.uint8, device="cuda")
    C_ref = torch.empty((T, N), dtype=torch.float16, device="cuda")
    abi.i8_linear_forward(X, CB, SCB, b, thr, C_ref, ws)
    assert abi.i8_sync_status() == 0
    assert _within_tolerance(C_ref, C_or)
    for _ in range(2):                       # two calls in a row share the fixed array
        C = torch.full((T, N), float("nan"), dtype=torch.float16, device="cuda")
        assert _noalloc_call(lib, X, CB, SCB, b, thr, C) == 0
        assert abi.i8_sync_status() == 0
        assert np.array_equal(_bits(C), _bits(C_ref))
        assert _within_tolerance(C, C_or)


def test_noalloc_prefill_decode_prefill_share_the_array():
    """A prefill call at threshold 0 fills the array with its index list 0, 1, 2, ...
    where a decode call keeps its counters; each call must still match its own workspace
    forward bit for bit."""
    lib = abi.load()
    K, N = 8192, 96
    calls = [(64, (), 0.0), (8, (5, 4000), 6.0), (64, (9,), 6.0), (16, (1, 8191), 6.0),
             (300, (), 0.0), (1, (77,), 6.0)]
    for i, (T, cols, thr) in enumerate(calls * 2):
        assert lib.i8_linear_workspace_size(T, N, K) <= LIMIT
        X, CB, SCB, b, C_or = _layer(T, K, N, cols, thr)
        ws = torch.empty((lib.i8_linear_workspace_size(T, N, K),), dtype=torch.uint8,
                         device="cuda")
        C_ref = torch.empty((T, N), dtype=torch.float16, device="cuda")
        abi.i8_linear_forward(X, CB, SCB, b, thr, C_ref, ws)
        C = torch.full((T, N), float("nan"), dtype=torch.float16, device="cuda")
        assert _noalloc_call(lib, X, CB, SCB, b, thr, C) == 0
        assert abi.i8_sync_status() == 0
        assert np.array_equal(_bits(C), _bits(C_ref)), (i, T, thr)
        assert _within_tolerance(C, C_or), (i, T, thr)


def test_noalloc_refuses_sizes_beyond_its_array():
    lib = abi.load()
    T, K, N = 2048, 4096, 16384              # needs far more than 32 MiB of workspace
    assert lib.i8_linear_workspace_size(T, N, K) > LIMIT
    X = torch.zeros((T, K), dtype=torch.float16, device="cuda")
    CB = torch.zeros((N, K), dtype=torch.int8, device="cuda")
    SCB = torch.ones((N,), dtype=torch.float32, device="cuda")
    C = torch.zeros((T, N), dtype=torch.float16, device="cuda")
    assert _noalloc_call(lib, X, CB, SCB, None, 6.0, C) == 1   # I8_ERR_INVALID_ARG
    assert abi.i8_sync_status() == 0
    assert not C.any()
