"""i8_linear_forward_noalloc: the forward for callers that cannot allocate device memory
(a plugin whose host application owns every device allocation and lends it no scratch, or
a serving loop that must not call cudaMalloc/cudaFree because those can synchronise the
device).  It takes no workspace and uses the library's fixed 32 MiB device array instead.

The check: through the C ABI, two calls in a row of the no-allocation entry point give
the same output as i8_linear_forward with a caller workspace, within the tests' fp16
tolerance, on the decode path and on the tcgen05 GEMM path; a size whose workspace would
exceed 32 MiB is refused before anything runs.  This file sorts last so that a run which
stops at the first failure has already run every other test; it also passes alone.
"""
import ctypes
import math

import numpy as np
import pytest
import torch

from bit_matmul_decomposition_b200 import abi, synth

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


def _within_tolerance(C, C_ref):
    C = C.float().cpu().numpy().astype(np.float64)
    R = C_ref.float().cpu().numpy().astype(np.float64)
    err = np.abs(C - R).max(axis=1)
    allowed = 2.0 ** -9 * np.abs(R).max(axis=1) + 1e-3
    return bool(np.isfinite(C).all() and (err <= allowed).all())


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
    w = synth.Workload("noalloc", T, K, N, seed=T + N,
                       fixed_cols=tuple(cols) if cols else None)
    X, W, b = _f16(synth.make_x(w)), _f16(synth.make_w(w)), _f16(synth.make_bias(w))
    CB = torch.empty((N, K), dtype=torch.int8, device="cuda")
    SCB = torch.empty((N,), dtype=torch.float32, device="cuda")
    abi.i8_quantize_weight(W, CB, SCB)
    ws = torch.empty((lib.i8_linear_workspace_size(T, N, K),), dtype=torch.uint8, device="cuda")
    C_ref = torch.empty((T, N), dtype=torch.float16, device="cuda")
    abi.i8_linear_forward(X, CB, SCB, b, thr, C_ref, ws)
    for _ in range(2):                       # two calls in a row share the fixed array
        C = torch.full((T, N), float("nan"), dtype=torch.float16, device="cuda")
        assert _noalloc_call(lib, X, CB, SCB, b, thr, C) == 0
        assert abi.i8_sync_status() == 0
        assert _within_tolerance(C, C_ref)


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
