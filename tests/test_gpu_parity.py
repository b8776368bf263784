"""CUDA path (through the C ABI) against the CPU oracle, on the same seeded inputs.

Bit-exact: outlier mask, index list and count; Xq and SCx; CB and SCB; the fp16 outlier
slice; the int32 accumulators.  Tolerance (fp16 output, per row):
    max|C - C_ref| <= 2^-9 * max_row|C_ref| + 1e-3.
Small cases span several tiles with ragged tails on every dimension; both the decode
path (T <= 16) and the tcgen05 GEMM path (T > 16) are covered.
"""
import math

import numpy as np
import pytest
import torch

from bit_matmul_decomposition_b200 import abi, synth
from oracle import oracle as O
from tests.gpu_util import (check_output, dev, gpu_forward, gpu_igemm, gpu_prepare,
                            gpu_quantize_act, gpu_quantize_weight, gpu_scan, host,
                            slice_to_matrix, sync_ok)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    abi.load()
    yield
    torch.cuda.synchronize()


def _case(T, K, N, seed, cols=(), n_fixed=0, random_frac=0.0, bias=True, b_sigma=0.02):
    w = synth.Workload("case", T, K, N, seed=seed,
                       fixed_cols=tuple(cols) if cols else None, n_fixed=n_fixed,
                       random_frac=random_frac, bias=bias, b_sigma=b_sigma)
    return w, synth.make_x(w), synth.make_w(w), synth.make_bias(w)


# ------------------------------------------------------------------ step 3
# The weight quantiser streams stages of R rows (R * K * 2 <= 32 KB, R a power of two, up
# to 256) through shared memory: warp per row for R >= 8, 8 / R warps per row below; rows
# longer than 64 KB take the one-CTA-per-row kernel.  The cases cover each R regime, a last
# stage holding fewer rows than R, fewer stages than SMs, many stages per CTA and the
# fallback.
@pytest.mark.parametrize("N,K", [(64, 64), (129, 80), (300, 4096), (17, 16400), (5, 16),
                                 (1000, 16), (4099, 64), (777, 4096), (2001, 2064),
                                 (150, 14336), (3, 32768), (2, 32784), (3000, 1040)])
def test_quantize_weight_bitexact(N, K):
    W = synth.random_fp16((N, K), seed=N * 7 + K, sigma=0.02)
    W[0, :] = 0  # an all-zero output channel
    CB, SCB = gpu_quantize_weight(dev(W))
    sync_ok()
    CBr, SCBr = O.quantize_weight(W)
    assert np.array_equal(host(CB), CBr)
    assert np.array_equal(host(SCB).view(np.uint32), SCBr.view(np.uint32))


# ------------------------------------------------------------------ steps 1 and 2
SCAN_CASES = [
    # T, K, cols, random_frac, threshold
    (16, 64, (3, 41), 0.0, 6.0),
    (300, 464, (0, 5, 200, 463), 0.003, 6.0),
    (1, 4096, (17,), 0.0, 6.0),
    (77, 208, (), 0.0, 2.5),
    (33, 96, (1,), 0.0, 0.0),
    (33, 96, (1,), 0.0, -1.0),
    (33, 96, (1, 2), 0.0, math.inf),
    (4100, 1040, (7, 1039), 1e-4, 6.0),
    (3000, 16384, (0, 9000, 16383), 0.0, 6.0),    # rows beyond the per-CTA cache
    # rows beyond the cache quantised early from global memory, some of them coded again
    # (a random outlier elsewhere flags the column of their largest value)
    (3000, 16384, (7, 12000), 3e-5, 6.0),
    (16, 14336, (100, 14000), 0.0, 6.0),
    (20, 10000, (), 0.0, 0.0),      # n_o = 10000: indices past the 8192 kept in shared memory
    # >= 8 cached rows per CTA: rows quantised before the grid barrier.  Random outliers
    # flag columns in which the other rows hold ordinary values, so some rows keep their
    # early codes (outlier columns cleared) and others, whose largest value sits in such a
    # column, are coded again; K = 2064 ends in a partial 128-column block
    (2000, 2064, (5, 100, 2063), 5e-5, 6.0),
    (1500, 1040, (), 0.0, math.inf),
    (1400, 256, (3,), 0.0, 0.0),
    # one row per CTA fits in shared memory: the other rows of a CTA pass through that one
    # slot, all 16 warps on each; and rows too long for any slot, read from global memory
    (300, 57344, (5, 30000, 57343), 1e-5, 6.0),
    (300, 131072, (0, 131071), 0.0, 6.0),
]


@pytest.mark.parametrize("fused", [False, True], ids=["two_pass", "fused"])
@pytest.mark.parametrize("T,K,cols,frac,thr", SCAN_CASES)
def test_scan_and_quantize_act_bitexact(T, K, cols, frac, thr, fused):
    w, X, _, _ = _case(T, K, 8, seed=T + K, cols=cols, random_frac=frac)
    X_d = dev(X)
    if fused:
        mask, idx, n_o, Xq, SCx, X_o = gpu_prepare(X_d, thr)
    else:
        mask, idx, n_o = gpu_scan(X_d, thr)
        Xq, SCx, X_o = gpu_quantize_act(X_d, mask, idx, n_o)
    sync_ok()
    flags, words, idx_r = O.outlier_scan(X, thr)
    n = int(host(n_o)[0])
    assert n == idx_r.size
    assert np.array_equal(host(mask).view(np.uint32), words)
    assert np.array_equal(host(idx)[:n], idx_r)
    Xq_r, SCx_r = O.absmax_quantize_rows(X, flags)
    assert np.array_equal(host(SCx).view(np.uint32), SCx_r.view(np.uint32))
    assert np.array_equal(host(Xq), Xq_r)
    xo = slice_to_matrix(host(X_o), T, K, n)
    ref = np.zeros_like(xo)
    ref[:, :n] = X[:, idx_r]
    assert np.array_equal(xo.view(np.uint16), ref.view(np.uint16))


def test_scan_infinities_at_inf_threshold():
    X = synth.random_fp16((40, 128), seed=3)
    X[5, 9] = np.float16(np.inf)
    X[30, 100] = np.float16(-np.inf)
    mask, idx, n_o = gpu_scan(dev(X), math.inf)
    sync_ok()
    assert host(idx)[: int(host(n_o)[0])].tolist() == [9, 100]


# ------------------------------------------------------------------ step 4
IGEMM_CASES = [
    # T, N, K  (T <= 16: decode GEMV kernels; T > 16: tcgen05 GEMM)
    (1, 1000, 3600), (3, 64, 64), (8, 257, 4096), (13, 1000, 208), (16, 2000, 14336),
    (17, 64, 64), (127, 300, 464), (129, 257, 128), (300, 600, 4096), (512, 1024, 1040),
]


@pytest.mark.parametrize("T,N,K", IGEMM_CASES)
def test_igemm_s32_bitexact(T, N, K):
    A = synth.random_int8((T, K), seed=T * 31 + K)
    B = synth.random_int8((N, K), seed=N * 17 + K + 1)
    acc = gpu_igemm(dev(A), dev(B))
    sync_ok()
    assert np.array_equal(host(acc), O.int_matmul(A, B))


@pytest.mark.parametrize("T", [4, 200])
def test_igemm_s32_extreme_codes(T):
    K = 14336
    A = np.full((T, K), 127, np.int8)
    A[1::2] = -127
    B = np.full((40, K), -127, np.int8)
    B[::3] = 127
    acc = gpu_igemm(dev(A), dev(B))
    sync_ok()
    assert np.array_equal(host(acc), O.int_matmul(A, B))


# ------------------------------------------------------------------ steps 1..6 (forward)
FORWARD_CASES = [
    # T, K, N, cols, random_frac, threshold, bias
    (16, 64, 64, (3, 41), 0.0, 6.0, True),          # the tiny [16 x 64] x [64 x 64] case
    (5, 3600, 1000, (10, 2000), 0.0, 6.0, True),    # decode path, ragged rows / slices
    (16, 1040, 300, (), 0.0, math.inf, False),      # decode, pure vector-wise int8
    (16, 208, 100, (4,), 0.0, 0.0, True),           # decode, every column fp16
    (300, 464, 600, (0, 5, 200, 463), 0.003, 6.0, True),   # GEMM, ragged everywhere
    (129, 1040, 513, tuple(range(0, 1040, 13)), 0.0, 6.0, True),  # 80 outlier cols
    (256, 4096, 512, (), 0.0, math.inf, True),      # GEMM, no outliers (2 TMEM buffers)
    (64, 208, 256, (9,), 0.0, 0.0, True),           # GEMM, thr 0: only the fp16 product
    (200, 128, 100, (1, 2, 3), 0.0, 6.0, False),
    # decode kernel: more than 32 outlier columns in one K-slice (bytes read from CB
    # instead of the copies), one token, a ragged 16-row tile
    (1, 14336, 257, tuple(range(0, 3584, 89)) + (9000, 14335), 0.0, 6.0, True),
    (9, 1024, 130, (), 0.0, 0.0, True),             # decode, n_o = K > 128 kept columns
    (8, 65536, 40, (0, 30000, 65535), 0.0, 6.0, True),     # decode, largest K (19 slices)
    (4, 65552, 33, (1, 65551), 0.0, 6.0, True),     # T <= 16 beyond 65536: GEMM path
    (12, 3584, 48, (3583,), 0.0, 6.0, False),       # one slice, last column an outlier
    (9, 8000, 333, (1, 4000, 7999), 0.0, 6.0, True),  # decode, X > 128 KB: split prologue
    (40, 9216, 96, (), 0.0, 0.0, True),             # GEMM, n_o = 9216 (> 8192 kept indices)
    # GEMM, one outlier chunk with adjacent and far-apart columns, and a single outlier
    # column on ragged tiles without bias
    (300, 1040, 700, (0, 1, 2, 3, 4, 5, 6, 1039), 0.0, 6.0, True),      # n_o = 8
    (300, 1040, 700, (0, 1, 2, 3, 4, 5, 6, 7, 1039), 0.0, 6.0, True),   # n_o = 9
    (513, 4096, 1000, (77,), 0.0, 6.0, False),      # n_o = 1
    # few outlier columns with N not a multiple of 8 (stores from registers instead of
    # TMA), with bias
    (257, 512, 1001, (3, 400), 0.0, 6.0, True),
    (1500, 1040, 300, (7, 1039), 5e-5, 6.0, True),  # rows quantised before the grid barrier
]


@pytest.mark.parametrize("T,K,N,cols,frac,thr,bias", FORWARD_CASES)
def test_linear_forward_parity(T, K, N, cols, frac, thr, bias):
    w, X, W, b = _case(T, K, N, seed=T * 3 + N, cols=cols, random_frac=frac, bias=bias)
    CB, SCB = gpu_quantize_weight(dev(W))
    C = gpu_forward(dev(X), CB, SCB, None if b is None else dev(b), thr)
    sync_ok()
    CBr, SCBr = O.quantize_weight(W)
    assert np.array_equal(host(CB), CBr)
    r = O.linear_forward(X, CBr, SCBr, b, thr)
    check_output(host(C), r["C"])


def test_forward_repeat_is_deterministic():
    w, X, W, b = _case(300, 464, 600, seed=5, cols=(7, 300))
    CB, SCB = gpu_quantize_weight(dev(W))
    X_d, b_d = dev(X), dev(b)
    C1 = host(gpu_forward(X_d, CB, SCB, b_d, 6.0))
    C2 = host(gpu_forward(X_d, CB, SCB, b_d, 6.0))
    sync_ok()
    assert np.array_equal(C1.view(np.uint16), C2.view(np.uint16))


@pytest.mark.parametrize("K", [2048, 12288], ids=["x_per_cta", "x_split"])
def test_decode_row_max_next_to_an_outlier_column(K):
    """SCx excludes outlier columns but keeps the other columns of their block: each row's
    largest non-outlier value sits right beside an outlier column (K = 2048: every CTA
    scans all of X; K = 12288, X > 128 KB: the CTAs split the scan)."""
    T, N = 6, 96
    w, X, W, b = _case(T, K, N, seed=21, cols=(300, 1500))
    X = np.clip(X.astype(np.float32), -3.0, 3.0).astype(np.float16)
    X[:, 300] = np.float16(9.0)
    X[:, 1500] = np.float16(-7.5)
    for t in range(T):
        X[t, 301 if t % 2 else 1499] = np.float16(5.5 - 0.25 * t)
    CB, SCB = gpu_quantize_weight(dev(W))
    C = gpu_forward(dev(X), CB, SCB, dev(b), 6.0)
    sync_ok()
    CBr, SCBr = O.quantize_weight(W)
    r = O.linear_forward(X, CBr, SCBr, b, 6.0)
    assert np.array_equal(r["SCx"], np.array([5.5 - 0.25 * t for t in range(T)], np.float32))
    check_output(host(C), r["C"])


@pytest.mark.parametrize("T", [1, 16])
def test_decode_workspace_garbage_and_reuse(T):
    """The decode kernel's counters and epoch-tagged words need no clearing: a workspace
    full of 0xff, then reused by further calls (also of another shape), gives the same
    output every time (T = 16: X > 128 KB, the cooperative prologue)."""
    w, X, W, b = _case(T, 4608, 1000, seed=T + 40, cols=(10, 2000))
    CB, SCB = gpu_quantize_weight(dev(W))
    X_d, b_d = dev(X), dev(b)
    nbytes = max(abi.i8_linear_workspace_size(T, 1000, 4608),
                 abi.i8_linear_workspace_size(2, 500, 4608))
    ws = torch.full((nbytes,), 255, dtype=torch.uint8, device="cuda")
    CBr, SCBr = O.quantize_weight(W)
    ref = O.linear_forward(X, CBr, SCBr, b, 6.0)["C"]
    outs = []
    for i in range(3):
        C = torch.full((T, 1000), float("nan"), dtype=torch.float16, device="cuda")
        abi.i8_linear_forward(X_d, CB, SCB, b_d, 6.0, C, ws)
        outs.append(host(C))
        if i == 1:  # another shape on the same workspace in between
            X2 = dev(synth.random_fp16((2, 4608), seed=7, sigma=1.0))
            C2 = torch.empty((2, 500), dtype=torch.float16, device="cuda")
            abi.i8_linear_forward(X2, CB[:500].contiguous(), SCB[:500].contiguous(), None,
                                  6.0, C2, ws)
    sync_ok()
    for C in outs:
        check_output(C, ref)
        assert np.array_equal(C.view(np.uint16), outs[0].view(np.uint16))


def test_power_of_two_row_scaling_gpu():
    """Metamorphic: scaling a token by 2 (exact, below the threshold) scales its output's
    int8 part exactly and leaves its codes unchanged."""
    w, X, W, b = _case(64, 256, 128, seed=9, cols=())
    X = np.clip(X.astype(np.float32), -2.9, 2.9).astype(np.float16)
    X2 = X.copy()
    X2[7] = (X[7].astype(np.float32) * 2).astype(np.float16)
    out = []
    for x in (X, X2):
        m, i, n = gpu_scan(dev(x), 6.0)
        Xq, SCx, _ = gpu_quantize_act(dev(x), m, i, n)
        out.append((host(Xq), host(SCx)))
    sync_ok()
    assert np.array_equal(out[0][0], out[1][0])
    assert out[1][1][7] == 2 * out[0][1][7]


# ------------------------------------------------------------------ failure path
def test_bounded_wait_times_out_and_context_survives():
    abi.i8_selftest_bounded_wait(2_000_000)   # 2 ms: nothing completes the barrier
    st = abi.i8_sync_status()
    assert abi.STATUS[st] == "I8_ERR_TIMEOUT"
    assert abi.i8_sync_status() == 0          # the word was cleared
    A = synth.random_int8((20, 64), seed=1)
    B = synth.random_int8((30, 64), seed=2)
    acc = gpu_igemm(dev(A), dev(B))
    sync_ok()
    assert np.array_equal(host(acc), O.int_matmul(A, B))


def test_invalid_arguments_launch_nothing():
    X = torch.zeros((4, 64), dtype=torch.float16, device="cuda")
    CB = torch.zeros((8, 64), dtype=torch.int8, device="cuda")
    SCB = torch.zeros((8,), dtype=torch.float32, device="cuda")
    C = torch.zeros((4, 8), dtype=torch.float16, device="cuda")
    small = torch.empty((16,), dtype=torch.uint8, device="cuda")
    with pytest.raises(abi.I8Error) as e:
        abi.i8_linear_forward(X, CB, SCB, None, 6.0, C, small)
    assert e.value.code == 1
    with pytest.raises(abi.I8Error):
        abi.i8_linear_forward(X, CB, SCB, None, float("nan"), C, small)
    sync_ok()
