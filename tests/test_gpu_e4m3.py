"""e4m3 (FP8) variant of the layer through the C ABI, against the CPU oracle.

Bit-exact: the weight's e4m3 codes and scales; the activation's mask, index list, e4m3
codes, row scales and fp16 outlier slice.  Tolerance (fp16 output, per row), the same form
as the int8 layer's:
    max|C - C_ref| <= 2^-9 * max_row|C_ref| + 1e-3.
C_ref is exact (the e4m3 products summed in fp64); the GPU sums the same products in
fp32 inside the tensor cores, in another order, and rounds the result to fp16 (2^-11
relative), so its error is the fp16 rounding plus fp32 accumulation error, well inside
the bound at these sizes.
"""
import math

import numpy as np
import pytest
import torch

from bit_matmul_decomposition_b200 import abi, synth
from oracle import oracle as O
from tests.gpu_util import DEV, check_output, dev, host, slice_to_matrix, sync_ok

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    abi.load()
    yield
    torch.cuda.synchronize()


def _case(T, K, N, seed, cols=(), random_frac=0.0, bias=True):
    w = synth.Workload("e4m3", T, K, N, seed=seed, fixed_cols=tuple(cols) if cols else None,
                       random_frac=random_frac, bias=bias)
    return synth.make_x(w), synth.make_w(w), synth.make_bias(w)


def _quantize_weight(W):
    N, K = W.shape
    CB = torch.empty((N, K), dtype=torch.uint8, device=DEV)
    SCB = torch.empty((N,), dtype=torch.float32, device=DEV)
    abi.i8_quantize_weight_e4m3(dev(W), CB, SCB)
    return CB, SCB


@pytest.mark.parametrize("N,K", [(64, 64), (129, 80), (300, 4096), (17, 16400), (5, 16),
                                 (1000, 16), (2001, 2064), (150, 14336), (2, 32784)])
def test_quantize_weight_e4m3_bitexact(N, K):
    W = synth.random_fp16((N, K), seed=N * 5 + K, sigma=0.02)
    W[0, :] = 0                      # an all-zero output channel
    W[1 % N, 3 % K] = -0.0           # a signed zero
    CB, SCB = _quantize_weight(W)
    sync_ok()
    CBr, SCBr = O.quantize_weight_e4m3(W)
    assert np.array_equal(host(CB), CBr)
    assert np.array_equal(host(SCB).view(np.uint32), SCBr.view(np.uint32))


PREP_CASES = [
    # T, K, cols, random_frac, threshold
    (16, 64, (3, 41), 0.0, 6.0),
    (300, 464, (0, 5, 200, 463), 0.003, 6.0),
    (77, 208, (), 0.0, 2.5),
    (33, 96, (1,), 0.0, 0.0),
    (33, 96, (1, 2), 0.0, math.inf),
    (3000, 16384, (0, 9000, 16383), 0.0, 6.0),
    (2000, 2064, (5, 100, 2063), 5e-5, 6.0),   # early codes kept for some rows, redone for others
]


@pytest.mark.parametrize("T,K,cols,frac,thr", PREP_CASES)
def test_prepare_act_e4m3_bitexact(T, K, cols, frac, thr):
    X, _, _ = _case(T, K, 8, seed=T + 2 * K, cols=cols, random_frac=frac)
    X_d = dev(X)
    mask = torch.empty(((K + 31) // 32 + 1,), dtype=torch.int32, device=DEV)
    idx = torch.empty((K,), dtype=torch.int32, device=DEV)
    n_o = torch.empty((4,), dtype=torch.int32, device=DEV)
    Xq = torch.empty((T, K), dtype=torch.uint8, device=DEV)
    SCx = torch.empty((T,), dtype=torch.float32, device=DEV)
    X_o = torch.empty((abi.i8_outlier_slice_elems(T, K),), dtype=torch.float16, device=DEV)
    abi.i8_prepare_act_e4m3(X_d, thr, mask, idx, n_o, Xq, SCx, X_o)
    sync_ok()
    r = O.linear_forward_e4m3(X, np.zeros((1, K), np.uint8), np.ones(1, np.float32), None,
                              thr, rows=np.arange(0))
    n = int(host(n_o)[0])
    assert n == r["n_o"]
    assert np.array_equal(host(mask)[: (K + 31) // 32].view(np.uint32), r["mask_words"])
    assert np.array_equal(host(idx)[:n], r["idx"])
    assert np.array_equal(host(Xq), r["Xq"])
    assert np.array_equal(host(SCx).view(np.uint32), r["SCx"].view(np.uint32))
    if n:
        Xo = slice_to_matrix(host(X_o), T, K, n)
        assert np.array_equal(Xo[:, :n].view(np.uint16), X[:, r["idx"]].view(np.uint16))
        assert not Xo[:, n:].view(np.uint16).any()


FORWARD_CASES = [
    # T, K, N, cols, random_frac, threshold, bias
    (16, 64, 64, (3, 41), 0.0, 6.0, True),          # the tiny case (T <= 16: still the GEMM)
    (5, 3600, 1000, (10, 2000), 0.0, 6.0, True),
    (300, 464, 600, (0, 5, 200, 463), 0.003, 6.0, True),     # ragged everywhere
    (129, 1040, 513, tuple(range(0, 1040, 13)), 0.0, 6.0, True),  # 80 outlier columns
    (256, 4096, 512, (), 0.0, math.inf, True),      # no outliers
    (64, 208, 256, (9,), 0.0, 0.0, True),           # thr 0: only the fp16 product
    (200, 128, 100, (1, 2, 3), 0.0, 6.0, False),
    (40, 9216, 96, (), 0.0, 0.0, True),             # n_o = 9216 (> 8192 kept indices)
    (300, 1040, 700, (0, 1, 2, 3, 4, 5, 6, 1039), 0.0, 6.0, True),     # n_o = 8
    (300, 1040, 700, (0, 1, 2, 3, 4, 5, 6, 7, 1039), 0.0, 6.0, True),  # n_o = 9
]


def _forward(X, CB, SCB, b, thr):
    T, K = X.shape
    N = CB.shape[0]
    ws = torch.empty((abi.i8_linear_workspace_size_e4m3(T, N, K),), dtype=torch.uint8,
                     device=DEV)
    ws.fill_(0x5A)
    C = torch.full((T, N), float("nan"), dtype=torch.float16, device=DEV)
    abi.i8_linear_forward_e4m3(dev(X), CB, SCB, None if b is None else dev(b), thr, C, ws)
    return C


@pytest.mark.parametrize("T,K,N,cols,frac,thr,bias", FORWARD_CASES)
def test_linear_forward_e4m3_parity(T, K, N, cols, frac, thr, bias):
    X, W, b = _case(T, K, N, seed=T * 7 + N, cols=cols, random_frac=frac, bias=bias)
    CB, SCB = _quantize_weight(W)
    C = _forward(X, CB, SCB, b, thr)
    sync_ok()
    CBr, SCBr = O.quantize_weight_e4m3(W)
    assert np.array_equal(host(CB), CBr)
    r = O.linear_forward_e4m3(X, CBr, SCBr, b, thr)
    check_output(host(C), r["C"])


def test_forward_e4m3_full_size_sampled_rows():
    """The OPT-6.7B FFN-up shape (2048 x 4096 x 16384, 6 outlier columns): the codes of
    the weight in full, the output on 12 sampled rows plus the first and last."""
    w = synth.opt_ffn_up_prefill()
    X, W, b = synth.make_x(w), synth.make_w(w), synth.make_bias(w)
    CB, SCB = _quantize_weight(W)
    C = _forward(X, CB, SCB, b, w.threshold)
    sync_ok()
    CBr, SCBr = O.quantize_weight_e4m3(W)
    assert np.array_equal(host(CB), CBr)
    rows = np.unique(np.concatenate([[0, w.T - 1], np.linspace(1, w.T - 2, 12).astype(int)]))
    r = O.linear_forward_e4m3(X, CBr, SCBr, b, w.threshold, rows=rows)
    check_output(host(C)[rows], r["C"])


def test_e4m3_and_int8_layers_agree_to_their_step_sizes():
    """Both variants approximate the same product: their outputs differ by no more than
    the two quantisations' error bounds allow (a cross-check of the e4m3 scale handling:
    a wrong 127 / 448 would move the e4m3 output by a factor of 3.5)."""
    X, W, b = _case(200, 1024, 300, seed=3, cols=(5, 700))
    CB8, SCB8 = _quantize_weight(W)
    C8 = host(_forward(X, CB8, SCB8, b, 6.0)).astype(np.float64)
    CBi = torch.empty((300, 1024), dtype=torch.int8, device=DEV)
    SCBi = torch.empty((300,), dtype=torch.float32, device=DEV)
    abi.i8_quantize_weight(dev(W), CBi, SCBi)
    ws = torch.empty((abi.i8_linear_workspace_size(200, 300, 1024),), dtype=torch.uint8,
                     device=DEV)
    Ci = torch.empty((200, 300), dtype=torch.float16, device=DEV)
    abi.i8_linear_forward(dev(X), CBi, SCBi, dev(b), 6.0, Ci, ws)
    sync_ok()
    ref = X.astype(np.float64) @ W.astype(np.float64).T + b.astype(np.float64)
    scale = np.abs(ref).max()
    assert np.abs(C8 - ref).max() < 0.08 * scale
    assert np.abs(host(Ci).astype(np.float64) - ref).max() < 0.08 * scale
