"""The backward of the fp16-weight training mode, through the C ABI, against the oracle's
fp64 backward ("用法": has_fp16_weights=True for int8/fp16 mixed-precision training; the
gradients pass straight through the quantisation):

    dX = dY W,   dW = dY^T X,   db = sum_t dY[t, :]

The two products run on the tcgen05 tensor cores with the weight / input read as MN-major
operands; each output row is held to the forward's tolerance,
    max_n |C - C_ref| <= 2^-9 * max_n |C_ref| + 1e-3,
which covers the final fp16 rounding (2^-11 relative) and fp32 summation.  The cases span
several 256 x 256 tiles with ragged edges on every dimension, a reduction shorter than
one 64-element stage, and a single row.  The dequantised weight W' = CB * SCB / 127 (e4m3:
values * SCB / 448) is compared bit for bit with the oracle's fp32 recovery rounded to fp16.
"""
import numpy as np
import pytest
import torch

from bit_matmul_decomposition_b200 import abi, synth
from oracle import oracle as O
from tests.gpu_util import DEV, dev, host, sync_ok

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    abi.load()
    yield
    torch.cuda.synchronize()


def _rows_close(C, ref):
    C = C.astype(np.float64)
    assert np.isfinite(C).all(), "non-finite output"
    err = np.abs(C - ref).max(axis=1)
    allowed = 2.0 ** -9 * np.abs(ref).max(axis=1) + 1e-3
    assert (err <= allowed).all(), "worst err/allowed %.3f" % float((err / allowed).max())


@pytest.mark.parametrize("T,N,K", [(1, 8, 16), (17, 264, 272), (300, 1000, 1040),
                                   (513, 4096, 64), (256, 512, 256), (40, 24, 4096)])
def test_backward_input_product(T, N, K):
    dY = synth.random_fp16((T, N), seed=T + N, sigma=0.5)
    W = synth.random_fp16((N, K), seed=N + K, sigma=0.02)
    dX = torch.full((T, K), float("nan"), dtype=torch.float16, device=DEV)
    abi.i8_linear_backward_input(dev(dY), dev(W), dX)
    sync_ok()
    _rows_close(host(dX), O.linear_backward(None, W, dY)[0])


@pytest.mark.parametrize("T,N,K", [(1, 8, 16), (7, 264, 272), (300, 1000, 1040),
                                   (1000, 512, 64), (256, 256, 256), (4097, 24, 48)])
def test_backward_weight_product(T, N, K):
    dY = synth.random_fp16((T, N), seed=3 * T + N, sigma=0.5)
    X = synth.random_fp16((T, K), seed=5 * T + K, sigma=1.0)
    dW = torch.full((N, K), float("nan"), dtype=torch.float16, device=DEV)
    abi.i8_linear_backward_weight(dev(dY), dev(X), dW)
    sync_ok()
    _rows_close(host(dW), O.linear_backward(X, None, dY)[1])


@pytest.mark.parametrize("T,N", [(1, 8), (37, 264), (4096, 1000), (5, 16392)])
def test_bias_grad(T, N):
    dY = synth.random_fp16((T, N), seed=T * 7 + N, sigma=0.5)
    db = torch.full((N,), float("nan"), dtype=torch.float16, device=DEV)
    abi.i8_bias_grad(dev(dY), db)
    sync_ok()
    ref = O.linear_backward(None, None, dY)[2]
    got = host(db).astype(np.float64)
    # fp16 rounding of the result plus fp32 summation of T terms
    bound = (2.0 ** -11 * np.abs(ref) + T * 2.0 ** -24 * np.abs(dY.astype(np.float64)).sum(0)
             + 1e-7)
    assert (np.abs(got - ref) <= bound).all()
    db2 = torch.empty_like(db)
    abi.i8_bias_grad(dev(dY), db2)
    sync_ok()
    assert torch.equal(db.view(torch.int16), db2.view(torch.int16))   # fixed order


@pytest.mark.parametrize("N,K", [(1, 16), (300, 1040), (4099, 64)])
def test_dequantize_weight_bitexact(N, K):
    W = synth.random_fp16((N, K), seed=N + 11 * K, sigma=0.02)
    W[0] = 0
    CB, SCB = O.quantize_weight(W)
    out = torch.full((N, K), float("nan"), dtype=torch.float16, device=DEV)
    abi.i8_dequantize_weight(dev(CB), dev(SCB), out)
    sync_ok()
    want = O.dequantize_weight(CB, SCB).astype(np.float16)
    assert np.array_equal(host(out).view(np.uint16), want.view(np.uint16))
    CB8, SCB8 = O.quantize_weight_e4m3(W)
    abi.i8_dequantize_weight(dev(CB8), dev(SCB8), out)
    sync_ok()
    want8 = O.dequantize_weight(CB8, SCB8, e4m3=True).astype(np.float16)
    assert np.array_equal(host(out).view(np.uint16), want8.view(np.uint16))


def test_backward_rejects_unaligned_rows():
    dY = torch.zeros((4, 12), dtype=torch.float16, device=DEV)   # 24-byte rows
    W = torch.zeros((12, 64), dtype=torch.float16, device=DEV)
    dX = torch.zeros((4, 64), dtype=torch.float16, device=DEV)
    with pytest.raises(abi.I8Error) as e:
        abi.i8_linear_backward_input(dY, W, dX)
    assert e.value.code == 1
    sync_ok()
