"""The nn.Module front end on the GPU against the CPU oracle: quantisation bit for bit,
outputs within the per-row tolerance on both the decode (T <= 16) and GEMM (T > 16)
paths, exact restore of the quantised state, and a small layer stack converted with the
replacement helper, checked layer by layer."""
import io

import numpy as np
import pytest
import torch

from bit_matmul_decomposition_b200 import abi, synth
from bit_matmul_decomposition_b200.linear import Linear8bitLt, replace_linear_with_int8
from oracle import oracle as O
from tests.gpu_util import check_output, host, sync_ok

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    abi.load()
    yield
    torch.cuda.synchronize()


def _fp16_linear(K, N, seed, bias=True):
    g = torch.Generator().manual_seed(seed)
    lin = torch.nn.Linear(K, N, bias=bias).half()
    with torch.no_grad():
        lin.weight.copy_((torch.randn(N, K, generator=g) * 0.02).half())
        if bias:
            lin.bias.copy_((torch.randn(N, generator=g) * 0.02).half())
    return lin.cuda()


def _x(shape, K, cols, seed):
    X = synth.random_fp16((int(np.prod(shape)), K), seed=seed)
    X = synth.plant_columns(X, cols, seed=seed + 1)
    return X.reshape(*shape, K)


@pytest.mark.parametrize("lead", [(1, 5), (3, 7)], ids=["decode_T5", "gemm_T21"])
def test_module_matches_oracle(lead):
    K, N = 1024, 768
    lin = _fp16_linear(K, N, seed=11)
    m = Linear8bitLt.from_linear(lin, threshold=6.0)
    W = host(lin.weight)
    CBr, SCBr = O.quantize_weight(W)
    assert np.array_equal(host(m.CB), CBr)
    assert np.array_equal(host(m.SCB).view(np.uint32), SCBr.view(np.uint32))
    X = _x(lead, K, (7, 500, 1000), seed=21)
    y = m(torch.from_numpy(X.view(np.int16)).view(torch.float16).cuda())
    sync_ok()
    assert tuple(y.shape) == (*lead, N)
    ref = O.linear_forward(X.reshape(-1, K), CBr, SCBr, host(lin.bias), 6.0)["C"]
    check_output(host(y).reshape(-1, N), ref)


def test_state_dict_restores_the_same_outputs():
    K, N = 512, 256
    m = Linear8bitLt.from_linear(_fp16_linear(K, N, seed=5))
    buf = io.BytesIO()
    torch.save(m.state_dict(), buf)
    buf.seek(0)
    m2 = Linear8bitLt(K, N, device="cuda")
    m2.load_state_dict(torch.load(buf))
    x = torch.from_numpy(_x((40,), K, (3,), seed=9).view(np.int16)).view(torch.float16).cuda()
    y1, y2 = host(m(x)), host(m2(x))
    sync_ok()
    assert np.array_equal(y1.view(np.uint16), y2.view(np.uint16))


def test_outlier_cache_layer_matches_and_follows_new_weights():
    K, N = 1024, 768
    lin1, lin2 = _fp16_linear(K, N, seed=31), _fp16_linear(K, N, seed=32)
    plain = Linear8bitLt.from_linear(lin1)
    cached = Linear8bitLt.from_linear(lin1, outlier_cache_cols=64)
    xs = [torch.from_numpy(_x((T,), K, cols, seed=40 + T).view(np.int16)).view(torch.float16).cuda()
          for T, cols in ((300, (7, 900)), (300, (7, 900)), (48, (7, 900)), (5, (2,)),
                          (300, (11,)))]
    for x in xs:                       # miss, hit, hit at another T, decode, miss
        assert torch.equal(plain(x).view(torch.int16), cached(x).view(torch.int16))
    # new codes through load_state_dict (same CB buffer): the cache must not serve the old
    cached.load_state_dict(Linear8bitLt.from_linear(lin2).state_dict())
    plain2 = Linear8bitLt.from_linear(lin2)
    for x in xs[:2]:
        assert torch.equal(plain2(x).view(torch.int16), cached(x).view(torch.int16))
    # and through quantize_
    cached.quantize_(lin1.weight.detach(), lin1.bias.detach())
    assert torch.equal(plain(xs[0]).view(torch.int16), cached(xs[0]).view(torch.int16))
    sync_ok()


@pytest.mark.parametrize("lead", [(1, 5), (3, 7)], ids=["T5", "T21"])
def test_e4m3_module_matches_oracle(lead):
    K, N = 1024, 768
    lin = _fp16_linear(K, N, seed=13)
    m = Linear8bitLt.from_linear(lin, code_format="e4m3")
    W = host(lin.weight)
    CBr, SCBr = O.quantize_weight_e4m3(W)
    assert np.array_equal(host(m.CB), CBr)
    X = _x(lead, K, (7, 500, 1000), seed=23)
    y = m(torch.from_numpy(X.view(np.int16)).view(torch.float16).cuda())
    sync_ok()
    ref = O.linear_forward_e4m3(X.reshape(-1, K), CBr, SCBr, host(lin.bias), 6.0)["C"]
    check_output(host(y).reshape(-1, N), ref)
    # the weight the layer computes with is the decoded codes times SCB / 448 (fp32
    # arithmetic, rounded to fp16)
    wd = host(m.dequantized_weight())
    want = (O.e4m3_decode(CBr).astype(np.float32)
            * (SCBr / np.float32(448.0)).astype(np.float32)[:, None]).astype(np.float16)
    assert np.array_equal(wd.view(np.uint16), want.view(np.uint16))


def test_replaced_layer_stack_layer_by_layer():
    """Linear -> GELU -> Linear (+ an fp16 head left alone): each int8 layer matches the
    oracle on the activations it actually received."""
    K, H = 512, 1024
    model = torch.nn.Sequential(_fp16_linear(K, H, seed=1), torch.nn.GELU(),
                                _fp16_linear(H, K, seed=2))
    model.lm_head = _fp16_linear(K, 64, seed=3)
    ws = [host(model[0].weight), host(model[2].weight)]
    bs = [host(model[0].bias), host(model[2].bias)]
    replace_linear_with_int8(model, threshold=6.0)
    assert isinstance(model[0], Linear8bitLt) and isinstance(model[2], Linear8bitLt)
    assert isinstance(model.lm_head, torch.nn.Linear)
    X = _x((2, 24), K, (10, 300), seed=31)
    x = torch.from_numpy(X.view(np.int16)).view(torch.float16).cuda()
    h1 = model[0](x)
    a1 = model[1](h1)
    h2 = model[2](a1)
    sync_ok()
    for layer, (W, b, xin, y) in enumerate([(ws[0], bs[0], X, h1),
                                            (ws[1], bs[1], host(a1), h2)]):
        CBr, SCBr = O.quantize_weight(W)
        ref = O.linear_forward(xin.reshape(-1, W.shape[1]), CBr, SCBr, b, 6.0)["C"]
        check_output(host(y).reshape(-1, W.shape[0]), ref)


def _ref_grads(X, W, gy):
    """Backward of y = x W^T + b (the oracle, fp64): dx = dy W, dW = dy^T x, db = sum(dy)."""
    return O.linear_backward(X, W, gy)


def _close(a, ref, rel=1e-2):
    a = a.astype(np.float64)
    assert np.isfinite(a).all()
    err = np.abs(a - ref).max()
    assert err <= rel * np.abs(ref).max() + 1e-3, (err, np.abs(ref).max())


@pytest.mark.parametrize("T", [6, 40], ids=["decode", "gemm"])
def test_training_mode_forward_backward_and_step(T):
    K, N = 512, 384
    lin = _fp16_linear(K, N, seed=7)
    m = Linear8bitLt.from_linear(lin, threshold=6.0, has_fp16_weights=True)
    X = _x((T,), K, (5, 77), seed=13)
    x = torch.from_numpy(X.view(np.int16)).view(torch.float16).cuda().requires_grad_(True)
    y = m(x)
    W = host(m.weight)
    CBr, SCBr = O.quantize_weight(W)
    check_output(host(y), O.linear_forward(X, CBr, SCBr, host(m.bias), 6.0)["C"])
    gy = synth.random_fp16((T, N), seed=17, sigma=0.5)
    y.backward(torch.from_numpy(gy.view(np.int16)).view(torch.float16).cuda())
    sync_ok()
    gx_r, gw_r, gb_r = _ref_grads(X, W, gy)
    _close(host(x.grad), gx_r)
    _close(host(m.weight.grad), gw_r)
    _close(host(m.bias.grad), gb_r)
    # one SGD step on the fp16 weight; the next forward quantises the new weight
    with torch.no_grad():
        m.weight -= 1e-4 * m.weight.grad
    y2 = m(x.detach())
    sync_ok()
    W2 = host(m.weight)
    CB2, SCB2 = O.quantize_weight(W2)
    assert np.array_equal(host(m.CB), CB2)
    check_output(host(y2), O.linear_forward(X, CB2, SCB2, host(m.bias), 6.0)["C"])


def test_inference_mode_passes_input_gradients():
    K, N, T = 256, 128, 20
    m = Linear8bitLt.from_linear(_fp16_linear(K, N, seed=19))
    X = _x((T,), K, (9,), seed=23)
    x = torch.from_numpy(X.view(np.int16)).view(torch.float16).cuda().requires_grad_(True)
    gy = synth.random_fp16((T, N), seed=29, sigma=0.5)
    m(x).backward(torch.from_numpy(gy.view(np.int16)).view(torch.float16).cuda())
    sync_ok()
    Wd = O.dequantize_weight(host(m.CB), host(m.SCB)).astype(np.float16)
    _close(host(x.grad), O.linear_backward(None, Wd, gy)[0])
    assert all(p.grad is None for p in m.parameters())
