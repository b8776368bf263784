"""Host-side checks of the Python binding (no GPU): every wrapper passes the shapes, sizes
and pointers the C call expects, and refuses a tensor of the wrong dtype or too few
elements before anything reaches the library.  The C calls take bare pointers, most with
no size argument, so a short output buffer would otherwise be written out of bounds on the
device.

The library is replaced by a recorder and pointers are taken from CPU tensors; the
checks under test run before either is used."""
import math

import pytest
import torch

from bit_matmul_decomposition_b200 import abi


class _Recorder:
    def __init__(self):
        self.calls = []

    def __getattr__(self, name):
        def fn(*args):
            self.calls.append((name, args))
            return 0
        return fn


@pytest.fixture
def rec(monkeypatch):
    r = _Recorder()
    monkeypatch.setattr(abi, "load", lambda *a, **k: r)
    monkeypatch.setattr(abi, "_ptr", lambda t: None if t is None else t.data_ptr())
    monkeypatch.setattr(abi, "_stream", lambda s: 0)
    return r


def _t(shape, dtype):
    return torch.zeros(shape, dtype=dtype)


T, K, N = 5, 96, 40
WORDS = (K + 31) // 32
SLICE = (K + 63) // 64 * T * 64


def _forward_args(codes=torch.int8):
    return dict(X=_t((T, K), torch.float16), CB=_t((N, K), codes), SCB=_t((N,), torch.float32),
                bias=_t((N,), torch.float16), C=_t((T, N), torch.float16))


def test_forward_marshals_shapes_and_sizes(rec):
    a = _forward_args()
    ws = _t((1000,), torch.uint8)
    abi.i8_linear_forward(a["X"], a["CB"], a["SCB"], a["bias"], 6.0, a["C"], ws)
    name, args = rec.calls[-1]
    assert name == "i8_linear_forward"
    assert args[1:3] == (T, K) and args[6] == N and args[7] == 6.0
    assert args[0] == a["X"].data_ptr() and args[8] == a["C"].data_ptr()
    assert args[9] == ws.data_ptr() and args[10] == 1000
    abi.i8_linear_forward(a["X"], a["CB"], a["SCB"], None, math.inf, a["C"], ws)
    assert rec.calls[-1][1][5] is None


def test_every_wrapper_accepts_well_formed_tensors(rec):
    a = _forward_args()
    ws = _t((64,), torch.uint8)
    cache = _t((64,), torch.uint8)
    mask, idx, n_o = _t((WORDS + 1,), torch.int32), _t((K,), torch.int32), _t((4,), torch.int32)
    Xq, SCx, X_o = _t((T, K), torch.int8), _t((T,), torch.float32), _t((SLICE,), torch.float16)
    W = _t((N, K), torch.float16)
    abi.i8_quantize_weight(W, a["CB"], a["SCB"])
    abi.i8_outlier_scan(a["X"], 6.0, mask[:WORDS], idx, n_o)
    abi.i8_quantize_act(a["X"], mask[:WORDS], idx, n_o, Xq, SCx, X_o)
    abi.i8_prepare_act(a["X"], 6.0, mask, idx, n_o, Xq, SCx, X_o)
    abi.i8_linear_forward_noalloc(a["X"], a["CB"], a["SCB"], a["bias"], 6.0, a["C"])
    abi.i8_linear_forward_cached(a["X"], a["CB"], a["SCB"], a["bias"], 6.0, a["C"], ws, cache)
    abi.i8_igemm_s32(Xq, a["CB"], _t((T, N), torch.int32), ws)
    e = _forward_args(torch.uint8)
    abi.i8_quantize_weight_e4m3(W, e["CB"], e["SCB"])
    abi.i8_prepare_act_e4m3(a["X"], 6.0, mask, idx, n_o, _t((T, K), torch.uint8), SCx, X_o)
    abi.i8_linear_forward_e4m3(e["X"], e["CB"], e["SCB"], e["bias"], 6.0, e["C"], ws)
    names = [c[0] for c in rec.calls]
    assert names == ["i8_quantize_weight", "i8_outlier_scan", "i8_quantize_act",
                     "i8_prepare_act", "i8_linear_forward_noalloc", "i8_linear_forward_cached",
                     "i8_igemm_s32", "i8_quantize_weight_e4m3", "i8_prepare_act_e4m3",
                     "i8_linear_forward_e4m3"]
    assert rec.calls[0][1][1:3] == (N, K)              # W's shape
    assert rec.calls[6][1][1:3] == (T, K) and rec.calls[6][1][4] == N


@pytest.mark.parametrize("field,bad,err", [
    ("X", _t((T, K), torch.float32), TypeError),
    ("X", _t((T * K,), torch.float16), ValueError),      # not 2-D
    ("CB", _t((N, K - 16), torch.int8), ValueError),     # K differs from X's
    ("CB", _t((N, K), torch.uint8), TypeError),          # e4m3 codes into the int8 call
    ("SCB", _t((N - 1,), torch.float32), ValueError),
    ("SCB", _t((N,), torch.float16), TypeError),
    ("bias", _t((N - 1,), torch.float16), ValueError),
    ("bias", _t((N,), torch.float32), TypeError),
    ("C", _t((T, N - 1), torch.float16), ValueError),    # one element short per row
    ("C", _t((T, N), torch.float32), TypeError),
])
def test_forward_rejects_wrong_tensors_before_the_call(rec, field, bad, err):
    a = _forward_args()
    a[field] = bad
    ws = _t((64,), torch.uint8)
    for call in (lambda: abi.i8_linear_forward(a["X"], a["CB"], a["SCB"], a["bias"], 6.0,
                                               a["C"], ws),
                 lambda: abi.i8_linear_forward_noalloc(a["X"], a["CB"], a["SCB"], a["bias"],
                                                       6.0, a["C"]),
                 lambda: abi.i8_linear_forward_cached(a["X"], a["CB"], a["SCB"], a["bias"],
                                                      6.0, a["C"], ws, ws)):
        with pytest.raises(err, match=field):
            call()
    assert rec.calls == []


def test_e4m3_forward_refuses_int8_codes(rec):
    a = _forward_args(torch.int8)
    with pytest.raises(TypeError, match="CB"):
        abi.i8_linear_forward_e4m3(a["X"], a["CB"], a["SCB"], a["bias"], 6.0, a["C"],
                                   _t((64,), torch.uint8))
    with pytest.raises(TypeError, match="CB"):
        abi.i8_quantize_weight_e4m3(_t((N, K), torch.float16), a["CB"], a["SCB"])
    assert rec.calls == []


def test_stage_calls_reject_short_outputs(rec):
    X = _t((T, K), torch.float16)
    mask, idx, n_o = _t((WORDS + 1,), torch.int32), _t((K,), torch.int32), _t((1,), torch.int32)
    Xq, SCx, X_o = _t((T, K), torch.int8), _t((T,), torch.float32), _t((SLICE,), torch.float16)
    with pytest.raises(ValueError, match="col_mask"):     # the fused pass needs one more word
        abi.i8_prepare_act(X, 6.0, mask[:WORDS], idx, n_o, Xq, SCx, X_o)
    with pytest.raises(ValueError, match="outlier_idx"):
        abi.i8_outlier_scan(X, 6.0, mask, idx[:K - 1], n_o)
    with pytest.raises(ValueError, match="n_outliers"):
        abi.i8_outlier_scan(X, 6.0, mask, idx, _t((0,), torch.int32))
    with pytest.raises(ValueError, match="X_o"):          # the slice is chunk-major, K rounded to 64
        abi.i8_quantize_act(X, mask, idx, n_o, Xq, SCx, _t((T * K,), torch.float16))
    with pytest.raises(ValueError, match="Xq"):
        abi.i8_quantize_act(X, mask, idx, n_o, Xq[:T - 1], SCx, X_o)
    with pytest.raises(ValueError, match="SCx"):
        abi.i8_prepare_act(X, 6.0, mask, idx, n_o, Xq, SCx[:T - 1], X_o)
    with pytest.raises(TypeError, match="Xq"):
        abi.i8_prepare_act_e4m3(X, 6.0, mask, idx, n_o, Xq, SCx, X_o)
    with pytest.raises(ValueError, match="CB"):
        abi.i8_quantize_weight(_t((N, K), torch.float16), _t((N, K - 16), torch.int8),
                               _t((N,), torch.float32))
    with pytest.raises(ValueError, match="acc"):
        abi.i8_igemm_s32(Xq, _t((N, K), torch.int8), _t((T, N - 1), torch.int32),
                         _t((64,), torch.uint8))
    with pytest.raises(ValueError, match="B has"):
        abi.i8_igemm_s32(Xq, _t((N, K + 16), torch.int8), _t((T, N), torch.int32),
                         _t((64,), torch.uint8))
    assert rec.calls == []


def test_slice_size_matches_the_library():
    """The binding's own copy of the slice size agrees with the library's."""
    import ctypes

    from bit_matmul_decomposition_b200 import build
    build.build()
    real = ctypes.CDLL(abi.LIB_PATH)
    real.i8_outlier_slice_elems.restype = ctypes.c_size_t
    real.i8_outlier_slice_elems.argtypes = [ctypes.c_int64, ctypes.c_int64]
    for rows, k in [(1, 16), (5, 96), (300, 464), (2048, 4096), (7, 65552)]:
        assert abi._slice_elems(rows, k) == real.i8_outlier_slice_elems(rows, k)


def test_backward_bindings_marshal_and_check(rec):
    dY, W, X = _t((T, N), torch.float16), _t((N, K), torch.float16), _t((T, K), torch.float16)
    dX, dW, db = _t((T, K), torch.float16), _t((N, K), torch.float16), _t((N,), torch.float16)
    abi.i8_linear_backward_input(dY, W, dX)
    assert rec.calls[-1][0] == "i8_linear_backward_input"
    assert rec.calls[-1][1][1:3] == (T, N) and rec.calls[-1][1][4] == K
    abi.i8_linear_backward_weight(dY, X, dW)
    assert rec.calls[-1][0] == "i8_linear_backward_weight" and rec.calls[-1][1][2:5] == (T, N, K)
    abi.i8_bias_grad(dY, db)
    assert rec.calls[-1][0] == "i8_bias_grad" and rec.calls[-1][1][1:3] == (T, N)
    with pytest.raises(ValueError):
        abi.i8_linear_backward_input(dY, _t((N + 1, K), torch.float16), dX)   # rows != N
    with pytest.raises(ValueError):
        abi.i8_linear_backward_input(dY, W, _t((T, K - 1), torch.float16))   # short dX
    with pytest.raises(ValueError):
        abi.i8_linear_backward_weight(dY, _t((T + 1, K), torch.float16), dW)  # rows != T
    with pytest.raises(TypeError):
        abi.i8_bias_grad(_t((T, N), torch.float32), db)
    with pytest.raises(ValueError):
        abi.i8_bias_grad(dY, _t((N - 1,), torch.float16))


def test_dequantize_binding_picks_the_code_format(rec):
    SCB, Wd = _t((N,), torch.float32), _t((N, K), torch.float16)
    abi.i8_dequantize_weight(_t((N, K), torch.int8), SCB, Wd)
    assert rec.calls[-1][0] == "i8_dequantize_weight" and rec.calls[-1][1][2:4] == (N, K)
    abi.i8_dequantize_weight(_t((N, K), torch.uint8), SCB, Wd)
    assert rec.calls[-1][0] == "i8_dequantize_weight_e4m3"
    with pytest.raises(ValueError):
        abi.i8_dequantize_weight(_t((N, K), torch.int8), SCB, _t((N, K - 1), torch.float16))
