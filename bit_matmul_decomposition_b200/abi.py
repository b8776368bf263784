"""Thin Python binding of libi8linear (include/i8linear.h): same names as the C ABI.

Argument marshalling only -- every step of the layer runs in the library's CUDA kernels.
Tensors are torch tensors on the current CUDA device (PyTorch provides device memory and
streams); their data pointers, sizes and the current stream go straight to the C calls.
A missing or unloadable library raises; nothing here falls back to another computation.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libi8linear.so")

STATUS = {0: "I8_OK", 1: "I8_ERR_INVALID_ARG", 2: "I8_ERR_UNSUPPORTED", 3: "I8_ERR_CUDA",
          4: "I8_ERR_TIMEOUT", 5: "I8_ERR_DEVICE"}

# every symbol the header declares, with (restype, argtypes)
_P = ctypes.c_void_p
_I64 = ctypes.c_int64
_F = ctypes.c_float
_SZ = ctypes.c_size_t
_ST = ctypes.c_int
SIGNATURES = {
    "i8_status_string": (ctypes.c_char_p, [_ST]),
    "i8_last_error": (ctypes.c_char_p, []),
    "i8_quantize_weight": (_ST, [_P, _I64, _I64, _P, _P, _P]),
    "i8_outlier_scan": (_ST, [_P, _I64, _I64, _F, _P, _P, _P, _P]),
    "i8_outlier_slice_elems": (_SZ, [_I64, _I64]),
    "i8_quantize_act": (_ST, [_P, _I64, _I64, _P, _P, _P, _P, _P, _P, _P]),
    "i8_prepare_act": (_ST, [_P, _I64, _I64, _F, _P, _P, _P, _P, _P, _P, _P]),
    "i8_linear_workspace_size": (_SZ, [_I64, _I64, _I64]),
    "i8_forward_kernel": (_ST, [_I64, _I64, _I64, _P]),
    "i8_linear_forward": (_ST, [_P, _I64, _I64, _P, _P, _P, _I64, _F, _P, _P, _SZ, _P]),
    "i8_igemm_s32": (_ST, [_P, _I64, _I64, _P, _I64, _P, _P, _SZ, _P]),
    "i8_linear_forward_noalloc": (_ST, [_P, _I64, _I64, _P, _P, _P, _I64, _F, _P, _P]),
    "i8_quantize_weight_e4m3": (_ST, [_P, _I64, _I64, _P, _P, _P]),
    "i8_prepare_act_e4m3": (_ST, [_P, _I64, _I64, _F, _P, _P, _P, _P, _P, _P, _P]),
    "i8_linear_workspace_size_e4m3": (_SZ, [_I64, _I64, _I64]),
    "i8_linear_forward_e4m3": (_ST, [_P, _I64, _I64, _P, _P, _P, _I64, _F, _P, _P, _SZ, _P]),
    "i8_outlier_cache_size": (_SZ, [_I64, _I64, _I64]),
    "i8_outlier_cache_reset": (_ST, [_P, _SZ, _P]),
    "i8_linear_forward_cached": (_ST, [_P, _I64, _I64, _P, _P, _P, _I64, _F, _P, _P, _SZ, _P,
                                       _SZ, _P]),
    "i8_linear_backward_input": (_ST, [_P, _I64, _I64, _P, _I64, _P, _P]),
    "i8_linear_backward_weight": (_ST, [_P, _P, _I64, _I64, _I64, _P, _P]),
    "i8_bias_grad": (_ST, [_P, _I64, _I64, _P, _P]),
    "i8_dequantize_weight": (_ST, [_P, _P, _I64, _I64, _P, _P]),
    "i8_dequantize_weight_e4m3": (_ST, [_P, _P, _I64, _I64, _P, _P]),
    "i8_sync_status": (_ST, [_P]),
    "i8_set_profile_events": (_ST, [_P, _P]),
    "i8_selftest_bounded_wait": (_ST, [_I64, _P]),
}


class I8Error(RuntimeError):
    def __init__(self, fn, code, detail=""):
        msg = "%s returned %s" % (fn, STATUS.get(code, code))
        super().__init__(msg + (" (%s)" % detail if detail else ""))
        self.code = code
        self.detail = detail


_lib = None


def load(path: str = LIB_PATH):
    """Load libi8linear.so (raises OSError when it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(path):
            raise OSError("libi8linear.so not built: run python -m bit_matmul_decomposition_b200.build")
        L = ctypes.CDLL(path)
        for name, (res, args) in SIGNATURES.items():
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _lib = L
    return _lib


def _check(fn, code):
    if code != 0:
        detail = ""
        if code == 3 and _lib is not None:   # I8_ERR_CUDA: which CUDA call failed
            detail = (_lib.i8_last_error() or b"").decode("utf-8", "replace")
        raise I8Error(fn, code, detail)


def _ptr(t) -> Optional[int]:
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("expected a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError("expected a contiguous tensor")
    import torch
    if t.device.index != torch.cuda.current_device():
        raise ValueError("tensor on %s, but the current device is cuda:%d: the call would "
                         "launch there (use torch.cuda.device)"
                         % (t.device, torch.cuda.current_device()))
    return t.data_ptr()


# The C calls take bare pointers, and most buffers have no size argument: the library
# trusts that X is [T, K], C is [T, N], and so on.  These checks hold every tensor to the
# dtype and the element count that its header comment states, so that a wrong or short
# buffer raises here instead of being read or written out of bounds on the device.
def _dt(*names):
    import torch
    return tuple(getattr(torch, n) for n in names)


def _arg(t, name, dtypes, elems):
    if t is None:
        raise ValueError("%s: a tensor is required" % name)
    if t.dtype not in dtypes:
        raise TypeError("%s: dtype %s, expected %s"
                        % (name, t.dtype, " or ".join(str(d) for d in dtypes)))
    if t.numel() < elems:
        raise ValueError("%s: %d elements, the call needs at least %d"
                         % (name, t.numel(), elems))


def _mat(t, name, dtypes):
    """A 2-D operand: checks its dtype and returns its shape."""
    if t is None or t.dim() != 2:
        raise ValueError("%s: a 2-D tensor is required" % name)
    _arg(t, name, dtypes, 0)
    return t.shape


def _slice_elems(rows, K):
    # host copy of i8_outlier_slice_elems: ceil(K/64) chunks of rows x 64 fp16
    return (K + 63) // 64 * rows * 64


def _check_weight(CB, SCB, K, codes):
    N, Kc = _mat(CB, "CB", codes)
    if Kc != K:
        raise ValueError("CB has %d columns, X has %d" % (Kc, K))
    _arg(SCB, "SCB", _dt("float32"), N)
    return N


def _check_forward(X, CB, SCB, bias, C, codes):
    T, K = _mat(X, "X", _dt("float16"))
    N = _check_weight(CB, SCB, K, codes)
    if bias is not None:
        _arg(bias, "bias", _dt("float16"), N)
    _arg(C, "C", _dt("float16"), T * N)
    return T, K, N


def _check_act_outputs(T, K, col_mask, mask_words, outlier_idx, n_outliers, Xq, SCx, X_o,
                       codes):
    w32 = _dt("int32", "uint32")
    _arg(col_mask, "col_mask", w32, mask_words)
    _arg(outlier_idx, "outlier_idx", w32, K)
    _arg(n_outliers, "n_outliers", w32, 1)
    _arg(Xq, "Xq", codes, T * K)
    _arg(SCx, "SCx", _dt("float32"), T)
    _arg(X_o, "X_o", _dt("float16"), _slice_elems(T, K))


def _stream(stream):
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream


# ----------------------------------------------------------------- the C calls
def i8_quantize_weight(W, CB, SCB, stream=None):
    N, K = _mat(W, "W", _dt("float16"))
    _arg(CB, "CB", _dt("int8"), N * K)
    _arg(SCB, "SCB", _dt("float32"), N)
    _check("i8_quantize_weight",
           load().i8_quantize_weight(_ptr(W), N, K, _ptr(CB), _ptr(SCB), _stream(stream)))


def i8_outlier_scan(X, threshold, col_mask, outlier_idx, n_outliers, stream=None):
    T, K = _mat(X, "X", _dt("float16"))
    w32 = _dt("int32", "uint32")
    _arg(col_mask, "col_mask", w32, (K + 31) // 32)
    _arg(outlier_idx, "outlier_idx", w32, K)
    _arg(n_outliers, "n_outliers", w32, 1)
    _check("i8_outlier_scan",
           load().i8_outlier_scan(_ptr(X), T, K, float(threshold), _ptr(col_mask),
                                  _ptr(outlier_idx), _ptr(n_outliers), _stream(stream)))


def i8_outlier_slice_elems(rows, K) -> int:
    return int(load().i8_outlier_slice_elems(rows, K))


def i8_quantize_act(X, col_mask, outlier_idx, n_outliers, Xq, SCx, X_o, stream=None):
    T, K = _mat(X, "X", _dt("float16"))
    _check_act_outputs(T, K, col_mask, (K + 31) // 32, outlier_idx, n_outliers, Xq, SCx, X_o,
                       _dt("int8"))
    _check("i8_quantize_act",
           load().i8_quantize_act(_ptr(X), T, K, _ptr(col_mask), _ptr(outlier_idx),
                                  _ptr(n_outliers), _ptr(Xq), _ptr(SCx), _ptr(X_o),
                                  _stream(stream)))


def i8_prepare_act(X, threshold, col_mask, outlier_idx, n_outliers, Xq, SCx, X_o, stream=None):
    """col_mask needs ceil(K/32) + 1 words (the last is scratch)."""
    T, K = _mat(X, "X", _dt("float16"))
    _check_act_outputs(T, K, col_mask, (K + 31) // 32 + 1, outlier_idx, n_outliers, Xq, SCx,
                       X_o, _dt("int8"))
    _check("i8_prepare_act",
           load().i8_prepare_act(_ptr(X), T, K, float(threshold), _ptr(col_mask),
                                 _ptr(outlier_idx), _ptr(n_outliers), _ptr(Xq), _ptr(SCx),
                                 _ptr(X_o), _stream(stream)))


def i8_linear_workspace_size(T, N, K) -> int:
    return int(load().i8_linear_workspace_size(T, N, K))


FORWARD_KERNELS = {0: "decode_kernel", 1: "i8_gemm_tcgen05_kernel", 2: "i8_gemm_wide_kernel"}


def i8_forward_kernel(T, N, K) -> str:
    """Name of the product kernel i8_linear_forward runs for these sizes on this device."""
    kind = ctypes.c_int32(-1)
    _check("i8_forward_kernel", load().i8_forward_kernel(T, N, K, ctypes.addressof(kind)))
    return FORWARD_KERNELS[kind.value]


def i8_linear_forward(X, CB, SCB, bias, threshold, C, workspace, stream=None):
    T, K, N = _check_forward(X, CB, SCB, bias, C, _dt("int8"))
    _check("i8_linear_forward",
           load().i8_linear_forward(_ptr(X), T, K, _ptr(CB), _ptr(SCB), _ptr(bias), N,
                                    float(threshold), _ptr(C), _ptr(workspace),
                                    workspace.numel() * workspace.element_size(),
                                    _stream(stream)))


def i8_linear_forward_noalloc(X, CB, SCB, bias, threshold, C, stream=None):
    """i8_linear_forward with the library's fixed 32 MiB device scratch (no workspace)."""
    T, K, N = _check_forward(X, CB, SCB, bias, C, _dt("int8"))
    _check("i8_linear_forward_noalloc",
           load().i8_linear_forward_noalloc(_ptr(X), T, K, _ptr(CB), _ptr(SCB), _ptr(bias), N,
                                            float(threshold), _ptr(C), _stream(stream)))


def i8_quantize_weight_e4m3(W, CB, SCB, stream=None):
    """e4m3 variant of i8_quantize_weight: CB is a uint8 [N, K] tensor of e4m3 codes."""
    N, K = _mat(W, "W", _dt("float16"))
    _arg(CB, "CB", _dt("uint8", "float8_e4m3fn"), N * K)
    _arg(SCB, "SCB", _dt("float32"), N)
    _check("i8_quantize_weight_e4m3",
           load().i8_quantize_weight_e4m3(_ptr(W), N, K, _ptr(CB), _ptr(SCB), _stream(stream)))


def i8_prepare_act_e4m3(X, threshold, col_mask, outlier_idx, n_outliers, Xq, SCx, X_o,
                        stream=None):
    T, K = _mat(X, "X", _dt("float16"))
    _check_act_outputs(T, K, col_mask, (K + 31) // 32 + 1, outlier_idx, n_outliers, Xq, SCx,
                       X_o, _dt("uint8", "float8_e4m3fn"))
    _check("i8_prepare_act_e4m3",
           load().i8_prepare_act_e4m3(_ptr(X), T, K, float(threshold), _ptr(col_mask),
                                      _ptr(outlier_idx), _ptr(n_outliers), _ptr(Xq), _ptr(SCx),
                                      _ptr(X_o), _stream(stream)))


def i8_linear_workspace_size_e4m3(T, N, K) -> int:
    return int(load().i8_linear_workspace_size_e4m3(T, N, K))


def i8_linear_forward_e4m3(X, CB, SCB, bias, threshold, C, workspace, stream=None):
    T, K, N = _check_forward(X, CB, SCB, bias, C, _dt("uint8", "float8_e4m3fn"))
    _check("i8_linear_forward_e4m3",
           load().i8_linear_forward_e4m3(_ptr(X), T, K, _ptr(CB), _ptr(SCB), _ptr(bias), N,
                                         float(threshold), _ptr(C), _ptr(workspace),
                                         workspace.numel() * workspace.element_size(),
                                         _stream(stream)))


def i8_outlier_cache_size(N, K, max_cols) -> int:
    return int(load().i8_outlier_cache_size(N, K, max_cols))


def i8_outlier_cache_reset(cache, stream=None):
    _check("i8_outlier_cache_reset",
           load().i8_outlier_cache_reset(_ptr(cache), cache.numel() * cache.element_size(),
                                         _stream(stream)))


def i8_linear_forward_cached(X, CB, SCB, bias, threshold, C, workspace, cache, stream=None):
    """i8_linear_forward keeping the weight's outlier-column codes in `cache` across calls."""
    T, K, N = _check_forward(X, CB, SCB, bias, C, _dt("int8"))
    _check("i8_linear_forward_cached",
           load().i8_linear_forward_cached(_ptr(X), T, K, _ptr(CB), _ptr(SCB), _ptr(bias), N,
                                           float(threshold), _ptr(C), _ptr(workspace),
                                           workspace.numel() * workspace.element_size(),
                                           _ptr(cache), cache.numel() * cache.element_size(),
                                           _stream(stream)))


def i8_igemm_s32(A, B, acc, workspace, stream=None):
    T, K = _mat(A, "A", _dt("int8"))
    N, Kb = _mat(B, "B", _dt("int8"))
    if Kb != K:
        raise ValueError("B has %d columns, A has %d" % (Kb, K))
    _arg(acc, "acc", _dt("int32"), T * N)
    _check("i8_igemm_s32",
           load().i8_igemm_s32(_ptr(A), T, K, _ptr(B), N, _ptr(acc), _ptr(workspace),
                               workspace.numel() * workspace.element_size(), _stream(stream)))


def i8_linear_backward_input(dY, W, dX, stream=None):
    """dX[T, K] = dY[T, N] W[N, K] (fp16, tensor cores, fp32 sums)."""
    T, N = _mat(dY, "dY", _dt("float16"))
    Nw, K = _mat(W, "W", _dt("float16"))
    if Nw != N:
        raise ValueError("W has %d rows, dY has %d columns" % (Nw, N))
    _arg(dX, "dX", _dt("float16"), T * K)
    _check("i8_linear_backward_input",
           load().i8_linear_backward_input(_ptr(dY), T, N, _ptr(W), K, _ptr(dX),
                                           _stream(stream)))


def i8_linear_backward_weight(dY, X, dW, stream=None):
    """dW[N, K] = dY[T, N]^T X[T, K] (fp16, tensor cores, fp32 sums)."""
    T, N = _mat(dY, "dY", _dt("float16"))
    Tx, K = _mat(X, "X", _dt("float16"))
    if Tx != T:
        raise ValueError("X has %d rows, dY has %d" % (Tx, T))
    _arg(dW, "dW", _dt("float16"), N * K)
    _check("i8_linear_backward_weight",
           load().i8_linear_backward_weight(_ptr(dY), _ptr(X), T, N, K, _ptr(dW),
                                            _stream(stream)))


def i8_bias_grad(dY, db, stream=None):
    """db[N] = sum over rows of dY[T, N] (fp32 sums, fp16 result)."""
    T, N = _mat(dY, "dY", _dt("float16"))
    _arg(db, "db", _dt("float16"), N)
    _check("i8_bias_grad", load().i8_bias_grad(_ptr(dY), T, N, _ptr(db), _stream(stream)))


def i8_dequantize_weight(CB, SCB, W, stream=None):
    """W[N, K] fp16 = CB * SCB / 127 (int8 codes) or the e4m3 codes' values * SCB / 448
    (uint8 / float8_e4m3fn codes)."""
    N, K = _mat(CB, "CB", _dt("int8", "uint8", "float8_e4m3fn"))
    _arg(SCB, "SCB", _dt("float32"), N)
    _arg(W, "W", _dt("float16"), N * K)
    import torch
    fn = "i8_dequantize_weight" if CB.dtype == torch.int8 else "i8_dequantize_weight_e4m3"
    _check(fn, getattr(load(), fn)(_ptr(CB), _ptr(SCB), N, K, _ptr(W), _stream(stream)))


def i8_sync_status(stream=None) -> int:
    """Returns the raw status code (0 = I8_OK); see STATUS."""
    return int(load().i8_sync_status(_stream(stream)))


def i8_set_profile_events(start=None, stop=None):
    s = None if start is None else start.cuda_event
    e = None if stop is None else stop.cuda_event
    if (start is not None and not s) or (stop is not None and not e):
        raise ValueError("record a torch.cuda.Event once before passing it: torch creates "
                         "the CUDA event lazily")
    _check("i8_set_profile_events", load().i8_set_profile_events(s, e))


def i8_selftest_bounded_wait(limit_ns, stream=None):
    _check("i8_selftest_bounded_wait",
           load().i8_selftest_bounded_wait(int(limit_ns), _stream(stream)))


# ----------------------------------------------------------------- allocating helpers
class Linear8bit:
    """A decomposed int8 linear layer holding CB/SCB/bias and a workspace (device memory
    from PyTorch); forward() is one i8_linear_forward call."""

    def __init__(self, W, bias=None, threshold: float = 6.0, stream=None):
        import torch
        N, K = W.shape
        self.N, self.K = N, K
        self.threshold = float(threshold)
        self.CB = torch.empty((N, K), dtype=torch.int8, device=W.device)
        self.SCB = torch.empty((N,), dtype=torch.float32, device=W.device)
        self.bias = bias
        i8_quantize_weight(W, self.CB, self.SCB, stream)
        self._ws = None

    def workspace(self, T):
        import torch
        need = i8_linear_workspace_size(T, self.N, self.K)
        if self._ws is None or self._ws.numel() < need:
            self._ws = torch.empty((need,), dtype=torch.uint8, device=self.CB.device)
        return self._ws

    def forward(self, X, out=None, stream=None):
        import torch
        T = X.shape[0]
        if out is None:
            out = torch.empty((T, self.N), dtype=torch.float16, device=X.device)
        i8_linear_forward(X, self.CB, self.SCB, self.bias, self.threshold, out,
                          self.workspace(T), stream)
        return out
