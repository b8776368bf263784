"""ctypes view of the plain-C oracle (i8_oracle.c) -- test infrastructure only.

Each function takes and returns numpy arrays; fp16 data is passed as its raw bits.
The arithmetic lives entirely in i8_oracle.c; this file only marshals arguments.
"""
import ctypes
import numpy as np

from . import build as _build

_lib = None
_override = None


class use_library:
    """Context manager: route every call to another build of i8_oracle.c (a copy with a
    planted mistake, compiled by a test) and restore the normal build afterwards."""

    def __init__(self, path):
        self.path = path

    def __enter__(self):
        global _override
        self._saved = _override
        _override = _load(self.path)
        return self

    def __exit__(self, *exc):
        global _override
        _override = self._saved
        return False


def lib():
    global _lib
    if _override is not None:
        return _override
    if _lib is None:
        _lib = _load(_build.build())
    return _lib


def _load(path):
    L = ctypes.CDLL(path)
    P = ctypes.c_void_p
    i64 = ctypes.c_int64
    L.oracle_half_to_float.argtypes = [ctypes.c_uint16]
    L.oracle_half_to_float.restype = ctypes.c_float
    L.oracle_outlier_scan.argtypes = [P, i64, i64, ctypes.c_float, P, P, P, P]
    L.oracle_outlier_scan.restype = None
    L.oracle_absmax_quantize_rows.argtypes = [P, i64, i64, P, P, P]
    L.oracle_absmax_quantize_rows.restype = None
    L.oracle_int_matmul.argtypes = [P, P, i64, P, i64, i64, P]
    L.oracle_int_matmul.restype = i64
    L.oracle_decomposed_output.argtypes = [P, i64, P, i64, P, P, P, P, P, i64, P,
                                           ctypes.c_int32, P]
    L.oracle_decomposed_output.restype = None
    L.oracle_linear_forward_rows.argtypes = [P, i64, i64, P, P, P, i64, ctypes.c_float,
                                             P, i64, P, P, P, P, P, P, P]
    L.oracle_linear_forward_rows.restype = i64
    L.oracle_linear_backward.argtypes = [P, P, P, i64, i64, i64, P, P, P]
    L.oracle_linear_backward.restype = None
    L.oracle_dequantize_weight.argtypes = [P, P, i64, i64, ctypes.c_int32, P]
    L.oracle_dequantize_weight.restype = None
    L.oracle_e4m3_to_double.argtypes = [ctypes.c_uint8]
    L.oracle_e4m3_to_double.restype = ctypes.c_double
    L.oracle_e4m3_from_float.argtypes = [ctypes.c_float]
    L.oracle_e4m3_from_float.restype = ctypes.c_uint8
    L.oracle_absmax_quantize_rows_e4m3.argtypes = [P, i64, i64, P, P, P]
    L.oracle_absmax_quantize_rows_e4m3.restype = None
    L.oracle_e4m3_matmul.argtypes = [P, P, i64, P, i64, i64, P]
    L.oracle_e4m3_matmul.restype = None
    L.oracle_linear_forward_rows_e4m3.argtypes = [P, i64, i64, P, P, P, i64, ctypes.c_float,
                                                  P, i64, P, P, P, P, P, P, P]
    L.oracle_linear_forward_rows_e4m3.restype = i64
    L.oracle_num_threads.argtypes = []
    L.oracle_num_threads.restype = ctypes.c_int
    return L


def _ptr(a):
    return None if a is None else a.ctypes.data


def _bits(a):
    a = np.ascontiguousarray(a)
    if a.dtype == np.float16:
        return a.view(np.uint16)
    assert a.dtype == np.uint16, a.dtype
    return a


def num_threads() -> int:
    return lib().oracle_num_threads()


def half_to_float(bits: int) -> float:
    return lib().oracle_half_to_float(int(bits))


def outlier_scan(X, threshold):
    """Step 1: returns (is_outlier uint8 [K], mask_words uint32 [ceil(K/32)], idx int32 [n_o])."""
    Xb = _bits(X)
    T, K = Xb.shape
    flags = np.zeros(K, np.uint8)
    words = np.zeros((K + 31) // 32, np.uint32)
    idx = np.zeros(max(K, 1), np.int32)
    n_o = np.zeros(1, np.int32)
    lib().oracle_outlier_scan(_ptr(Xb), T, K, float(threshold), _ptr(flags), _ptr(words),
                              _ptr(idx), _ptr(n_o))
    return flags, words, idx[: int(n_o[0])].copy()


def absmax_quantize_rows(A, skip=None):
    """Steps 2/3: returns (codes int8 [R,K], scale float32 [R])."""
    Ab = _bits(A)
    R, K = Ab.shape
    q = np.zeros((R, K), np.int8)
    s = np.zeros(R, np.float32)
    sk = None if skip is None else np.ascontiguousarray(skip, dtype=np.uint8)
    lib().oracle_absmax_quantize_rows(_ptr(Ab), R, K, _ptr(sk), _ptr(q), _ptr(s))
    return q, s


def quantize_weight(W):
    """Step 3: per-output-channel quantisation of W [N,K] -> (CB int8 [N,K], SCB float32 [N])."""
    return absmax_quantize_rows(W, None)


def int_matmul(A, B, rows=None):
    """Step 4: acc int32 [len(rows) or A.shape[0], N]; raises on int32 overflow."""
    A = np.ascontiguousarray(A, np.int8)
    B = np.ascontiguousarray(B, np.int8)
    K = A.shape[1]
    assert B.shape[1] == K
    r = None if rows is None else np.ascontiguousarray(rows, np.int64)
    nrows = A.shape[0] if r is None else r.shape[0]
    N = B.shape[0]
    acc = np.zeros((nrows, N), np.int32)
    ov = lib().oracle_int_matmul(_ptr(A), _ptr(B), nrows, _ptr(r), N, K, _ptr(acc))
    if ov:
        raise OverflowError("int32 accumulator overflow in %d results" % ov)
    return acc


def linear_forward(X, CB, SCB, bias, threshold, rows=None):
    """Whole forward (steps 1,2 over all rows; 4-6 for `rows`, default all rows).

    Returns a dict with mask_words, idx, n_o, Xq, SCx, acc (rows) and C (fp64, rows).
    """
    Xb = _bits(X)
    T, K = Xb.shape
    CB = np.ascontiguousarray(CB, np.int8)
    SCB = np.ascontiguousarray(SCB, np.float32)
    N = CB.shape[0]
    bb = None if bias is None else _bits(bias)
    r = None if rows is None else np.ascontiguousarray(rows, np.int64)
    nrows = T if r is None else r.shape[0]
    words = np.zeros((K + 31) // 32, np.uint32)
    idx = np.zeros(max(K, 1), np.int32)
    n_o = np.zeros(1, np.int32)
    Xq = np.zeros((T, K), np.int8)
    SCx = np.zeros(T, np.float32)
    acc = np.zeros((nrows, N), np.int32)
    C = np.zeros((nrows, N), np.float64)
    ov = lib().oracle_linear_forward_rows(_ptr(Xb), T, K, _ptr(CB), _ptr(SCB), _ptr(bb), N,
                                          float(threshold), _ptr(r), nrows, _ptr(words),
                                          _ptr(idx), _ptr(n_o), _ptr(Xq), _ptr(SCx),
                                          _ptr(acc), _ptr(C))
    if ov < 0:
        raise MemoryError("oracle allocation failed")
    if ov:
        raise OverflowError("int32 accumulator overflow in %d results" % ov)
    n = int(n_o[0])
    return dict(mask_words=words, idx=idx[:n].copy(), n_o=n, Xq=Xq, SCx=SCx, acc=acc, C=C)


# ------------------------------------------------------------------- e4m3 variant
def e4m3_to_float(code: int) -> float:
    return lib().oracle_e4m3_to_double(int(code) & 0xFF)


def e4m3_from_float(v: float) -> int:
    return int(lib().oracle_e4m3_from_float(float(v)))


def e4m3_decode(codes):
    """Exact values (float64) of an array of e4m3 codes."""
    table = np.array([e4m3_to_float(c) for c in range(256)], np.float64)
    return table[np.asarray(codes, np.uint8)]


def absmax_quantize_rows_e4m3(A, skip=None):
    """Row-wise absmax e4m3 codes: returns (codes uint8 [R,K], scale float32 [R])."""
    Ab = _bits(A)
    R, K = Ab.shape
    q = np.zeros((R, K), np.uint8)
    s = np.zeros(R, np.float32)
    sk = None if skip is None else np.ascontiguousarray(skip, dtype=np.uint8)
    lib().oracle_absmax_quantize_rows_e4m3(_ptr(Ab), R, K, _ptr(sk), _ptr(q), _ptr(s))
    return q, s


def quantize_weight_e4m3(W):
    """Per-output-channel e4m3 quantisation of W [N,K] -> (CB uint8 [N,K], SCB float32 [N])."""
    return absmax_quantize_rows_e4m3(W, None)


def e4m3_matmul(A, B, rows=None):
    """Exact product of e4m3 code matrices: float64 [len(rows) or A.shape[0], N]."""
    A = np.ascontiguousarray(A, np.uint8)
    B = np.ascontiguousarray(B, np.uint8)
    K = A.shape[1]
    assert B.shape[1] == K
    r = None if rows is None else np.ascontiguousarray(rows, np.int64)
    nrows = A.shape[0] if r is None else r.shape[0]
    N = B.shape[0]
    acc = np.zeros((nrows, N), np.float64)
    lib().oracle_e4m3_matmul(_ptr(A), _ptr(B), nrows, _ptr(r), N, K, _ptr(acc))
    return acc


def linear_forward_e4m3(X, CB, SCB, bias, threshold, rows=None):
    """The e4m3 forward (mask and SCx over all rows; product and output for `rows`).

    Returns a dict with mask_words, idx, n_o, Xq (uint8 codes), SCx, acc (fp64) and C.
    """
    Xb = _bits(X)
    T, K = Xb.shape
    CB = np.ascontiguousarray(CB, np.uint8)
    SCB = np.ascontiguousarray(SCB, np.float32)
    N = CB.shape[0]
    bb = None if bias is None else _bits(bias)
    r = None if rows is None else np.ascontiguousarray(rows, np.int64)
    nrows = T if r is None else r.shape[0]
    words = np.zeros((K + 31) // 32, np.uint32)
    idx = np.zeros(max(K, 1), np.int32)
    n_o = np.zeros(1, np.int32)
    Xq = np.zeros((T, K), np.uint8)
    SCx = np.zeros(T, np.float32)
    acc = np.zeros((nrows, N), np.float64)
    C = np.zeros((nrows, N), np.float64)
    st = lib().oracle_linear_forward_rows_e4m3(_ptr(Xb), T, K, _ptr(CB), _ptr(SCB), _ptr(bb),
                                               N, float(threshold), _ptr(r), nrows,
                                               _ptr(words), _ptr(idx), _ptr(n_o), _ptr(Xq),
                                               _ptr(SCx), _ptr(acc), _ptr(C))
    if st < 0:
        raise MemoryError("oracle allocation failed")
    n = int(n_o[0])
    return dict(mask_words=words, idx=idx[:n].copy(), n_o=n, Xq=Xq, SCx=SCx, acc=acc, C=C)


def linear_backward(X, W, dY):
    """Backward of y = x W^T + b straight through the quantisation, fp64: returns
    (dX [T,K], dW [N,K], db [N]).  X may be None (no dW) and W may be None (no dX)."""
    dY = np.ascontiguousarray(_bits(dY))
    T, N = dY.shape
    Xb = None if X is None else np.ascontiguousarray(_bits(X))
    Wb = None if W is None else np.ascontiguousarray(_bits(W))
    K = Xb.shape[1] if Xb is not None else (Wb.shape[1] if Wb is not None else 0)
    assert Xb is None or Xb.shape == (T, K)
    assert Wb is None or Wb.shape == (N, K)
    dX = None if Wb is None else np.empty((T, K), np.float64)
    dW = None if Xb is None else np.empty((N, K), np.float64)
    db = np.empty((N,), np.float64)
    lib().oracle_linear_backward(_ptr(Xb), _ptr(Wb), _ptr(dY), T, N, K, _ptr(dX), _ptr(dW),
                                 _ptr(db))
    return dX, dW, db


def dequantize_weight(CB, SCB, e4m3=False):
    """The recovered weight in fp32 (CB * fl32(SCB / 127), or e4m3 values * fl32(SCB / 448))."""
    CB = np.ascontiguousarray(CB).view(np.uint8)
    SCB = np.ascontiguousarray(SCB, np.float32)
    N, K = CB.shape
    W = np.empty((N, K), np.float32)
    lib().oracle_dequantize_weight(_ptr(CB), _ptr(SCB), N, K, 1 if e4m3 else 0, _ptr(W))
    return W
