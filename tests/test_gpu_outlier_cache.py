"""Outlier cache (i8_linear_forward_cached) against the oracle and the uncached forward.

The cached forward must give the uncached forward's output bit for bit, whatever state the
cache is in: empty, keyed to this call's outlier set (hit: the gather is skipped), keyed to
another set or weight (miss: gathered into the cache, which is re-keyed), or too small for
this call's set (gathered into the workspace; the cache keeps its key).  The header words
are read back to check which of these happened; a poisoned slice shows that a hit reads the
cache and that a miss rewrites it.
"""
import math

import numpy as np
import pytest
import torch

from bit_matmul_decomposition_b200 import abi, synth
from oracle import oracle as O
from tests.gpu_util import DEV, check_output, dev, gpu_quantize_weight, host, sync_ok

pytestmark = pytest.mark.gpu

HDR = 8  # header words before the cached mask


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    abi.load()
    yield
    torch.cuda.synchronize()


def _x(T, K, cols, seed, frac=0.0):
    w = synth.Workload("cache", T, K, 8, seed=seed, fixed_cols=tuple(cols) or None,
                       random_frac=frac)
    return synth.make_x(w)


def _weight(N, K, seed):
    w = synth.Workload("cache_w", 4, K, N, seed=seed)
    return synth.make_w(w), synth.make_bias(w)


class _Layer:
    def __init__(self, N, K, seed=11, max_cols=128):
        W, b = _weight(N, K, seed)
        self.W, self.b = W, b
        self.N, self.K = N, K
        self.CB, self.SCB = gpu_quantize_weight(dev(W))
        self.bias = dev(b)
        self.cache = torch.empty((abi.i8_outlier_cache_size(N, K, max_cols),), dtype=torch.uint8,
                                 device=DEV)
        self.cache.fill_(0xA5)   # undefined contents until the reset
        abi.i8_outlier_cache_reset(self.cache)

    def forward(self, X, thr=6.0, cached=True, CB=None):
        X_d = dev(X) if isinstance(X, np.ndarray) else X
        T = X_d.shape[0]
        ws = torch.empty((abi.i8_linear_workspace_size(T, self.N, self.K),), dtype=torch.uint8,
                         device=DEV)
        ws.fill_(0x5A)
        C = torch.full((T, self.N), float("nan"), dtype=torch.float16, device=DEV)
        cb = self.CB if CB is None else CB
        if cached:
            abi.i8_linear_forward_cached(X_d, cb, self.SCB, self.bias, thr, C, ws, self.cache)
        else:
            abi.i8_linear_forward(X_d, cb, self.SCB, self.bias, thr, C, ws)
        return C

    def header(self):
        words = (self.K + 31) // 32
        h = host(self.cache[: 4 * (HDR + words)].view(torch.int32)).view(np.uint32)
        return dict(valid=int(h[0]), n_o=int(h[1]), N=int(h[2]), K=int(h[3]),
                    cb=int(h[4]) | (int(h[5]) << 32), mask=h[HDR:HDR + words].copy())

    def slice_view(self):
        words = (self.K + 31) // 32
        head = (4 * (HDR + words) + 255) // 256 * 256
        return self.cache[head:]


def _mask_words(X, thr, K):
    _, words, _ = O.outlier_scan(X, thr)
    return np.asarray(words, dtype=np.uint32)[: (K + 31) // 32]


def _same(a, b):
    return np.array_equal(host(a).view(np.uint16), host(b).view(np.uint16))


def _check_vs_oracle(L, X, C, thr=6.0):
    CBr, SCBr = O.quantize_weight(L.W)
    r = O.linear_forward(X, CBr, SCBr, L.b, thr)
    check_output(host(C), r["C"])


@pytest.mark.parametrize("T,K,N", [(300, 1040, 600), (40, 4096, 520)])
def test_hit_miss_sequence_matches_uncached(T, K, N):
    L = _Layer(N, K)
    XA = _x(T, K, (5, 200, K - 1), seed=1)          # few columns: per-item gather
    XB = _x(T, K, (9, 1000), seed=2)
    XC = _x(T, K, tuple(range(3, K, K // 80))[:80], seed=3)   # n_o * 32 >= K: row copies
    h0 = L.header()
    assert h0["valid"] == 0
    for X, name in ((XA, "A miss"), (XA, "A hit"), (XB, "B miss"), (XC, "C miss"),
                    (XC, "C hit"), (XA, "A again")):
        C = L.forward(X)
        C_ref = L.forward(X, cached=False)
        sync_ok()
        assert _same(C, C_ref), name
        _check_vs_oracle(L, X, C)
        h = L.header()
        assert h["valid"] == 1, name
        assert np.array_equal(h["mask"], _mask_words(X, 6.0, K)), name
        assert h["n_o"] == int(np.unpackbits(h["mask"].view(np.uint8)).sum())
        assert (h["N"], h["K"], h["cb"]) == (N, K, L.CB.data_ptr())


def test_hit_reads_the_cache_and_a_miss_rewrites_it():
    T, K, N = 300, 1040, 600
    L = _Layer(N, K)
    X = _x(T, K, (17, 512), seed=4)
    C_ref = L.forward(X, cached=False)
    L.forward(X)                                   # miss: fills the cache
    sync_ok()
    L.slice_view().view(torch.int16).fill_(0x7E00)  # fp16 NaN over the cached slice
    C_hit = L.forward(X)
    sync_ok()
    assert torch.isnan(C_hit.float()).all()         # every row has an outlier term
    abi.i8_outlier_cache_reset(L.cache)             # empty again: the next call gathers
    C_miss = L.forward(X)
    sync_ok()
    assert _same(C_miss, C_ref)
    # the same codes at another address: a different key, so a miss and a fresh gather
    L.slice_view().view(torch.int16).fill_(0x7E00)
    CB2 = L.CB.clone()
    C2 = L.forward(X, CB=CB2)
    sync_ok()
    assert _same(C2, C_ref)
    assert L.header()["cb"] == CB2.data_ptr()


def test_set_beyond_capacity_goes_to_the_workspace():
    T, K, N = 200, 2048, 300
    L = _Layer(N, K, max_cols=64)
    XA = _x(T, K, (1, 2, 1500), seed=5)
    XB = _x(T, K, tuple(range(0, 2048, 20))[:100], seed=6)    # 100 columns > 64
    L.forward(XA)
    sync_ok()
    h_before = L.header()
    assert h_before["valid"] == 1 and h_before["n_o"] == 3
    C = L.forward(XB)
    C_ref = L.forward(XB, cached=False)
    sync_ok()
    assert _same(C, C_ref)
    _check_vs_oracle(L, XB, C)
    h = L.header()
    assert h["valid"] == 1 and h["n_o"] == 3
    assert np.array_equal(h["mask"], h_before["mask"])
    C = L.forward(XA)                                # still a hit on the kept set
    C_ref = L.forward(XA, cached=False)
    sync_ok()
    assert _same(C, C_ref)


def test_other_batch_sizes_share_the_cache_and_decode_leaves_it():
    K, N = 1040, 600
    L = _Layer(N, K)
    cols = (33, 700)
    X1 = _x(300, K, cols, seed=7)
    X2 = _x(64, K, cols, seed=8)                     # same outlier set, other tokens
    X3 = _x(9, K, (3,), seed=9)                      # decode batch: no CB_o
    L.forward(X1)
    sync_ok()
    h1 = L.header()
    for X in (X2, X3):
        C = L.forward(X)
        C_ref = L.forward(X, cached=False)
        sync_ok()
        assert _same(C, C_ref)
        _check_vs_oracle(L, X, C)
        h = L.header()
        assert h["valid"] == 1 and np.array_equal(h["mask"], h1["mask"])
    # no outlier columns (threshold +inf): nothing to cache, the key stays
    C = L.forward(X1, thr=math.inf)
    C_ref = L.forward(X1, thr=math.inf, cached=False)
    sync_ok()
    assert _same(C, C_ref)
    assert np.array_equal(L.header()["mask"], h1["mask"])


def test_all_columns_outliers_with_full_capacity():
    T, K, N = 64, 208, 256
    L = _Layer(N, K, max_cols=K)
    X = _x(T, K, (9,), seed=10)
    for _ in range(2):                               # miss, then hit
        C = L.forward(X, thr=0.0)
        C_ref = L.forward(X, thr=0.0, cached=False)
        sync_ok()
        assert _same(C, C_ref)
        _check_vs_oracle(L, X, C, thr=0.0)
        assert L.header()["n_o"] == K
