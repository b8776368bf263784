"""Parity at the workloads' full sizes, through the same i8_linear_forward calls that
bench.py times.

For every workload: CB/SCB compared bit for bit over the whole weight; mask, index list,
count, Xq and SCx bit for bit over all of X, from the two-pass calls (i8_outlier_scan,
i8_quantize_act) and from the fused prepare pass that the forward runs (i8_prepare_act,
whose fp16 outlier slice X_o is compared too).  The fp16 output is compared with the
oracle: in full on the OPT-6.7B FFN-up layer; elsewhere on every row and column of the
four corner 256 x 256 output tiles (the GEMM's first and last m-tile against its first
and last n-tile) plus sampled rows x sampled columns -- the oracle computes each output
from its own row of X and its own output channel, so a sample is exact.  Tolerance per
row:  max|C - C_ref| <= 2^-9 * max_row|C_ref| + 1e-3.
"""
import math

import numpy as np
import pytest
import torch

from bit_matmul_decomposition_b200 import abi, synth
from oracle import oracle as O
from tests.gpu_util import (check_output, dev, gpu_forward, gpu_prepare, gpu_quantize_act,
                            gpu_quantize_weight, gpu_scan, host, slice_to_matrix, sync_ok)

pytestmark = [pytest.mark.gpu, pytest.mark.slow]

_WCACHE = {}


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    abi.load()
    yield
    _WCACHE.clear()
    torch.cuda.empty_cache()


def _weights(w):
    """W, bias on host; CB/SCB on device (GPU-quantised, checked once against the oracle)."""
    key = (w.N, w.K, w.seed)
    if key not in _WCACHE:
        _WCACHE.clear()
        torch.cuda.empty_cache()
        W = synth.make_w(w)
        b = synth.make_bias(w)
        W_d = dev(W)
        CB, SCB = gpu_quantize_weight(W_d)
        del W_d
        sync_ok()
        CBr, SCBr = O.quantize_weight(W)
        assert np.array_equal(host(CB), CBr), "CB differs from the oracle"
        assert np.array_equal(host(SCB).view(np.uint32), SCBr.view(np.uint32))
        del W
        _WCACHE[key] = (CB, SCB, CBr, SCBr, b)
    return _WCACHE[key]


def _sample(n, extra, count, seed):
    rng = np.random.Generator(np.random.PCG64(seed))
    s = set(int(i) for i in extra if 0 <= i < n)
    s.update(int(i) for i in rng.choice(n, size=min(n, count), replace=False))
    return np.array(sorted(s), np.int64)


def _edges(n, tile=256):
    """Every index of the first and the last `tile`-wide tile of [0, n)."""
    return list(range(min(n, tile))) + list(range(max(0, n - tile), n))


def _run(w, n_rows=12, n_cols=768, full=False):
    CB, SCB, CBr, SCBr, b = _weights(w)
    X = synth.make_x(w)
    X_d = dev(X)
    flags, words, idx_r = O.outlier_scan(X, w.threshold)
    Xq_r, SCx_r = O.absmax_quantize_rows(X, flags)
    n = idx_r.size
    planted = synth.outlier_columns(w)
    if not math.isinf(w.threshold):
        assert set(planted.tolist()) <= set(idx_r.tolist())
    # the two-pass stage calls, in full
    mask, idx, n_o = gpu_scan(X_d, w.threshold)
    Xq, SCx, _ = gpu_quantize_act(X_d, mask, idx, n_o)
    sync_ok()
    assert int(host(n_o)[0]) == n
    assert np.array_equal(host(mask).view(np.uint32), words)
    assert np.array_equal(host(idx)[:n], idx_r)
    assert np.array_equal(host(SCx).view(np.uint32), SCx_r.view(np.uint32))
    assert np.array_equal(host(Xq), Xq_r)
    del Xq, SCx, mask, idx, n_o
    # the fused prepare pass, in full (the forward's own first launch on the GEMM path)
    mask, idx, n_o, Xq, SCx, X_o = gpu_prepare(X_d, w.threshold)
    sync_ok()
    assert int(host(n_o)[0]) == n
    assert np.array_equal(host(mask).view(np.uint32), words)
    assert np.array_equal(host(idx)[:n], idx_r)
    assert np.array_equal(host(SCx).view(np.uint32), SCx_r.view(np.uint32))
    assert np.array_equal(host(Xq), Xq_r)
    got_o = slice_to_matrix(host(X_o), w.T, w.K, n)
    assert np.array_equal(got_o[:, :n].view(np.uint16), X[:, idx_r].view(np.uint16))
    assert not got_o[:, n:].view(np.uint16).any()
    del Xq, SCx, mask, idx, n_o, X_o, got_o
    torch.cuda.empty_cache()
    # the forward
    b_d = None if b is None else dev(b)
    C = gpu_forward(X_d, CB, SCB, b_d, w.threshold)
    sync_ok()
    if full:
        r = O.linear_forward(X, CBr, SCBr, b, w.threshold)
        assert r["n_o"] == n
        check_output(host(C), r["C"])
        return n
    rows = _sample(w.T, [0, 127, 128, w.T - 1] + _edges(w.T), n_rows, w.seed + 1)
    cols = _sample(w.N, [0, 255, 256, 511, w.N - 1] + _edges(w.N), n_cols, w.seed + 2)
    Cs = host(C[torch.from_numpy(rows).cuda()][:, torch.from_numpy(cols).cuda()])
    r = O.linear_forward(X, CBr[cols], SCBr[cols], None if b is None else b[cols],
                         w.threshold, rows=rows)
    assert r["n_o"] == n
    check_output(Cs, r["C"])
    return n


def test_opt_ffn_up_prefill_2048x4096x16384():
    n = _run(synth.opt_ffn_up_prefill(), full=True)
    assert n >= 6


@pytest.mark.parametrize("T", [1, 8, 16])
def test_bloom_ffn_decode_Tx14336x57344(T):
    n = _run(synth.bloom_ffn_decode(T), n_rows=T, n_cols=2048)
    assert n >= 8


def test_bloom_qkv_prefill_4096x14336x43008():
    n = _run(synth.bloom_qkv_prefill(), n_rows=8, n_cols=512)
    # 8 fixed columns plus 0.01% random entries >= 6 in 4096 rows: about a third of the
    # 14336 columns become outlier columns
    assert 3000 < n < 7000


@pytest.mark.parametrize("cols", [0, 8, 64, 256])
@pytest.mark.parametrize("thr", [6.0, math.inf])
def test_opt175b_sweep_8192x12288x49152(cols, thr):
    n = _run(synth.opt175b_sweep(cols, thr), n_rows=8, n_cols=512)
    if math.isinf(thr):
        assert n == 0
    else:
        assert n >= cols
