"""Pins for the CPU oracle: checks against what the pages and the mathematics fix.

Each pin raises AssertionError on failure.  They are collected by test_oracle_pins.py and
re-run by test_oracle_mutations.py against copies of the oracle with a planted mistake,
to show that every such mistake trips at least one pin.

Sources: "A Gentle Introduction to 8-bit Matrix Multiplication for transformers at
scale" (Hugging Face blog, Chinese translation), sections "零点量化", "absmax 量化",
"LLM.int8() 的总结", "内部的 MatMul" and "用法".
"""
import math
from fractions import Fraction

import numpy as np

from oracle import oracle as O
from tests.conftest import read_golden
from bit_matmul_decomposition_b200 import synth


def _f16(vals):
    return np.array(vals, dtype=np.float16)


# ---------------------------------------------------------------- format decoding

def pin_half_to_float_exhaustive():
    """The oracle's own binary16 decoder against numpy's cast, for all 65536 patterns."""
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ref = bits.view(np.float16).astype(np.float32)
    got = np.array([O.half_to_float(int(b)) for b in bits[::1]], np.float32)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan])
    assert np.array_equal(np.signbit(got[~nan]), np.signbit(ref[~nan]))


# ---------------------------------------------------------------- page examples

def pin_absmax_page_example():
    """'absmax 量化': [1.2,-0.5,-4.3,1.2,-3.1,0.8,2.4,5.4] -> [28,-12,-101,28,-73,19,56,127]."""
    g = {r[0]: r[1:] for r in read_golden("absmax_example.txt")}
    x = _f16([float(v) for v in g["input"]])[None, :]
    codes, scale = O.absmax_quantize_rows(x)
    assert codes[0].tolist() == [int(v) for v in g["codes"]], codes
    assert scale[0] == np.float32(np.float16(5.4))
    # the printed factor 23.5 is 127/5.4 shown to one decimal
    assert round(127.0 / float(scale[0]), 1) == float(g["scale_printed"][0])


def pin_zero_point_page_example():
    """'零点量化': 0.3 -> 38.1 -> 38 -> 38/127 = 0.2992 with the range [-1, 1]."""
    g = {r[0]: r[1:] for r in read_golden("zero_point_example.txt")}
    x = _f16([float(v) for v in g["input"]])[None, :]
    codes, scale = O.absmax_quantize_rows(x)
    assert codes[0].tolist() == [int(v) for v in g["codes"]]
    rec = codes[0].astype(np.float64) * float(scale[0]) / 127.0
    assert [round(v, 4) for v in rec] == [float(v) for v in g["recovered_printed"]]


def _weight_printout():
    rows = read_golden("weight_printout.txt")
    cols = [int(c) for c in rows[0][1:]]
    out = []
    for r in rows[1:]:
        bar = r.index("|")
        out.append((int(r[0]), [float(v) for v in r[1:bar]], [int(v) for v in r[bar + 1:]]))
    return cols, out


def _fp16_between(lo, hi):
    allpos = np.arange(0x0001, 0x7C00, dtype=np.uint16).view(np.float16)
    f = allpos.astype(np.float32)
    return allpos[(f >= lo) & (f <= hi)]


def pin_weight_printout_rowwise():
    """'用法': each visible row of the printed int8 weight is reproduced by quantising that
    row with ONE absmax (per output channel), the row's max not always being visible.

    A 64-wide row is built from the six visible fp16 values plus one filler entry of
    magnitude a; some fp16 a >= the visible max must give all six printed codes."""
    cols, rows = _weight_printout()
    for r, vals, codes in rows:
        w = _f16(vals)
        vmax = float(np.abs(w.astype(np.float32)).max())
        hit = False
        for a in _fp16_between(vmax, 0.2):
            row = np.zeros((1, 64), np.float16)
            row[0, cols] = w
            row[0, 30] = a
            q, _ = O.absmax_quantize_rows(row)
            if q[0, cols].tolist() == codes:
                hit = True
                break
        assert hit, "printed row %d not reproduced by one per-row absmax" % r


def pin_weight_printout_not_columnwise():
    """The same printout rules out a per-input-column scale: no single absmax explains the
    six printed codes of column 0 (so the per-row pin above is discriminating)."""
    cols, rows = _weight_printout()
    w = _f16([vals[0] for _, vals, _ in rows])
    codes = [c[0] for _, _, c in rows]
    vmax = float(np.abs(w.astype(np.float32)).max())
    for a in _fp16_between(vmax, 0.2):
        col = np.zeros((1, 64), np.float16)
        col[0, :6] = w
        col[0, 30] = a
        q, _ = O.absmax_quantize_rows(col)
        assert q[0, :6].tolist() != codes


# ---------------------------------------------------------------- rounding and degenerate rows

def pin_round_half_away_from_zero():
    """'四舍五入' read as round half away from zero: with absmax 127 the scale is exactly 1,
    so exact halves reach the rounding step unchanged (RNE would give 0, 0, 2, 2, -2)."""
    x = _f16([[127.0, 0.5, -0.5, 2.5, 1.5, -2.5]])
    q, s = O.absmax_quantize_rows(x)
    assert s[0] == 127.0
    assert q[0].tolist() == [127, 1, -1, 3, 2, -3]


def pin_zero_and_all_outlier_rows():
    """A zero row, and a row whose every column is an outlier column, get scale 0 and all
    zero codes (no division is made)."""
    X = _f16([[0.0, 0.0, 0.0, 0.0], [7.0, -9.0, 6.0, 100.0], [0.0, 1.0, -2.0, 0.5]])
    q, s = O.absmax_quantize_rows(X[:1])
    assert s[0] == 0.0 and not q.any()
    flags, words, idx = O.outlier_scan(X[1:2], 6.0)
    assert idx.tolist() == [0, 1, 2, 3]
    q, s = O.absmax_quantize_rows(X[1:2], flags)
    assert s[0] == 0.0 and not q.any()


def pin_codes_reach_127_and_stay_in_range():
    """Absmax invariants: every row with a nonzero scale has a code of +-127 (at its
    absmax), no code exceeds 127 in magnitude, and outlier columns are coded 0."""
    w = synth.Workload("pin", 33, 96, 8, seed=11, fixed_cols=(5, 50, 95))
    X = synth.make_x(w)
    flags, _, idx = O.outlier_scan(X, 6.0)
    q, s = O.absmax_quantize_rows(X, flags)
    assert set(idx.tolist()) >= {5, 50, 95}
    assert np.abs(q.astype(np.int32)).max() <= 127
    assert not q[:, idx].any()
    for t in range(X.shape[0]):
        if s[t] > 0:
            assert 127 in np.abs(q[t].astype(np.int32))


def pin_power_of_two_row_scaling():
    """Scaling a row by 2^j (exact in fp16, kept below the threshold) leaves its codes
    unchanged and scales its absmax by 2^j."""
    X = synth.random_fp16((5, 64), seed=12, sigma=0.5)
    X = np.clip(X, -1.4, 1.4).astype(np.float16)
    q0, s0 = O.absmax_quantize_rows(X)
    for j in (-3, 1, 2):
        Xj = (X.astype(np.float32) * np.float32(2.0 ** j)).astype(np.float16)
        assert np.array_equal(Xj.astype(np.float32), X.astype(np.float32) * 2.0 ** j)
        qj, sj = O.absmax_quantize_rows(Xj)
        assert np.array_equal(qj, q0)
        assert np.array_equal(sj, s0 * np.float32(2.0 ** j))


# ---------------------------------------------------------------- outlier scan

def pin_threshold_boundaries():
    """'6 or larger': |x| = 6 is an outlier, the largest fp16 below 6 is not, the sign does
    not matter; +inf flags only infinite entries; 0 flags every column."""
    below6 = float(np.nextafter(np.float16(6.0), np.float16(0.0)))
    X = _f16([[6.0, below6, -6.0, 1.0, 0.0, -below6, 3.0, 65504.0]])
    _, _, idx = O.outlier_scan(X, 6.0)
    assert idx.tolist() == [0, 2, 7]
    _, _, idx = O.outlier_scan(X, math.inf)
    assert idx.tolist() == []
    Xi = X.copy()
    Xi[0, 3] = np.float16(-np.inf)
    _, _, idx = O.outlier_scan(Xi, math.inf)
    assert idx.tolist() == [3]
    _, _, idx = O.outlier_scan(X, 0.0)
    assert idx.tolist() == list(range(8))


def pin_mask_matches_columnwise_any():
    """The column mask equals numpy's any-over-rows of |X| >= thr; idx is ascending; the
    packed words put column k at bit k % 32 of word k // 32."""
    w = synth.Workload("pin", 37, 200, 8, seed=13, n_fixed=7, random_frac=0.002)
    X = synth.make_x(w)
    for thr in (6.0, 2.5, 9.0):
        flags, words, idx = O.outlier_scan(X, thr)
        ref = (np.abs(X.astype(np.float32)) >= np.float32(thr)).any(axis=0)
        assert np.array_equal(flags.astype(bool), ref)
        assert idx.tolist() == np.nonzero(ref)[0].tolist()
        bits = np.zeros(words.size * 32, bool)
        bits[: ref.size] = ref
        packed = (bits.reshape(-1, 32) * (1 << np.arange(32, dtype=np.uint64))).sum(1)
        assert np.array_equal(words.astype(np.uint64), packed.astype(np.uint64))


# ---------------------------------------------------------------- integer product

def pin_int_matmul_against_numpy():
    """The int8 x int8 -> int32 product against numpy's int64 matmul (non-square shapes,
    B in the [out, in] layout, a row subset)."""
    A = synth.random_int8((7, 96), seed=14)
    B = synth.random_int8((5, 96), seed=15)
    ref = A.astype(np.int64) @ B.astype(np.int64).T
    assert np.array_equal(O.int_matmul(A, B).astype(np.int64), ref)
    rows = np.array([6, 0, 3])
    assert np.array_equal(O.int_matmul(A, B, rows).astype(np.int64), ref[rows])


def pin_int_matmul_extremes():
    """|acc| <= K * 127^2: at K = 14336 the extreme codes still fit in int32; at
    K = 140000 the all-127 product does not, and the oracle reports it."""
    K = 14336
    A = np.full((1, K), 127, np.int8)
    B = np.stack([np.full(K, 127, np.int8), np.full(K, -127, np.int8)])
    assert O.int_matmul(A, B).tolist() == [[K * 16129, -K * 16129]]
    K = 140000
    A = np.full((1, K), 127, np.int8)
    try:
        O.int_matmul(A, A)
    except OverflowError:
        pass
    else:
        raise AssertionError("int32 overflow not reported")


# ---------------------------------------------------------------- whole decomposition

def _linear_case(T, K, N, seed, cols, thr, bias_sigma=0.02):
    w = synth.Workload("pin", T, K, N, seed=seed, fixed_cols=cols, b_sigma=bias_sigma)
    X = synth.make_x(w)
    W = synth.make_w(w)
    b = synth.make_bias(w)
    CB, SCB = O.quantize_weight(W)
    r = O.linear_forward(X, CB, SCB, b, thr)
    return X, W, b, CB, SCB, r


def pin_threshold_zero_is_fp16_gemm():
    """thr = 0 makes every column an outlier column, so the layer reduces to the plain
    product X @ (CB * SCB / 127)^T + bias ('用法': fp16 weights recovered as CB*SCB/127),
    checked against numpy's fp64 matmul."""
    X, W, b, CB, SCB, r = _linear_case(9, 48, 11, 16, (2, 30), 0.0)
    assert r["n_o"] == 48 and not r["Xq"].any() and not r["SCx"].any()
    Wr = CB.astype(np.float64) * SCB.astype(np.float64)[:, None] / 127.0
    ref = X.astype(np.float64) @ Wr.T + b.astype(np.float64)
    assert np.allclose(r["C"], ref, rtol=1e-12, atol=1e-12)


def pin_threshold_inf_is_vectorwise_int8():
    """thr = +inf gives no outliers: the int8 part alone, i.e. the outer-product dequant of
    the int32 product ('absmax 量化', A*B=C paragraph).  Checked through numpy's int64
    matmul of the oracle's codes and the np.outer of the two absmax vectors."""
    X, W, b, CB, SCB, r = _linear_case(6, 64, 10, 17, (4,), math.inf)
    assert r["n_o"] == 0
    acc = r["Xq"].astype(np.int64) @ CB.astype(np.int64).T
    assert np.array_equal(r["acc"].astype(np.int64), acc)
    ref = acc * np.outer(r["SCx"].astype(np.float64), SCB.astype(np.float64)) / 127.0 ** 2
    ref += b.astype(np.float64)
    assert np.allclose(r["C"], ref, rtol=1e-12, atol=1e-12)


def pin_error_bound_against_unquantised_product():
    """Closed-form bound versus the unquantised X W^T + b (numpy fp64).  With codes within
    half a step (plus fp32 slack) of x*127/SCx and w*127/SCB:
      non-outlier k: |x w - x^ w^| <= |x| dW + (|w| + dW) dX,  dX = 0.5001 SCx/127
      outlier k:     |x w - x w^|  <= |x| dW,                    dW = 0.5001 SCB/127
    Shapes are non-square and the bias is large so that a transposed operand, a dropped
    term or a wrong scale breaks the bound."""
    X, W, b, CB, SCB, r = _linear_case(13, 80, 9, 18, (1, 33, 70), 6.0, bias_sigma=3.0)
    assert set(r["idx"].tolist()) >= {1, 33, 70}
    x = X.astype(np.float64)
    w = W.astype(np.float64)
    ref = x @ w.T + b.astype(np.float64)
    out = np.zeros(80, bool)
    out[r["idx"]] = True
    dX = 0.5001 * r["SCx"].astype(np.float64) / 127.0
    dW = 0.5001 * SCB.astype(np.float64) / 127.0
    ax, aw = np.abs(x), np.abs(w)
    bound = ax @ np.ones_like(aw).T * dW[None, :]
    bound += ((aw[:, ~out] + dW[:, None]).sum(1)[None, :]) * dX[:, None]
    bound += 1e-9
    err = np.abs(r["C"] - ref)
    assert (err <= bound).all(), float((err - bound).max())
    # the bound is not vacuous: the outlier columns alone move the result far beyond it
    contrib = np.abs(x[:, out] @ w[:, out].T)
    assert (contrib > 3 * bound).mean() > 0.5


def pin_hand_worked_example():
    """A 1x4 by 4x2 case worked by hand with exact fractions (threshold 6):
      X = [1, 2, 8, -4]: column 2 is the outlier; SCx = 4, scale 127/4 = 31.75;
          codes [32, 64 (63.5 rounds away), 0, -127].
      W row 0 = [1, .5, .25, -1]: SCB 1, codes [127, 64, 32, -127];
      W row 1 = [.5, .5, .5, .5]: SCB .5, codes [127, 127, 127, 127].
      acc = [32*127 + 64*64 + 127*127, 32*127 + 64*127 - 127*127] = [24289, -3937].
      C0 = 24289*4*1/127^2 + 8*32*1/127 + 0       = 129668/16129
      C1 = -3937*4*.5/127^2 + 8*127*.5/127 + 1     = 72771/16129"""
    X = _f16([[1.0, 2.0, 8.0, -4.0]])
    W = _f16([[1.0, 0.5, 0.25, -1.0], [0.5, 0.5, 0.5, 0.5]])
    b = _f16([0.0, 1.0])
    CB, SCB = O.quantize_weight(W)
    assert CB.tolist() == [[127, 64, 32, -127], [127, 127, 127, 127]]
    assert SCB.tolist() == [1.0, 0.5]
    r = O.linear_forward(X, CB, SCB, b, 6.0)
    assert r["idx"].tolist() == [2] and r["SCx"].tolist() == [4.0]
    assert r["Xq"].tolist() == [[32, 64, 0, -127]]
    assert r["acc"].tolist() == [[24289, -3937]]
    exp = [Fraction(129668, 16129), Fraction(72771, 16129)]
    for got, e in zip(r["C"][0], exp):
        assert abs(Fraction(got) - e) < Fraction(1, 10 ** 12)


def pin_column_permutation_invariance():
    """Permuting the input features of X and W together leaves the output unchanged (the
    mask, scales and codes move with the columns)."""
    X, W, b, CB, SCB, r = _linear_case(8, 64, 7, 19, (9, 40), 6.0)
    p = np.random.Generator(np.random.PCG64(5)).permutation(64)
    r2 = O.linear_forward(X[:, p], CB[:, p], SCB, b, 6.0)
    assert np.array_equal(r2["SCx"], r["SCx"])
    assert np.allclose(r2["C"], r["C"], rtol=1e-12, atol=1e-12)


def pin_row_subset_matches_full():
    """Computing a row subset gives exactly the same rows as the full computation (the
    mask and row scales still come from every row)."""
    X, W, b, CB, SCB, r = _linear_case(12, 64, 6, 20, (3,), 6.0)
    rows = np.array([11, 0, 5])
    rs = O.linear_forward(X, CB, SCB, b, 6.0, rows=rows)
    assert np.array_equal(rs["acc"], r["acc"][rows])
    assert np.array_equal(rs["C"], r["C"][rows])


# ---------------------------------------------------------------- e4m3 variant
# The pages name 8-bit floating point only as the next step; the variant keeps every step
# of the decomposition with e4m3 codes (scale 448 / absmax) in place of int8 ones.  The
# pins below tie the e4m3 arithmetic to the format's definition (OCP 8-bit floating point,
# e4m3 "fn": bias 7, 3 fraction bits, max 448, no infinities) through an independent
# library cast and brute force, and the forward to the same closed forms as the int8 one.

def _e4m3_values():
    """The 127 finite non-negative e4m3 values, by code 0x00..0x7E, from torch's cast."""
    import torch
    codes = torch.arange(0, 0x7F, dtype=torch.uint8)
    return codes.view(torch.float8_e4m3fn).float().double().numpy()


def pin_e4m3_decode_against_torch():
    """All 256 codes decode as torch's float8_e4m3fn (NaN exactly at S.1111.111)."""
    import torch
    ref = torch.arange(256, dtype=torch.int32).to(torch.uint8).view(torch.float8_e4m3fn)
    ref = ref.float().double().numpy()
    got = np.array([O.e4m3_to_float(c) for c in range(256)])
    nan = np.isnan(ref)
    assert nan.tolist() == np.isnan(got).tolist() and nan.sum() == 2
    assert np.array_equal(got[~nan], ref[~nan])


def pin_e4m3_encode_against_torch():
    """Encoding (nearest, ties to even) agrees with torch's float8_e4m3fn cast on every
    finite fp16 value below 464 in magnitude, on the exact midpoints between neighbouring
    e4m3 values (the ties), and on random fp32 values."""
    import torch
    h = np.arange(0, 0x10000, dtype=np.uint32).astype(np.uint16).view(np.float16)
    h = h[np.isfinite(h)].astype(np.float32)
    h = h[np.abs(h) < 464.0]
    v = _e4m3_values()
    mids = ((v[1:] + v[:-1]) / 2).astype(np.float32)
    rng = np.random.default_rng(7)
    rnd = (rng.standard_normal(20000) * np.exp2(rng.uniform(-12, 8, 20000))).astype(np.float32)
    rnd = rnd[np.abs(rnd) < 464.0]
    x = np.concatenate([h, mids, -mids, rnd])
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = np.array([O.e4m3_from_float(float(t)) for t in x], np.uint8)
    bad = np.nonzero(got != ref)[0]
    assert bad.size == 0, (x[bad[:5]], got[bad[:5]], ref[bad[:5]])


def pin_e4m3_encode_brute_force():
    """Independent of any library: the code is the nearest of the 127 finite magnitudes
    (ties to the even code), the sign is kept, and 448 and beyond saturate to 448."""
    v = _e4m3_values()
    rng = np.random.default_rng(8)
    xs = np.concatenate([rng.uniform(0, 460, 3000), np.exp2(rng.uniform(-12, 9, 3000)),
                         (v[1:] + v[:-1]) / 2]).astype(np.float32)
    for x in xs[:4000]:
        a = float(abs(x))
        d = np.abs(v - a)
        best = np.nonzero(d == d.min())[0]
        want = best[0] if best.size == 1 else [c for c in best if c % 2 == 0][0]
        if a >= 448.0:
            want = 0x7E
        assert O.e4m3_from_float(float(x)) == want, (x, want)
        assert O.e4m3_from_float(-float(x)) == (want | 0x80 if want else 0x80), x
    assert O.e4m3_from_float(1e6) == 0x7E and O.e4m3_from_float(-1e6) == 0xFE


def pin_e4m3_rows_absmax_and_scaling():
    """Row quantisation: the absmax element codes to +-448 (0x7E / 0xFE), skipped columns
    and zero rows give code 0 and scale 0, and scaling a row by 2^j (exact in fp16) keeps
    its codes and scales its absmax by 2^j."""
    rng = np.random.default_rng(9)
    A = (rng.standard_normal((5, 40)) * 0.7).astype(np.float16)
    A[2] = 0
    A[3, 7] = -2.5          # the largest magnitude of row 3
    skip = np.zeros(40, np.uint8)
    skip[[4, 11]] = 1
    q, s = O.absmax_quantize_rows_e4m3(A, skip)
    assert not q[2].any() and s[2] == 0
    assert not q[:, [4, 11]].any()
    assert q[3, 7] == 0xFE and s[3] == 2.5
    for r in (0, 1, 3, 4):
        kept = np.abs(A[r].astype(np.float32)) * (1 - skip)
        assert s[r] == kept.max()
        k = int(np.argmax(kept))
        assert q[r, k] & 0x7F == 0x7E
    q2, s2 = O.absmax_quantize_rows_e4m3((A.astype(np.float32) * 4).astype(np.float16), skip)
    assert np.array_equal(q2, q) and np.array_equal(s2, s * 4)


def pin_e4m3_hand_worked_example():
    """A 1x4 by 4x2 case worked by hand with exact fractions (threshold 6):
      X = [1, 0.15185546875, 8, -0.5]: column 2 is the outlier; SCx = 1, scale 448;
          0.15185546875 * 448 = 68.03125 lies just past the midpoint 68 of the e4m3 step
          [64, 72], so it codes to 72 (0x69); codes [448, 72, 0, -224] = [7E, 69, 00, F6].
      W row 0 = [1, .5, .25, -1]: SCB 1, codes [448, 224, 112, -448] = [7E, 76, 6E, FE];
      W row 1 = [.5, .5, .5, .5]: SCB .5, scale 896, codes all 448.
      acc = [448*448 + 72*224 + 224*448, 448*448 + 72*448 - 224*448] = [317184, 132608].
      C0 = 317184 * 1 * 1 / 448^2 + 8 * 112 * 1 / 448 + 0
      C1 = 132608 * 1 * .5 / 448^2 + 8 * 448 * .5 / 448 + 1"""
    X = _f16([[1.0, 0.15185546875, 8.0, -0.5]])
    assert float(X[0, 1]) == 0.15185546875
    W = _f16([[1.0, 0.5, 0.25, -1.0], [0.5, 0.5, 0.5, 0.5]])
    b = _f16([0.0, 1.0])
    CB, SCB = O.quantize_weight_e4m3(W)
    assert CB.tolist() == [[0x7E, 0x76, 0x6E, 0xFE], [0x7E] * 4]
    assert SCB.tolist() == [1.0, 0.5]
    r = O.linear_forward_e4m3(X, CB, SCB, b, 6.0)
    assert r["idx"].tolist() == [2] and r["SCx"].tolist() == [1.0]
    assert r["Xq"].tolist() == [[0x7E, 0x69, 0x00, 0xF6]]
    assert r["acc"].tolist() == [[317184.0, 132608.0]]
    exp = [Fraction(317184, 448 ** 2) + Fraction(8 * 112, 448),
           Fraction(132608, 2 * 448 ** 2) + Fraction(8 * 448, 2 * 448) + 1]
    for got, e in zip(r["C"][0], exp):
        assert abs(Fraction(got) - e) < Fraction(1, 10 ** 12)


def _linear_case_e4m3(T, K, N, seed, cols, thr, bias_sigma=0.02):
    w = synth.Workload("pin8", T, K, N, seed=seed, fixed_cols=cols, b_sigma=bias_sigma)
    X, W, b = synth.make_x(w), synth.make_w(w), synth.make_bias(w)
    CB, SCB = O.quantize_weight_e4m3(W)
    return X, W, b, CB, SCB, O.linear_forward_e4m3(X, CB, SCB, b, thr)


def pin_e4m3_threshold_zero_is_fp16_gemm():
    """thr = 0: every column is an outlier column, so the e4m3 layer is the plain product
    X @ (dec(CB) * SCB / 448)^T + bias, against numpy's fp64 matmul."""
    X, W, b, CB, SCB, r = _linear_case_e4m3(9, 48, 11, 26, (2, 30), 0.0)
    assert r["n_o"] == 48 and not r["Xq"].any() and not r["SCx"].any()
    Wr = O.e4m3_decode(CB) * SCB.astype(np.float64)[:, None] / 448.0
    ref = X.astype(np.float64) @ Wr.T + b.astype(np.float64)
    assert np.allclose(r["C"], ref, rtol=1e-12, atol=1e-12)


def pin_e4m3_threshold_inf_is_vectorwise():
    """thr = +inf: the e4m3 part alone.  The exact product equals numpy's fp64 matmul of
    the decoded codes (every partial sum is exact), and the output is its outer-product
    dequantisation by SCx * SCB / 448^2 plus the bias."""
    X, W, b, CB, SCB, r = _linear_case_e4m3(6, 64, 10, 27, (4,), math.inf)
    assert r["n_o"] == 0
    acc = O.e4m3_decode(r["Xq"]) @ O.e4m3_decode(CB).T
    assert np.array_equal(r["acc"], acc)
    ref = acc * np.outer(r["SCx"].astype(np.float64), SCB.astype(np.float64)) / 448.0 ** 2
    ref += b.astype(np.float64)
    assert np.allclose(r["C"], ref, rtol=1e-12, atol=1e-12)


def pin_e4m3_error_bound_against_unquantised_product():
    """Closed-form bound versus the unquantised X W^T + b (numpy fp64).  An e4m3 code is
    within half a step of the scaled value: relative 2^-4 for normal values, 2^-10 absolute
    below 2^-6 (plus fp32 slack), so with e(x) = 2^-4 |x| + 2^-10 SCx / 448:
      non-outlier k: |x w - x^ w^| <= |x| e(w) + (|w| + e(w)) e(x)
      outlier k:     |x w - x w^|  <= |x| e(w)"""
    X, W, b, CB, SCB, r = _linear_case_e4m3(13, 80, 9, 28, (1, 33, 70), 6.0, bias_sigma=3.0)
    assert set(r["idx"].tolist()) >= {1, 33, 70}
    x, w = X.astype(np.float64), W.astype(np.float64)
    ref = x @ w.T + b.astype(np.float64)
    out = np.zeros(80, bool)
    out[r["idx"]] = True
    slack = 1 + 2.0 ** -20
    ex = (2.0 ** -4 * np.abs(x) + 2.0 ** -10 * r["SCx"].astype(np.float64)[:, None] / 448) * slack
    ew = (2.0 ** -4 * np.abs(w) + 2.0 ** -10 * SCB.astype(np.float64)[:, None] / 448) * slack
    ax, aw = np.abs(x), np.abs(w)
    bound = ax @ ew.T                                    # every column: |x| e(w)
    keep = ~out
    bound += ex[:, keep] @ (aw[:, keep] + ew[:, keep]).T  # non-outlier columns: e(x) terms
    bound += 1e-9
    err = np.abs(r["C"] - ref)
    assert (err <= bound).all(), float((err - bound).max())
    # and the bound is not vacuous: dropping the outlier columns breaks it
    contrib = np.abs(x[:, out] @ w[:, out].T)
    assert (contrib > 3 * bound).mean() > 0.5



def pin_e4m3_row_subset_matches_full():
    """The e4m3 forward on a row subset gives exactly the same rows as on all rows (the
    mask and row scales still come from every row, and each selected row keeps its own
    scale)."""
    X, W, b, CB, SCB, r = _linear_case_e4m3(12, 64, 6, 29, (3,), 6.0)
    rows = np.array([11, 0, 5])
    rs = O.linear_forward_e4m3(X, CB, SCB, b, 6.0, rows=rows)
    assert np.array_equal(rs["SCx"], r["SCx"])
    assert np.array_equal(rs["acc"], r["acc"][rows])
    assert np.array_equal(rs["C"], r["C"][rows])

# ---------------------------------------------------------------- training-mode backward
# ("用法": has_fp16_weights=True keeps fp16 weights for int8/fp16 mixed-precision training;
# the gradients pass straight through the quantisation, i.e. they are those of the linear
# map y = x W^T + b.)

def _grad_case():
    X = synth.random_fp16((3, 5), seed=61, sigma=1.0)
    W = synth.random_fp16((4, 5), seed=62, sigma=0.5)
    dY = synth.random_fp16((3, 4), seed=63, sigma=1.0)
    b = synth.random_fp16((4,), seed=64, sigma=0.5)
    return X, W, dY, b


def pin_backward_matches_finite_differences_of_the_linear_map():
    """Each gradient entry equals the central difference of f = sum(dY * (X W^T + b)) along
    that entry (f is linear, so the difference is exact up to fp64 rounding); the forward
    map here is numpy's matmul, never the product dY W the oracle forms."""
    X, W, dY, b = _grad_case()
    x, w, g, bb = (a.astype(np.float64) for a in (X, W, dY, b))

    def f(x_, w_, b_):
        return float((g * (x_ @ w_.T + b_)).sum())

    dX, dW, db = O.linear_backward(X, W, dY)
    h = 2.0 ** -8
    for arr, grad, fn in ((x, dX, lambda a: f(a, w, bb)), (w, dW, lambda a: f(x, a, bb)),
                          (bb, db, lambda a: f(x, w, a))):
        for idx in np.ndindex(arr.shape):
            up, dn = arr.copy(), arr.copy()
            up[idx] += h
            dn[idx] -= h
            fd = (fn(up) - fn(dn)) / (2 * h)
            assert abs(fd - grad[idx]) <= 1e-9 * (1.0 + abs(fd)), (idx, fd, grad[idx])


def pin_backward_one_hot_output_gradient_selects_rows_and_columns():
    """dY with a single 1 at (t, n): dX is row n of W in row t, dW is row t of X in row n,
    db is the unit vector at n."""
    X, W, _, _ = _grad_case()
    dY = np.zeros((3, 4), np.float16)
    dY[2, 1] = 1.0
    dX, dW, db = O.linear_backward(X, W, dY)
    assert np.array_equal(dX[2], W[1].astype(np.float64)) and not dX[:2].any()
    assert np.array_equal(dW[1], X[2].astype(np.float64)) and not np.delete(dW, 1, 0).any()
    assert np.array_equal(db, np.eye(4)[1])


def pin_dequantized_weight_within_half_a_code_step():
    """The recovered weight CB * SCB / 127 lies within half a code step (SCB / 254, plus the
    fp32 product's rounding) of the weight it was quantised from; a row's absmax entry is
    recovered as +-SCB up to that rounding; e4m3 codes within the e4m3 half step (2^-4
    relative, SCB / 448 * 2^-10 absolute)."""
    W = synth.random_fp16((6, 40), seed=65, sigma=0.02)
    W[2] = 0
    w = W.astype(np.float64)
    CB, SCB = O.quantize_weight(W)
    Wd = O.dequantize_weight(CB, SCB).astype(np.float64)
    s = SCB.astype(np.float64)[:, None]
    assert (np.abs(Wd - w) <= s / 254.0 * (1 + 1e-6) + 1e-12).all()
    assert not Wd[2].any()
    k = np.abs(w).argmax(axis=1)
    rows = np.arange(6)
    assert np.allclose(np.abs(Wd[rows, k]), SCB.astype(np.float64), rtol=1e-6)
    C8, S8 = O.quantize_weight_e4m3(W)
    W8 = O.dequantize_weight(C8, S8, e4m3=True).astype(np.float64)
    s8 = S8.astype(np.float64)[:, None]
    assert (np.abs(W8 - w) <= 2.0 ** -4 * np.abs(w) + s8 / 448.0 * 2.0 ** -10 + 1e-12).all()


ALL_PINS = [v for k, v in sorted(globals().items()) if k.startswith("pin_")]
