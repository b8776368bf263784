"""The kernels round an absmax code as trunc(fl32(v + copysign(0.5, v))) with
v = fl32(x * fl32(127 / absmax)).  That equals round-half-away-from-zero for every |v|
below 2^22 except |v| = 0.5 - 2^-25, and needs no clamp while |v| < 127.5.  These checks
show, on the CPU, that no fp16 input reaches either exception: the kernels' shortcut and
the oracle's roundf agree on every input the layer can see."""
import numpy as np


def _fp16_positive():
    return np.arange(0x0001, 0x7C00, dtype=np.uint16).view(np.float16).astype(np.float32)


def test_no_fp16_pair_reaches_the_rounding_exception():
    target = np.float32(0.5) - np.float32(2.0 ** -25)
    xs = _fp16_positive()
    for a in xs:
        s = np.float32(127.0) / a
        lo = (a / np.float32(254.0)) * np.float32(1 - 2 ** -8)
        hi = (a / np.float32(254.0)) * np.float32(1 + 2 ** -8)
        i0 = np.searchsorted(xs, lo)
        i1 = np.searchsorted(xs, hi, side="right")
        if i1 > i0:
            v = (xs[i0:i1] * s).astype(np.float32)
            assert not (v == target).any()


def test_codes_stay_within_127_without_clamp():
    a = _fp16_positive()
    v = (a * (np.float32(127.0) / a)).astype(np.float32)
    assert float(v.max()) < 127.5


def test_add_half_truncate_matches_half_away_on_a_dense_grid():
    # every fp32 value in [0, 128) on a fine grid, plus the exact half-integers
    v = np.concatenate([np.arange(0, 2 ** 22, dtype=np.uint32).view(np.float32)[1:],
                        np.linspace(0, 127.999, 2000001, dtype=np.float32),
                        np.arange(0, 128, dtype=np.float32) + np.float32(0.5)])
    v = v[(v < 128) & np.isfinite(v)]
    v = v[v != np.float32(0.5) - np.float32(2.0 ** -25)]
    fast = np.trunc((v + np.float32(0.5)).astype(np.float32))
    exact = np.floor(v.astype(np.float64) + 0.5)
    assert np.array_equal(fast, exact)
