"""The kernels round an absmax code without a float-to-int conversion: with
v = fl32(x * fl32(127 / absmax)) and a = |v|, the code's magnitude is
floor(fl_rz(a + 0.5)), read from the bit pattern of fl_rz(fl_rz(a + 0.5) + 1.5 * 2^23).
The byte form the kernels store applies the sign by negating the whole 32-bit pattern:
the low byte of (pattern ^ s) - s, s = 0 or all ones by the sign of v, is the code in two's
complement.  These checks show, on the CPU with IEEE round-toward-zero additions, that both
equal the oracle's roundf (round half away from zero) for every fp32 value the product can
take, of either sign, and that no code needs a clamp."""
import subprocess

import numpy as np

CHECK = r"""
#include <fenv.h>
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <string.h>
#pragma STDC FENV_ACCESS ON
int main(void) {
    float lim = 128.0f;
    uint32_t top;
    memcpy(&top, &lim, 4);
    unsigned long long bad = 0;
    for (uint32_t b = 0; b < top; ++b) {          /* every fp32 value in [0, 128) */
        float a;
        memcpy(&a, &b, 4);
        fesetround(FE_TOWARDZERO);
        volatile float r = a + 0.5f;
        volatile float t = r + 12582912.0f;
        fesetround(FE_TONEAREST);
        float tt = t;
        uint32_t tb;
        memcpy(&tb, &tt, 4);
        if ((int)tb - 0x4B400000 != (int)roundf(a)) ++bad;
        /* the stored byte, for +a and for -a (codes fit a byte for |v| < 127.5; the
           products stay below 127.0000077) */
        for (int neg = 0; neg < 2 && a < 127.5f; ++neg) {
            uint32_t s = neg ? 0xFFFFFFFFu : 0u;
            uint8_t byte = (uint8_t)((tb ^ s) - s);
            int want = (int)roundf(neg ? -a : a);
            if ((int8_t)byte != want) ++bad;
        }
    }
    printf("%llu\n", bad);
    return bad != 0;
}
"""


def test_round_toward_zero_adds_give_half_away_rounding_on_every_fp32_below_128(tmp_path):
    src = tmp_path / "rz.c"
    src.write_text(CHECK, encoding="utf-8")
    exe = tmp_path / "rz"
    subprocess.check_call(["gcc", "-O1", "-frounding-math", str(src), "-o", str(exe), "-lm"])
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=600)
    assert out.returncode == 0 and out.stdout.strip() == "0", out.stdout


def _fp16_positive():
    return np.arange(0x0001, 0x7C00, dtype=np.uint16).view(np.float16).astype(np.float32)


def test_codes_stay_within_127_without_clamp():
    a = _fp16_positive()
    v = (a * (np.float32(127.0) / a)).astype(np.float32)
    assert float(v.max()) < 127.5
