"""Host-side checks of the C ABI that need no GPU: the library builds and loads, exports
every function include/i8linear.h declares, and rejects bad arguments before touching
CUDA (validation runs before any device call)."""
import ctypes
import math
import os
import re

import pytest

from bit_matmul_decomposition_b200 import abi, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "i8linear.h")

INVALID = 1


def declared_functions():
    text = open(HEADER, encoding="utf-8").read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*[A-Za-z_][\w\s\*]*?\b(i8_\w+)\s*\(", text, flags=re.M)))


@pytest.fixture(scope="module")
def lib():
    build.build()
    return abi.load()


def test_header_declares_the_four_layer_calls():
    names = declared_functions()
    for n in ("i8_quantize_weight", "i8_outlier_scan", "i8_quantize_act", "i8_linear_forward"):
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    names = declared_functions()
    assert len(names) >= 10
    for n in names:
        assert hasattr(lib, n), n
        assert n in abi.SIGNATURES, "binding lacks %s" % n
    assert set(abi.SIGNATURES) == set(names)


def test_status_strings(lib):
    for code, name in abi.STATUS.items():
        assert lib.i8_status_string(code).decode() == name


def test_workspace_size_host_logic(lib):
    ws = lib.i8_linear_workspace_size
    assert ws(0, 64, 64) == 0 and ws(16, 0, 64) == 0 and ws(16, 64, 0) == 0
    assert ws(16, 64, 72) == 0                      # K % 16 != 0
    prefill = ws(2048, 16384, 4096)
    # X_o + CB_o slices dominate: 64 chunks x (2048 + 16384) rows x 64 x 2 bytes
    assert prefill >= 64 * (2048 + 16384) * 64 * 2 + 2048 * 4096
    assert prefill % 256 == 0
    decode = ws(16, 57344, 14336)
    assert decode >= 4 * 16 * 57344 * 4             # K-slice partial sums
    assert lib.i8_outlier_slice_elems(10, 65) == 2 * 10 * 64
    assert lib.i8_outlier_slice_elems(10, 64) == 10 * 64


def test_forward_kernel_query_host_logic(lib):
    # decode sizes are decided without a device; invalid sizes and a NULL result are refused
    assert abi.i8_forward_kernel(1, 64, 64) == "decode_kernel"
    assert abi.i8_forward_kernel(16, 57344, 14336) == "decode_kernel"
    assert abi.i8_forward_kernel(4, 33, 65536) == "decode_kernel"
    for T, N, K in [(0, 64, 64), (16, 0, 64), (16, 64, 72)]:
        with pytest.raises(abi.I8Error) as e:
            abi.i8_forward_kernel(T, N, K)
        assert e.value.code == 1
    assert lib.i8_forward_kernel(1, 64, 64, None) == 1


FAKE = 0x10000  # aligned, never dereferenced: validation rejects before any launch


def test_forward_rejects_bad_arguments_without_cuda(lib):
    f = lib.i8_linear_forward
    ws_ok = lib.i8_linear_workspace_size(32, 64, 64)
    good = dict(X=FAKE, T=32, K=64, CB=FAKE, SCB=FAKE, bias=None, N=64, thr=6.0, C=FAKE,
                ws=FAKE, wsb=ws_ok, s=None)

    def call(**kw):
        a = dict(good, **kw)
        return f(a["X"], a["T"], a["K"], a["CB"], a["SCB"], a["bias"], a["N"], a["thr"],
                 a["C"], a["ws"], a["wsb"], a["s"])

    assert call(X=None) == INVALID
    assert call(C=None) == INVALID
    assert call(ws=None) == INVALID
    assert call(X=FAKE + 4) == INVALID               # misaligned
    assert call(bias=FAKE + 2) == INVALID
    assert call(T=0) == INVALID
    assert call(T=-5) == INVALID
    assert call(N=0) == INVALID
    assert call(K=72) == INVALID                     # K % 16
    assert call(thr=math.nan) == INVALID
    assert call(wsb=ws_ok - 1) == INVALID


def test_other_calls_reject_bad_arguments_without_cuda(lib):
    assert lib.i8_quantize_weight(None, 64, 64, FAKE, FAKE, None) == INVALID
    assert lib.i8_quantize_weight(FAKE, 64, 40, FAKE, FAKE, None) == INVALID
    assert lib.i8_outlier_scan(FAKE, 4, 64, math.nan, FAKE, FAKE, FAKE, None) == INVALID
    assert lib.i8_outlier_scan(FAKE, 4, 64, 6.0, None, FAKE, FAKE, None) == INVALID
    assert lib.i8_quantize_act(FAKE, 4, 64, FAKE, FAKE, FAKE, FAKE, FAKE, None, None) == INVALID
    assert lib.i8_igemm_s32(FAKE, 4, 64, FAKE, 8, FAKE, FAKE, 0, None) == INVALID
    assert lib.i8_igemm_s32(FAKE, 4, 140000, FAKE, 8, FAKE, FAKE, 1 << 40, None) == INVALID
    assert lib.i8_selftest_bounded_wait(10, None) == INVALID


def test_product_path_fails_loudly_without_library(tmp_path):
    saved = abi._lib
    abi._lib = None
    try:
        with pytest.raises(OSError):
            abi.load(str(tmp_path / "missing.so"))
    finally:
        abi._lib = saved


def test_outlier_cache_size_host_logic(lib):
    cs = lib.i8_outlier_cache_size
    assert cs(0, 64, 64) == 0 and cs(64, 0, 64) == 0 and cs(64, 72, 64) == 0
    assert cs(64, 64, 0) == 0
    head = 256                                        # 8 + 2 mask words, padded to 256 B
    assert cs(64, 64, 1) == head + 64 * 64 * 2        # rounded up to one 64-column chunk
    assert cs(64, 64, 1000) == head + 64 * 64 * 2     # at most K rounded up to 64
    assert cs(300, 1040, 65) == head + 2 * 300 * 64 * 2
    big = cs(16384, 4096, 256)                        # header: 8 + 128 words -> 768 B
    assert big == 768 + 4 * 16384 * 64 * 2


def test_cached_forward_rejects_bad_arguments_without_cuda(lib):
    f = lib.i8_linear_forward_cached
    ws_ok = lib.i8_linear_workspace_size(32, 64, 64)
    c_ok = lib.i8_outlier_cache_size(64, 64, 64)

    def call(cache=FAKE, cb=c_ok, X=FAKE, T=32, thr=6.0):
        return f(X, T, 64, FAKE, FAKE, None, 64, thr, FAKE, FAKE, ws_ok, cache, cb, None)

    assert call(cache=None) == INVALID
    assert call(cache=FAKE + 8) == INVALID            # misaligned
    assert call(cb=c_ok - 1) == INVALID               # less than one 64-column chunk
    assert call(X=None) == INVALID
    assert call(T=0) == INVALID
    assert call(thr=math.nan) == INVALID
    assert lib.i8_outlier_cache_reset(None, c_ok, None) == INVALID
    assert lib.i8_outlier_cache_reset(FAKE, 16, None) == INVALID


def test_e4m3_calls_reject_bad_arguments_without_cuda(lib):
    # the e4m3 forward always takes the GEMM path, so its workspace for a decode-size batch
    # is the GEMM layout (outlier slices sized for n_o = K), larger than the decode one
    assert lib.i8_linear_workspace_size_e4m3(8, 4096, 4096) > \
        lib.i8_linear_workspace_size(8, 4096, 4096)
    assert lib.i8_linear_workspace_size_e4m3(2048, 16384, 4096) == \
        lib.i8_linear_workspace_size(2048, 16384, 4096)
    assert lib.i8_linear_workspace_size_e4m3(0, 64, 64) == 0
    assert lib.i8_linear_workspace_size_e4m3(8, 64, 72) == 0
    ws_ok = lib.i8_linear_workspace_size_e4m3(32, 64, 64)
    f = lib.i8_linear_forward_e4m3
    assert f(None, 32, 64, FAKE, FAKE, None, 64, 6.0, FAKE, FAKE, ws_ok, None) == INVALID
    assert f(FAKE, 32, 64, FAKE, FAKE, None, 64, math.nan, FAKE, FAKE, ws_ok, None) == INVALID
    assert f(FAKE, 32, 64, FAKE, FAKE, None, 64, 6.0, FAKE, FAKE, ws_ok - 1, None) == INVALID
    assert f(FAKE, 32, 72, FAKE, FAKE, None, 64, 6.0, FAKE, FAKE, ws_ok, None) == INVALID
    assert lib.i8_quantize_weight_e4m3(FAKE, 64, 40, FAKE, FAKE, None) == INVALID
    assert lib.i8_quantize_weight_e4m3(None, 64, 64, FAKE, FAKE, None) == INVALID
    assert lib.i8_prepare_act_e4m3(FAKE, 4, 64, 6.0, FAKE, FAKE, FAKE, None, FAKE, FAKE,
                                   None) == INVALID


def test_header_serves_a_plain_c_caller(lib, tmp_path):
    """The boundary is a C ABI: a C99 program (no C++, no CUDA headers) includes
    i8linear.h with every warning on, links against the library and calls it; the call
    with NULL pointers is refused before any CUDA work, so this runs without a GPU."""
    src = tmp_path / "caller.c"
    src.write_text(
        '#include "i8linear.h"\n'
        "#include <stdio.h>\n"
        "int main(void) {\n"
        "    size_t ws = i8_linear_workspace_size(2048, 16384, 4096);\n"
        "    i8_status s = i8_linear_forward(NULL, 4, 64, NULL, NULL, NULL, 8, 6.0f, NULL,\n"
        "                                    NULL, 0, NULL);\n"
        '    printf("%zu %s\\n", ws, i8_status_string(s));\n'
        "    return (s == I8_ERR_INVALID_ARG && ws > 0) ? 0 : 1;\n"
        "}\n", encoding="utf-8")
    exe = tmp_path / "caller"
    libdir = os.path.dirname(abi.LIB_PATH)
    import subprocess
    subprocess.check_call(["gcc", "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror",
                           "-I", os.path.join(ROOT, "include"), str(src),
                           "-L", libdir, "-l:libi8linear.so", "-Wl,-rpath," + libdir,
                           "-o", str(exe)])
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert out.returncode == 0, out.stdout + out.stderr
    ws, name = out.stdout.split()
    assert int(ws) == lib.i8_linear_workspace_size(2048, 16384, 4096)
    assert name == "I8_ERR_INVALID_ARG"
