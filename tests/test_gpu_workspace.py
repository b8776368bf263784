"""A workspace shared by calls of different paths and shapes.

The decode kernel keeps its tile arrival counters and the cooperative prologue's mask,
row-maximum and barrier words in the caller's workspace, 64-bit words tagged in their
upper half with the launch's epoch (a process-wide counter).  A word left in the
workspace by anything else -- another call's data, another user of the memory -- whose
upper half happens to equal a launch's epoch would pose as a live counter: a tile would
complete early or never, or a column would turn into a spurious outlier column.  The
library clears those words before every decode launch; these tests check that no leftover
bytes reach the output:

  * words carrying the NEXT launch's epoch are planted in every 8 bytes of the workspace
    (the epoch is read back from the counters a previous launch left at (epoch, 0));
  * a prefill call at K = 65536 and threshold 0 (every column an outlier: its index list
    0, 1, 2, ... lands where the decode path keeps its counters) alternates with a decode
    call on one workspace, and on the fixed array of i8_linear_forward_noalloc, for enough
    calls that the process epoch passes the indices' values;
  * the module front end alternates prefill and decode batches on its cached workspace.

Every decode output is compared bit for bit with a call on a fresh workspace, and with
the oracle ("内部的 MatMul": per-call outlier set and scales).
"""
import ctypes

import numpy as np
import pytest
import torch

from bit_matmul_decomposition_b200 import abi, synth
from oracle import oracle as O
from tests.gpu_util import DEV, check_output, dev, gpu_quantize_weight, host, sync_ok

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    abi.load()
    yield
    torch.cuda.synchronize()


def _layer(T, K, N, cols, seed, thr=6.0):
    w = synth.Workload("ws", T, K, N, seed=seed, fixed_cols=tuple(cols) or None)
    X, W, b = synth.make_x(w), synth.make_w(w), synth.make_bias(w)
    return X, W, b


def _fresh_forward(X_d, CB, SCB, b_d, thr):
    T, K = X_d.shape
    N = CB.shape[0]
    ws = torch.zeros((abi.i8_linear_workspace_size(T, N, K),), dtype=torch.uint8, device=DEV)
    C = torch.empty((T, N), dtype=torch.float16, device=DEV)
    abi.i8_linear_forward(X_d, CB, SCB, b_d, thr, C, ws)
    return C


def _epoch_left_behind(ws):
    """The epoch of the last decode launch on `ws`.  The decode layout puts the slice
    records first and the control words last (the tile counters, then the cooperative
    prologue's words); a launch clears the control words and writes them only with its own
    epoch, and its tile counters end at (epoch, 0).  The records are scratch: the kernel
    drops them from the L2 once summed, so they may read back as any earlier bytes of the
    memory, (epoch, 0) words of older launches included.  So the last (epoch, 0) word of
    the workspace is one of this launch's control words."""
    words = ws.cpu().numpy().view(np.uint64)
    hi, lo = words >> np.uint64(32), words & np.uint64(0xFFFFFFFF)
    at = np.nonzero((lo == 0) & (hi > 0) & (hi < (1 << 24)))[0]
    assert at.size > 0, "no counter found"
    return int(hi[at[-1]])


@pytest.mark.parametrize("T,K,N,cols", [
    (1, 4096, 700, (5, 4000)),      # per-CTA prologue
    (8, 4096, 1000, (7,)),          # per-CTA prologue, two token groups of 4
    (16, 4608, 1000, (10, 2000)),   # 2*T*K > 128 KB: cooperative prologue (grid barriers)
])
def test_decode_ignores_words_tagged_with_its_own_epoch(T, K, N, cols):
    X, W, b = _layer(T, K, N, cols, seed=T + 77)
    CB, SCB = gpu_quantize_weight(dev(W))
    X_d, b_d = dev(X), dev(b)
    ref = _fresh_forward(X_d, CB, SCB, b_d, 6.0)
    nbytes = abi.i8_linear_workspace_size(T, N, K)
    ws = torch.zeros((nbytes,), dtype=torch.uint8, device=DEV)
    C = torch.empty((T, N), dtype=torch.float16, device=DEV)
    abi.i8_linear_forward(X_d, CB, SCB, b_d, 6.0, C, ws)
    sync_ok()
    for step in range(3):
        # the next decode launch in this process takes the epoch after the one left behind;
        # every 8 bytes get (that epoch, 1): one phantom arrival, mask bit 0 set, a row
        # maximum of 1.4e-45, one barrier arrival
        nxt = _epoch_left_behind(ws) + 1
        pattern = np.full(nbytes // 8, (nxt << 32) | 1, dtype=np.uint64)
        ws.copy_(torch.from_numpy(pattern.view(np.uint8)).to(DEV))
        C = torch.full((T, N), float("nan"), dtype=torch.float16, device=DEV)
        abi.i8_linear_forward(X_d, CB, SCB, b_d, 6.0, C, ws)
        sync_ok()
        assert torch.equal(C.view(torch.int16), ref.view(torch.int16)), step
        assert _epoch_left_behind(ws) == nxt
    CBr, SCBr = O.quantize_weight(W)
    check_output(host(ref), O.linear_forward(X, CBr, SCBr, b, 6.0)["C"])


def _noalloc(X, CB, SCB, b, thr, C):
    T, K = X.shape
    N = CB.shape[0]
    return abi.load().i8_linear_forward_noalloc(
        X.data_ptr(), T, K, CB.data_ptr(), SCB.data_ptr(), None if b is None else b.data_ptr(),
        N, ctypes.c_float(thr), C.data_ptr(), torch.cuda.current_stream().cuda_stream)


@pytest.mark.parametrize("scratch", ["workspace", "noalloc"])
def test_prefill_index_ramp_then_decode_on_one_scratch(scratch):
    K, N = 65536, 32
    Tp, Td = 32, 8
    Xp = synth.random_fp16((Tp, K), seed=11)
    Xd, W, b = _layer(Td, K, N, (3, 40000), seed=12)
    CB, SCB = gpu_quantize_weight(dev(W))
    Xp_d, Xd_d, b_d = dev(Xp), dev(Xd), dev(b)
    ref_d = _fresh_forward(Xd_d, CB, SCB, b_d, 6.0)
    ref_p = _fresh_forward(Xp_d, CB, SCB, b_d, 0.0)
    sync_ok()
    nbytes = max(abi.i8_linear_workspace_size(Tp, N, K), abi.i8_linear_workspace_size(Td, N, K))
    ws = torch.empty((nbytes,), dtype=torch.uint8, device=DEV)
    Cp = torch.empty((Tp, N), dtype=torch.float16, device=DEV)
    Cd = torch.empty((Td, N), dtype=torch.float16, device=DEV)
    bad = torch.zeros((), dtype=torch.int64, device=DEV)
    iters = 7000
    for i in range(iters):
        if scratch == "workspace":
            abi.i8_linear_forward(Xp_d, CB, SCB, b_d, 0.0, Cp, ws)   # idx = 0 .. 65535
            abi.i8_linear_forward(Xd_d, CB, SCB, b_d, 6.0, Cd, ws)
        else:
            assert _noalloc(Xp_d, CB, SCB, b_d, 0.0, Cp) == 0
            assert _noalloc(Xd_d, CB, SCB, b_d, 6.0, Cd) == 0
        bad += (Cd.view(torch.int16) != ref_d.view(torch.int16)).any()
        if i % 1000 == 999:
            bad += (Cp.view(torch.int16) != ref_p.view(torch.int16)).any()
    sync_ok()
    assert int(bad) == 0
    CBr, SCBr = O.quantize_weight(W)
    check_output(host(ref_d), O.linear_forward(Xd, CBr, SCBr, b, 6.0)["C"])


def test_module_alternates_prefill_and_decode_batches():
    from bit_matmul_decomposition_b200.linear import Linear8bitLt
    K, N = 2048, 600
    W = synth.random_fp16((N, K), seed=21, sigma=0.02)
    b = synth.random_fp16((N,), seed=22, sigma=0.02)
    lin = torch.nn.Linear(K, N, bias=True).to(DEV).half()
    with torch.no_grad():
        lin.weight.copy_(dev(W))
        lin.bias.copy_(dev(b))
    m = Linear8bitLt.from_linear(lin, threshold=6.0)
    CBr, SCBr = O.quantize_weight(W)
    assert np.array_equal(host(m.CB), CBr)
    for i in range(12):
        T = 40 if i % 2 == 0 else 5
        X = synth.plant_columns(synth.random_fp16((T, K), seed=100 + i),
                                (3 + i, 1000 + 7 * i), seed=200 + i)
        y = m(dev(X))
        sync_ok()
        check_output(host(y), O.linear_forward(X, CBr, SCBr, b, 6.0)["C"])
