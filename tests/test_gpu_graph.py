"""The forward captured in a CUDA graph and replayed with new inputs written in place.

A captured launch keeps its kernel arguments, the decode kernel's launch epoch included,
so every replay must start from workspace words that the previous replay left behind: the
tile counters and the cooperative prologue's mask, row-maximum and barrier words have to
be back in a state that the next replay reads as empty.  Each replay is checked against
the oracle, with outlier sets that change from replay to replay (columns that were
outliers in the previous replay and are not now must not leak into the mask).
"""
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


def _x(T, K, cols, seed):
    w = synth.Workload("graph", T, K, 8, seed=seed, fixed_cols=tuple(cols) or None)
    return synth.make_x(w)


CASES = [
    # T, K, N, outlier sets of the successive replays
    (1, 4096, 700, [(5,), (77, 4000), (), (5,)]),                 # decode, per-CTA prologue
    (16, 14336, 300, [(3, 9000), (100,), (3, 9000), (14335,)]),   # decode, cooperative
    (9, 8000, 333, [(1, 4000, 7999), (2,), (1, 4000, 7999)]),     # decode, cooperative
    (300, 1040, 600, [(5, 200), (9,), (), (5, 200, 1039)]),       # prepare + GEMM
]


@pytest.mark.parametrize("cached", [False, True], ids=["plain", "outlier_cache"])
@pytest.mark.parametrize("T,K,N,sets", CASES)
def test_graph_replays_match_the_oracle(T, K, N, sets, cached):
    w = synth.Workload("graph_w", 4, K, N, seed=T + N)
    W, b = synth.make_w(w), synth.make_bias(w)
    CB, SCB = gpu_quantize_weight(dev(W))
    bias = dev(b)
    CBr, SCBr = O.quantize_weight(W)
    X_d = dev(_x(T, K, sets[0], seed=1))
    C = torch.empty((T, N), dtype=torch.float16, device=DEV)
    ws = torch.empty((abi.i8_linear_workspace_size(T, N, K),), dtype=torch.uint8, device=DEV)
    cache = None
    if cached:
        cache = torch.empty((abi.i8_outlier_cache_size(N, K, 64),), dtype=torch.uint8,
                            device=DEV)
        abi.i8_outlier_cache_reset(cache)

    def fwd():
        if cached:
            abi.i8_linear_forward_cached(X_d, CB, SCB, bias, 6.0, C, ws, cache)
        else:
            abi.i8_linear_forward(X_d, CB, SCB, bias, 6.0, C, ws)

    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        fwd()                                 # one-time setup outside the capture
    torch.cuda.current_stream().wait_stream(side)
    sync_ok()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fwd()
    for r, cols in enumerate(sets * 2):
        X = _x(T, K, cols, seed=10 + r)
        X_d.copy_(dev(X))
        C.fill_(float("nan"))
        g.replay()
        torch.cuda.synchronize()
        sync_ok()
        ref = O.linear_forward(X, CBr, SCBr, b, 6.0)["C"]
        check_output(host(C), ref)
    del g
