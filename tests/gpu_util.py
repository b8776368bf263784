"""Helpers for the GPU parity tests: device buffers, the stage calls of the C ABI, and the
output tolerance.

Tolerance (fp16 output): per row t,
    max_n |C[t,n] - C_ref[t,n]| <= 2^-9 * max_n |C_ref[t,n]| + 1e-3
with C_ref the oracle's fp64 result.  The int8/int32 stages are compared bit for bit.
"""
import numpy as np
import torch

from bit_matmul_decomposition_b200 import abi

DEV = "cuda"


def dev(a: np.ndarray) -> torch.Tensor:
    if a.dtype == np.float16:
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.float16).to(DEV)
    return torch.from_numpy(np.ascontiguousarray(a)).to(DEV)


def host(t: torch.Tensor) -> np.ndarray:
    t = t.detach().cpu()
    if t.dtype == torch.float16:
        return t.view(torch.int16).numpy().view(np.float16)
    if t.dtype == torch.uint32:
        return t.view(torch.int32).numpy().view(np.uint32)
    return t.numpy()


def sync_ok():
    st = abi.i8_sync_status()
    assert st == 0, abi.STATUS.get(st, st)


def gpu_quantize_weight(W_d):
    N, K = W_d.shape
    CB = torch.empty((N, K), dtype=torch.int8, device=DEV)
    SCB = torch.empty((N,), dtype=torch.float32, device=DEV)
    abi.i8_quantize_weight(W_d, CB, SCB)
    return CB, SCB


def gpu_scan(X_d, thr):
    T, K = X_d.shape
    words = (K + 31) // 32
    mask = torch.empty((words,), dtype=torch.int32, device=DEV)
    idx = torch.empty((K,), dtype=torch.int32, device=DEV)
    n_o = torch.empty((4,), dtype=torch.int32, device=DEV)
    abi.i8_outlier_scan(X_d, thr, mask, idx, n_o)
    return mask, idx, n_o


def gpu_quantize_act(X_d, mask, idx, n_o):
    T, K = X_d.shape
    Xq = torch.empty((T, K), dtype=torch.int8, device=DEV)
    SCx = torch.empty((T,), dtype=torch.float32, device=DEV)
    X_o = torch.full((abi.i8_outlier_slice_elems(T, K),), float("nan"), dtype=torch.float16,
                     device=DEV)
    abi.i8_quantize_act(X_d, mask, idx, n_o, Xq, SCx, X_o)
    return Xq, SCx, X_o


def gpu_prepare(X_d, thr):
    """The fused one-pass scan + quantisation (i8_prepare_act)."""
    T, K = X_d.shape
    words = (K + 31) // 32
    mask = torch.empty((words + 1,), dtype=torch.int32, device=DEV)
    idx = torch.empty((K,), dtype=torch.int32, device=DEV)
    n_o = torch.empty((4,), dtype=torch.int32, device=DEV)
    Xq = torch.empty((T, K), dtype=torch.int8, device=DEV)
    SCx = torch.empty((T,), dtype=torch.float32, device=DEV)
    X_o = torch.full((abi.i8_outlier_slice_elems(T, K),), float("nan"), dtype=torch.float16,
                     device=DEV)
    abi.i8_prepare_act(X_d, thr, mask, idx, n_o, Xq, SCx, X_o)
    return mask[:words], idx, n_o, Xq, SCx, X_o


def gpu_forward(X_d, CB, SCB, bias_d, thr):
    T, K = X_d.shape
    N = CB.shape[0]
    ws = torch.empty((abi.i8_linear_workspace_size(T, N, K),), dtype=torch.uint8, device=DEV)
    C = torch.full((T, N), float("nan"), dtype=torch.float16, device=DEV)
    abi.i8_linear_forward(X_d, CB, SCB, bias_d, thr, C, ws)
    return C


def gpu_igemm(A_d, B_d):
    T, K = A_d.shape
    N = B_d.shape[0]
    ws = torch.empty((abi.i8_linear_workspace_size(T, N, K),), dtype=torch.uint8, device=DEV)
    acc = torch.empty((T, N), dtype=torch.int32, device=DEV)
    abi.i8_igemm_s32(A_d, B_d, acc, ws)
    return acc


def slice_to_matrix(X_o_flat: np.ndarray, rows: int, K: int, n_o: int) -> np.ndarray:
    """Chunk-major outlier slice -> [rows, round_up(n_o, 64)] (includes the zero pad)."""
    chunks = (K + 63) // 64
    s = X_o_flat.reshape(chunks, rows, 64)
    used = (n_o + 63) // 64
    return np.concatenate([s[c] for c in range(used)], axis=1) if used else np.zeros((rows, 0),
                                                                                      s.dtype)


def check_output(C: np.ndarray, C_ref: np.ndarray):
    """Row-wise tolerance; returns the worst ratio err / allowed (must be <= 1)."""
    C = C.astype(np.float64)
    assert np.isfinite(C).all(), "non-finite output"
    err = np.abs(C - C_ref).max(axis=1)
    allowed = 2.0 ** -9 * np.abs(C_ref).max(axis=1) + 1e-3
    ratio = float((err / allowed).max())
    assert (err <= allowed).all(), "tolerance exceeded: worst err/allowed = %.3f" % ratio
    return ratio
