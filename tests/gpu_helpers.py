"""Shared helpers of the GPU parity tests: run the CUDA path through the C ABI
and compare with the oracle.

Tolerance on Y (the only floating-point output): the GPU sums exact int32 group
partials times fp16 scales in fp32 and rounds once to fp16, so its error is the
fp16 output rounding (<= 2^-11 = 4.9e-4 relative) plus fp32 rounding of G
products (<= G 2^-24 of the sum of |terms|).  The bar is 2e-3 relative:
per element |Y - Y_ref| <= 2e-3 |Y_ref| + 2e-3 rms(Y_ref of that token), and
||Y - Y_ref||_2 <= 2e-3 ||Y_ref||_2 over the compared set.
"""
import numpy as np
import torch

from mixed_precision_quantized_mx_b200 import binding as mx

RTOL = 2e-3


def dev():
    return torch.device("cuda", 0)


def to_dev(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a)).to(dev())


def gpu_quant(X: np.ndarray):
    Xd = to_dev(X)
    M, K = X.shape
    Aq = torch.empty((M, K), dtype=torch.int8, device=dev())
    sa = torch.empty((M,), dtype=torch.float16, device=dev())
    mx.mx_quant_act(Xd, Aq, sa)
    torch.cuda.synchronize()
    return Aq, sa


def gpu_quant_grouped(X: np.ndarray, act_group: int):
    """Group-wise codes and scales: Aq [M, K], s_a [M, K / act_group] (or [M] for 0)."""
    Xd = to_dev(X)
    M, K = X.shape
    Aq = torch.empty((M, K), dtype=torch.int8, device=dev())
    sa = torch.empty((M, K // act_group) if act_group else (M,), dtype=torch.float16, device=dev())
    mx.mx_quant_act_grouped(Xd, Aq, sa, act_group)
    torch.cuda.synchronize()
    return Aq, sa


def gpu_pack(W: np.ndarray, is8: np.ndarray, group: int, n8: int | None = None, status=None):
    N, K = W.shape
    n8 = int(is8.sum()) if n8 is None else n8
    L = mx.mx_layout_init(N, K, group, n8)
    blob = torch.empty(L.total_bytes, dtype=torch.uint8, device=dev())
    mx.mx_pack_weights(L, to_dev(W), to_dev(is8.astype(np.uint8)), blob, status=status)
    torch.cuda.synchronize()
    return L, blob


def gpu_gemm(L, blob, Aq, sa, path=0, split=0, debug=False, ldy=None):
    M = Aq.shape[0]
    ldy = ldy or L.N
    Yfull = torch.full((M, ldy), float("nan"), dtype=torch.float16, device=dev())
    Y = Yfull[:, :L.N]
    ws_bytes = mx.mx_gemm_workspace_size(L, M, path=path, split=split)
    ws = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device=dev())
    P = None
    if debug:                      # guard zones on both sides catch writes outside P
        pad = 64
        Pbig = torch.full((M * L.N * L.G + 2 * pad,), -12345, dtype=torch.int32, device=dev())
        P = Pbig[pad:pad + M * L.N * L.G].view(M, L.N, L.G)
        P.zero_()
    mx.mx_gemm(L, blob, Aq, sa, Y, workspace=ws, path=path, split=split, debug_partials=P)
    torch.cuda.synchronize()
    if debug:
        assert (Pbig[:pad] == -12345).all() and (Pbig[-pad:] == -12345).all()
    return Y, P, Yfull


def f16bits(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().view(torch.int16).numpy().view(np.uint16)


def assert_y_close(Y16: np.ndarray, Yref: np.ndarray, rows_rms: np.ndarray | None = None):
    Y = Y16.astype(np.float64)
    assert np.isfinite(Y).all()
    err = np.abs(Y - Yref)
    if rows_rms is None:
        rows_rms = np.sqrt(np.mean(Yref ** 2, axis=-1, keepdims=True)) if Yref.ndim == 2 \
            else np.sqrt(np.mean(Yref ** 2))
    bound = RTOL * np.abs(Yref) + RTOL * rows_rms
    bad = err > bound
    assert not bad.any(), f"{bad.sum()} elements out of tolerance; worst {np.max(err - bound)}"
    assert np.linalg.norm(Y - Yref) <= RTOL * np.linalg.norm(Yref)
