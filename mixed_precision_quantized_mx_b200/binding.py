"""Thin ctypes binding of the C ABI in include/mx.h.

Argument marshalling only: every function forwards torch tensors' device
pointers, sizes and the current CUDA stream to the function of the same name in
libmx.so.  There is no host-side computation and no fallback: if the library is
missing, or a call fails, an exception is raised.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmx.so")

MX_OK = 0
STATUS_NAMES = {
    0: "MX_OK", 1: "MX_ERR_INVALID_ARG", 2: "MX_ERR_UNSUPPORTED", 3: "MX_ERR_ALIGNMENT",
    4: "MX_ERR_CUDA", 5: "MX_ERR_TIMEOUT", 6: "MX_ERR_BAD_BLOB", 7: "MX_ERR_WORKSPACE",
}
MX_F32, MX_F16 = 0, 1
TILE_ROWS, KBLOCK, HEADER_BYTES = 128, 128, 256
PATH_AUTO, PATH_SPLITK, PATH_TENSOR, PATH_ROWS, PATH_PAIR, PATH_PAIR256, PATH_TC_DECODE = 0, 1, 2, 3, 4, 5, 6

EXPORTED = ("mx_version", "mx_last_error", "mx_layout_init", "mx_layout_from_header",
            "mx_pack_weights", "mx_quant_act", "mx_gemm_workspace_size", "mx_gemm_select_path",
            "mx_gemm", "mx_linear_workspace_size", "mx_linear", "mx_linear_noalloc",
            "mx_quant_act_grouped", "mx_copy_mapped", "mx_saliency", "mx_select_top_workspace_size",
            "mx_select_top", "mx_bw_layout_init", "mx_bw_pack", "mx_bw_gemm")


class MXError(RuntimeError):
    def __init__(self, status: int, fn: str, msg: str):
        super().__init__(f"{fn}: {STATUS_NAMES.get(status, status)}: {msg}")
        self.status = status


class Layout(ctypes.Structure):
    """mirror of mx_layout"""
    _fields_ = [(n, ctypes.c_int32) for n in
                ("N", "K", "group", "n8", "n4", "G", "t8", "t4", "kblocks", "reserved0")] + \
               [(n, ctypes.c_uint64) for n in
                ("off_rowmap", "off_scales8", "off_codes8", "off_scales4", "off_zeros4",
                 "off_codes4", "total_bytes")]


class BwLayout(ctypes.Structure):
    """mirror of mx_bw_layout (block-wise bit widths)"""
    _fields_ = [(n, ctypes.c_int32) for n in ("N", "K", "NB", "KB")] + \
               [("table", ctypes.c_uint8 * 4), ("reserved0", ctypes.c_int32)] + \
               [(n, ctypes.c_uint64) for n in
                ("off_meta", "off_offsets", "off_scales", "off_zeros", "off_codes", "code_bytes", "total_bytes")]


class GemmOpts(ctypes.Structure):
    """mirror of mx_gemm_opts"""
    _fields_ = [("path", ctypes.c_int32), ("split", ctypes.c_int32),
                ("debug_partials", ctypes.c_void_p), ("status", ctypes.c_void_p),
                ("wait_timeout_us", ctypes.c_int32), ("test_stall", ctypes.c_int32),
                ("act_group", ctypes.c_int32)]


_lib = None


def lib() -> ctypes.CDLL:
    """Load libmx.so (built in-tree); raise if it is missing."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with "
                          "`python -m mixed_precision_quantized_mx_b200.build`")
    L = ctypes.CDLL(LIB_PATH)
    P, I, I64, Z = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_size_t
    L.mx_version.restype = I
    L.mx_last_error.restype = ctypes.c_char_p
    L.mx_layout_init.argtypes = [I, I, I, I, ctypes.POINTER(Layout)]
    L.mx_layout_from_header.argtypes = [P, Z, ctypes.POINTER(Layout)]
    L.mx_pack_weights.argtypes = [ctypes.POINTER(Layout), P, I, I64, P, P, P, P]
    L.mx_quant_act.argtypes = [P, I, I, I, I64, P, P, P]
    L.mx_quant_act_grouped.argtypes = [P, I, I, I, I64, I, P, P, P]
    L.mx_gemm_workspace_size.argtypes = [ctypes.POINTER(Layout), I, ctypes.POINTER(GemmOpts),
                                         ctypes.POINTER(Z)]
    L.mx_gemm_select_path.argtypes = [ctypes.POINTER(Layout), I, ctypes.POINTER(GemmOpts)]
    L.mx_gemm_select_path.restype = I
    L.mx_gemm.argtypes = [ctypes.POINTER(Layout), P, P, P, I, P, I64, P, Z,
                          ctypes.POINTER(GemmOpts), P]
    L.mx_linear_workspace_size.argtypes = [ctypes.POINTER(Layout), I, I, ctypes.POINTER(GemmOpts),
                                           ctypes.POINTER(Z)]
    L.mx_linear.argtypes = [ctypes.POINTER(Layout), P, P, I, I, I64, P, I64, P, Z,
                            ctypes.POINTER(GemmOpts), P]
    L.mx_linear_noalloc.argtypes = [ctypes.POINTER(Layout), P, P, I, I, I64, P, I64,
                                    ctypes.POINTER(GemmOpts), P]
    L.mx_copy_mapped.argtypes = [P, P, Z, P]
    L.mx_saliency.argtypes = [P, I, I64, P, I, I64, I, I, I, P, P]
    L.mx_select_top_workspace_size.argtypes = [I64, ctypes.POINTER(Z)]
    L.mx_select_top.argtypes = [P, I64, I64, P, P, Z, P]
    L.mx_bw_layout_init.argtypes = [I, I, P, P, ctypes.POINTER(BwLayout)]
    L.mx_bw_pack.argtypes = [ctypes.POINTER(BwLayout), P, P, I, I64, P, P]
    L.mx_bw_gemm.argtypes = [ctypes.POINTER(BwLayout), P, P, P, I, P, I64, P, P]
    for n in ("mx_layout_init", "mx_layout_from_header", "mx_pack_weights", "mx_quant_act",
              "mx_quant_act_grouped", "mx_gemm_workspace_size", "mx_gemm", "mx_linear_workspace_size", "mx_linear",
              "mx_linear_noalloc", "mx_copy_mapped", "mx_saliency", "mx_select_top_workspace_size",
              "mx_select_top", "mx_bw_layout_init", "mx_bw_pack", "mx_bw_gemm"):
        getattr(L, n).restype = I
    _lib = L
    return L


def _check(st: int, fn: str):
    if st != MX_OK:
        raise MXError(st, fn, lib().mx_last_error().decode())


def _ptr(t: torch.Tensor | None) -> int | None:
    if t is None:
        return None
    return t.data_ptr()


def _stream(stream) -> int | None:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.float16:
        return MX_F16
    if t.dtype == torch.float32:
        return MX_F32
    raise TypeError(f"unsupported dtype {t.dtype}")


def _opts(path=0, split=0, debug_partials=None, status=None, wait_timeout_us=0,
          test_stall=0, act_group=0) -> GemmOpts:
    return GemmOpts(path, split, _ptr(debug_partials), _ptr(status), wait_timeout_us, test_stall, act_group)


# ------------------------------------------------------------------ entry points
def mx_version() -> int:
    return lib().mx_version()


def mx_layout_init(N: int, K: int, group: int, n8: int) -> Layout:
    L = Layout()
    _check(lib().mx_layout_init(N, K, group, n8, ctypes.byref(L)), "mx_layout_init")
    return L


def mx_layout_from_header(header) -> Layout:
    """header: bytes, or a host uint8 tensor holding the blob's first 256 bytes."""
    if isinstance(header, torch.Tensor):
        header = bytes(header[:HEADER_BYTES].cpu().numpy().tobytes())
    buf = ctypes.create_string_buffer(bytes(header), len(header))
    L = Layout()
    _check(lib().mx_layout_from_header(buf, len(header), ctypes.byref(L)), "mx_layout_from_header")
    return L


def mx_pack_weights(L: Layout, W: torch.Tensor, is8: torch.Tensor, blob: torch.Tensor,
                    status: torch.Tensor | None = None, stream=None) -> None:
    assert W.dim() == 2 and W.stride(1) == 1
    _check(lib().mx_pack_weights(ctypes.byref(L), _ptr(W), _dtype_code(W), W.stride(0), _ptr(is8),
                                 _ptr(blob), _ptr(status), _stream(stream)), "mx_pack_weights")


def mx_quant_act(X: torch.Tensor, Aq: torch.Tensor, s_a: torch.Tensor, stream=None) -> None:
    assert X.dim() == 2 and X.stride(1) == 1
    M, K = X.shape
    _check(lib().mx_quant_act(_ptr(X), _dtype_code(X), M, K, X.stride(0), _ptr(Aq), _ptr(s_a),
                              _stream(stream)), "mx_quant_act")


def mx_quant_act_grouped(X: torch.Tensor, Aq: torch.Tensor, s_a: torch.Tensor, act_group: int,
                         stream=None) -> None:
    """s_a: fp16 [M] (act_group 0) or [M, K / act_group]."""
    assert X.dim() == 2 and X.stride(1) == 1
    M, K = X.shape
    _check(lib().mx_quant_act_grouped(_ptr(X), _dtype_code(X), M, K, X.stride(0), act_group, _ptr(Aq),
                                      _ptr(s_a), _stream(stream)), "mx_quant_act_grouped")


def mx_gemm_workspace_size(L: Layout, M: int, path: int = 0, split: int = 0) -> int:
    n = ctypes.c_size_t(0)
    o = _opts(path, split)
    _check(lib().mx_gemm_workspace_size(ctypes.byref(L), M, ctypes.byref(o), ctypes.byref(n)),
           "mx_gemm_workspace_size")
    return n.value


def mx_gemm_select_path(L: Layout, M: int, path: int = 0, split: int = 0) -> int:
    o = _opts(path, split)
    r = lib().mx_gemm_select_path(ctypes.byref(L), M, ctypes.byref(o))
    if r < 0:
        _check(-r, "mx_gemm_select_path")
    return r


def mx_gemm(L: Layout, blob: torch.Tensor, Aq: torch.Tensor, s_a: torch.Tensor, Y: torch.Tensor,
            workspace: torch.Tensor | None = None, path: int = 0, split: int = 0,
            debug_partials: torch.Tensor | None = None, status: torch.Tensor | None = None,
            wait_timeout_us: int = 0, test_stall: int = 0, act_group: int = 0, stream=None) -> None:
    M = Aq.shape[0]
    o = _opts(path, split, debug_partials, status, wait_timeout_us, test_stall, act_group)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib().mx_gemm(ctypes.byref(L), _ptr(blob), _ptr(Aq), _ptr(s_a), M, _ptr(Y), Y.stride(0),
                         _ptr(workspace), ws_bytes, ctypes.byref(o), _stream(stream)), "mx_gemm")


def mx_linear_workspace_size(L: Layout, M: int, xdtype=torch.float16, path: int = 0, split: int = 0,
                             act_group: int = 0) -> int:
    n = ctypes.c_size_t(0)
    o = _opts(path, split, act_group=act_group)
    code = MX_F16 if xdtype == torch.float16 else MX_F32
    _check(lib().mx_linear_workspace_size(ctypes.byref(L), M, code, ctypes.byref(o), ctypes.byref(n)),
           "mx_linear_workspace_size")
    return n.value


def mx_linear(L: Layout, blob: torch.Tensor, X: torch.Tensor, Y: torch.Tensor,
              workspace: torch.Tensor | None = None, path: int = 0, split: int = 0,
              debug_partials: torch.Tensor | None = None, status: torch.Tensor | None = None,
              act_group: int = 0, stream=None) -> None:
    assert X.dim() == 2 and X.stride(1) == 1
    M = X.shape[0]
    o = _opts(path, split, debug_partials, status, act_group=act_group)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib().mx_linear(ctypes.byref(L), _ptr(blob), _ptr(X), _dtype_code(X), M, X.stride(0),
                           _ptr(Y), Y.stride(0), _ptr(workspace), ws_bytes, ctypes.byref(o),
                           _stream(stream)), "mx_linear")


NOALLOC_SCRATCH_BYTES = 4 << 20      # MX_NOALLOC_SCRATCH_BYTES


def mx_linear_noalloc(L: Layout, blob: torch.Tensor, X: torch.Tensor, Y: torch.Tensor, path: int = 0,
                      split: int = 0, debug_partials: torch.Tensor | None = None,
                      status: torch.Tensor | None = None, act_group: int = 0, stream=None) -> None:
    assert X.dim() == 2 and X.stride(1) == 1
    o = _opts(path, split, debug_partials, status, act_group=act_group)
    _check(lib().mx_linear_noalloc(ctypes.byref(L), _ptr(blob), _ptr(X), _dtype_code(X), X.shape[0],
                                   X.stride(0), _ptr(Y), Y.stride(0), ctypes.byref(o), _stream(stream)),
           "mx_linear_noalloc")


def mx_copy_mapped(dst: torch.Tensor, src: torch.Tensor, stream=None) -> None:
    """Copy src into dst with a kernel; either may be pinned host memory (see mx.h)."""
    if dst.nbytes != src.nbytes:
        raise ValueError(f"mx_copy_mapped: {dst.nbytes} bytes into {src.nbytes}")
    if not (dst.is_contiguous() and src.is_contiguous()):
        raise ValueError("mx_copy_mapped: contiguous tensors only")
    for t, n in ((dst, "dst"), (src, "src")):
        if not t.is_cuda and not t.is_pinned():
            raise ValueError(f"mx_copy_mapped: {n} is pageable host memory (pin it first)")
    _check(lib().mx_copy_mapped(_ptr(dst), _ptr(src), dst.nbytes, _stream(stream)), "mx_copy_mapped")


def mx_saliency(W: torch.Tensor, G: torch.Tensor, group: int, S: torch.Tensor | None = None,
                stream=None) -> torch.Tensor:
    """Per-row channel saliency of one layer (see mx.h); returns S (device fp32 [N])."""
    assert W.dim() == 2 and W.stride(1) == 1 and G.shape == W.shape and G.stride(1) == 1
    N, K = W.shape
    if S is None:
        S = torch.empty(N, dtype=torch.float32, device=W.device)
    _check(lib().mx_saliency(_ptr(W), _dtype_code(W), W.stride(0), _ptr(G), _dtype_code(G), G.stride(0), N, K,
                             group, _ptr(S), _stream(stream)), "mx_saliency")
    return S


def mx_select_top(S: torch.Tensor, n_top: int, is8: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """The n_top largest of the concatenated scores, ties to the lower index (see mx.h);
    returns the uint8 mask."""
    assert S.dim() == 1 and S.dtype == torch.float32 and S.is_contiguous()
    n = S.numel()
    if is8 is None:
        is8 = torch.empty(n, dtype=torch.uint8, device=S.device)
    nb = ctypes.c_size_t(0)
    _check(lib().mx_select_top_workspace_size(n, ctypes.byref(nb)), "mx_select_top_workspace_size")
    ws = torch.empty(max(nb.value, 16), dtype=torch.uint8, device=S.device)
    _check(lib().mx_select_top(_ptr(S), n, n_top, _ptr(is8), _ptr(ws), ws.numel(), _stream(stream)),
           "mx_select_top")
    return is8


# ------------------------------------------------------------------ block-wise bit widths
def _host_bytes(a) -> ctypes.Array:
    b = bytes(np.ascontiguousarray(np.asarray(a, dtype=np.uint8)).tobytes())
    return (ctypes.c_uint8 * max(1, len(b))).from_buffer_copy(b if b else b"\0")


def mx_bw_layout_init(N: int, K: int, table, meta) -> BwLayout:
    """Geometry of a block-wise layer (see mx_blockwise.h); table: four widths, meta: the
    packed 2-bit block codes (host bytes)."""
    L = BwLayout()
    _check(lib().mx_bw_layout_init(N, K, _host_bytes(table), _host_bytes(meta), ctypes.byref(L)),
           "mx_bw_layout_init")
    return L


def mx_bw_pack(L: BwLayout, meta, W: torch.Tensor, blob: torch.Tensor, stream=None) -> None:
    assert W.dim() == 2 and W.stride(1) == 1 and tuple(W.shape) == (L.N, L.K)
    assert blob.numel() * blob.element_size() >= L.total_bytes
    _check(lib().mx_bw_pack(ctypes.byref(L), _host_bytes(meta), _ptr(W), _dtype_code(W), W.stride(0), _ptr(blob),
                            _stream(stream)), "mx_bw_pack")


def mx_bw_gemm(L: BwLayout, blob: torch.Tensor, Aq: torch.Tensor, s_a: torch.Tensor, Y: torch.Tensor,
               partials: torch.Tensor | None = None, stream=None) -> None:
    assert Aq.dim() == 2 and Aq.is_contiguous() and Aq.dtype == torch.int8 and Aq.shape[1] == L.K
    assert s_a.dtype == torch.float16 and Y.dtype == torch.float16 and Y.stride(1) == 1
    M = Aq.shape[0]
    assert blob.numel() * blob.element_size() >= L.total_bytes and s_a.numel() >= M
    assert Y.shape[0] >= M and Y.shape[1] >= L.N
    assert partials is None or (partials.dtype == torch.int32 and partials.is_contiguous()
                                and partials.numel() >= M * L.N * L.KB)
    _check(lib().mx_bw_gemm(ctypes.byref(L), _ptr(blob), _ptr(Aq), _ptr(s_a), Aq.shape[0], _ptr(Y), Y.stride(0),
                            _ptr(partials), _stream(stream)), "mx_bw_gemm")
