"""MixedPrecisionLinear: the user-facing object around the C ABI.

It owns the packed weight blob (torch device memory), sizes the workspace, and
runs one forward pass with mx_linear (quantize activations, mixed-precision
GEMM) on the current CUDA stream.  All arithmetic happens in libmx.so's kernels.
"""
from __future__ import annotations

import torch

from . import binding as mx


class MixedPrecisionLinear:
    """Y = X W^T with W split into 8-bit symmetric / 4-bit asymmetric rows (MixLLM)."""

    def __init__(self, W: torch.Tensor, is8: torch.Tensor, group: int = 128, n8: int | None = None):
        if not W.is_cuda:
            raise ValueError("W must be a CUDA tensor")
        N, K = W.shape
        if n8 is None:
            n8 = int(is8.count_nonzero().item())
        self.layout = mx.mx_layout_init(N, K, group, n8)
        self.blob = torch.empty(self.layout.total_bytes, dtype=torch.uint8, device=W.device)
        self._status = torch.zeros(1, dtype=torch.int32, device=W.device)
        mx.mx_pack_weights(self.layout, W, is8.to(W.device, torch.uint8), self.blob, status=self._status)
        self._ws = {}

    @classmethod
    def from_blob(cls, blob: torch.Tensor) -> "MixedPrecisionLinear":
        """Re-open a packed blob (for example one saved with torch.save)."""
        self = cls.__new__(cls)
        self.layout = mx.mx_layout_from_header(blob[:mx.HEADER_BYTES].cpu())
        if blob.numel() < self.layout.total_bytes:
            raise ValueError("blob shorter than its header says")
        self.blob = blob
        self._status = torch.zeros(1, dtype=torch.int32, device=blob.device)
        self._ws = {}
        return self

    @property
    def N(self) -> int:
        return self.layout.N

    @property
    def K(self) -> int:
        return self.layout.K

    def check_pack_status(self) -> None:
        """Raise if the packer reported an error (mask count mismatch)."""
        st = int(self._status.item())
        if st != 0:
            raise mx.MXError(st, "mx_pack_weights", "device-side error while packing")

    def workspace(self, M: int, xdtype=torch.float16, path: int = 0, act_group: int = 0) -> torch.Tensor | None:
        """Device scratch for mx_linear at M tokens (None when it needs none); cached."""
        key = (M, xdtype, path, act_group)
        if key not in self._ws:
            n = mx.mx_linear_workspace_size(self.layout, M, xdtype, path=path, act_group=act_group)
            self._ws[key] = torch.empty(n, dtype=torch.uint8, device=self.blob.device) if n else None
        return self._ws[key]

    def forward(self, X: torch.Tensor, out: torch.Tensor | None = None, path: int = 0,
                act_group: int = 0) -> torch.Tensor:
        """act_group: 0 -- one activation scale per token; the weight group -- group-wise."""
        M, K = X.shape
        if K != self.K:
            raise ValueError(f"X has K={K}, layer expects {self.K}")
        Y = out if out is not None else torch.empty((M, self.N), dtype=torch.float16, device=self.blob.device)
        mx.mx_linear(self.layout, self.blob, X, Y, workspace=self.workspace(M, X.dtype, path, act_group),
                     path=path, act_group=act_group)
        return Y

    __call__ = forward

    def graphed(self, x_host: torch.Tensor, y_host: torch.Tensor | None = None, path: int = 0,
                act_group: int = 0) -> "GraphedLinear":
        """Capture host-in / host-out calls for this input buffer (see GraphedLinear)."""
        return GraphedLinear(self, x_host, y_host, path, act_group)


class GraphedLinear:
    """A MixedPrecisionLinear call captured once as a CUDA graph for a fixed M.

    The graph copies the pinned host input into the device, runs mx_linear
    (quantize + GEMM, one kernel for decode-sized M) and copies Y back into the
    pinned host output, so one `replay()` per
    step is the whole host-to-host pass with a single launch from the host.
    The copies are kernels that read and write the mapped host buffers
    (mx_copy_mapped), so the graph holds kernels only and mx_linear's weight
    stream starts while the input crosses the bus.
    The caller rewrites `x_host` between replays and reads `y_host` after the
    stream is synchronised (or after an event recorded after `replay()`).
    """

    def __init__(self, layer: MixedPrecisionLinear, x_host: torch.Tensor, y_host: torch.Tensor | None = None,
                 path: int = 0, act_group: int = 0):
        if not x_host.is_pinned():
            raise ValueError("x_host must be pinned host memory")
        if y_host is not None and not y_host.is_pinned():
            raise ValueError("y_host must be pinned host memory")
        M, K = x_host.shape
        dev = layer.blob.device
        self.layer = layer
        self.x_host = x_host
        self.y_host = y_host if y_host is not None else torch.empty((M, layer.N), dtype=torch.float16).pin_memory()
        self.x_dev = torch.empty((M, K), dtype=x_host.dtype, device=dev)
        self.y_dev = torch.empty((M, layer.N), dtype=torch.float16, device=dev)
        ws = layer.workspace(M, x_host.dtype, path, act_group)
        self.stream = torch.cuda.Stream(dev)

        def body():
            mx.mx_copy_mapped(self.x_dev, self.x_host)
            mx.mx_linear(layer.layout, layer.blob, self.x_dev, self.y_dev, workspace=ws, path=path,
                         act_group=act_group)
            mx.mx_copy_mapped(self.y_host, self.y_dev)

        with torch.cuda.stream(self.stream):        # configure kernels outside capture
            body()
        self.stream.synchronize()
        self.graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(self.graph, stream=self.stream):
            body()

    def replay(self) -> None:
        """Launch the captured pass on `self.stream` (a graph replays on the current stream)."""
        with torch.cuda.stream(self.stream):
            self.graph.replay()
