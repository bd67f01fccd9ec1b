"""B200-native MixLLM mixed-precision quantized linear layer (W4.4A8).

Public API: the C ABI in include/mx.h (libmx.so) and its Python mirror in
``binding`` (same function names), plus ``MixedPrecisionLinear``.  The library
is loaded on first use; nothing here computes on the host.
"""
from . import binding
from .binding import (MXError, mx_gemm, mx_gemm_select_path, mx_gemm_workspace_size,
                      mx_layout_from_header, mx_layout_init, mx_linear, mx_linear_workspace_size,
                      mx_pack_weights, mx_quant_act, mx_version)


def __getattr__(name):
    if name == "MixedPrecisionLinear":
        from .layer import MixedPrecisionLinear
        return MixedPrecisionLinear
    raise AttributeError(name)
