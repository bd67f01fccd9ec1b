"""Algorithmic work model of one mixed-precision linear call (bytes and integer ops).

Used by the benchmark to turn measured times into GB/s, TOPS and roofline
fractions.  The counts are the minimum traffic of the method, not of any kernel:

* ops   = 2 M N K (every int8 multiply-accumulate counted twice; the widening
          and the per-group rescale are not counted)
* bytes = weights + activations + output, with
    weights     = N8 K + N4 K/2        codes (8-bit rows, 4-bit rows)
                + 2 N G                fp16 group scales
                + N4 G / 2             uint4 zero points
                + 4 N                  int32 row permutation
    activations = M K + 2 M            int8 codes + fp16 per-token scales
    output      = 2 M N                fp16 Y
* quantize-activation bytes = (2 or 4) M K in + M K + 2 M out
* linear bytes (the layer as a whole, quantized activations being an
  intermediate) = weights + (2 or 4) M K of X + 2 M N of Y

The compute-intensity form I = 2MNK / (M K B_act + K N B_weight) is the one the
MixLLM paper uses to argue for 8-bit activations and 4-bit weights (section 3.1.2).
"""
from __future__ import annotations


def intensity(M: int, N: int, K: int, b_act: float, b_weight: float) -> float:
    """ops per byte with b_act / b_weight BYTES per element (section 3.1.2)."""
    return 2.0 * M * N * K / (M * K * b_act + K * N * b_weight)


def gemm_ops(M: int, N: int, K: int) -> float:
    return 2.0 * M * N * K


def weight_bytes(N: int, K: int, group: int, n8: int) -> float:
    G = K // group
    n4 = N - n8
    return n8 * K + n4 * K / 2 + 2.0 * N * G + n4 * G / 2 + 4.0 * N


def gemm_bytes(M: int, N: int, K: int, group: int, n8: int) -> float:
    return weight_bytes(N, K, group, n8) + (M * K + 2.0 * M) + 2.0 * M * N


def quant_act_bytes(M: int, K: int, in_bytes: int = 2) -> float:
    return float(in_bytes) * M * K + M * K + 2.0 * M


def step_bytes(M: int, N: int, K: int, group: int, n8: int, in_bytes: int = 2) -> float:
    """quantize activations + GEMM: X in, Aq/s_a round trip through HBM, Y out."""
    return quant_act_bytes(M, K, in_bytes) + gemm_bytes(M, N, K, group, n8)


def linear_bytes(M: int, N: int, K: int, group: int, n8: int, in_bytes: int = 2) -> float:
    """The layer end to end: X in, packed weights, Y out."""
    return weight_bytes(N, K, group, n8) + float(in_bytes) * M * K + 2.0 * M * N


def bw_weight_bytes(N: int, K: int, code_bytes: int) -> float:
    """Block-wise bit widths: the blocks' codes (code_bytes, b / 8 bytes per weight), an fp16
    scale and a uint8 zero per (row, 128-column block), the 2-bit block codes and the
    uint32 block offsets."""
    KB = K // 128
    NB = (N + 63) // 64
    return code_bytes + 3 * N * KB + (NB * KB + 3) // 4 + 4 * (NB * KB + 1)


def bw_gemm_bytes(M: int, N: int, K: int, code_bytes: int) -> float:
    """One block-wise GEMM call: weights, int8 activations with fp16 token scales, fp16 Y."""
    return bw_weight_bytes(N, K, code_bytes) + M * K + 2 * M + 2 * M * N
