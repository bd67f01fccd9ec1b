"""CPU oracle for the MixLLM mixed-precision quantized linear layer.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this
package.  The product path (the C-ABI library and its Python binding) never
imports, links or runs it, and the two share no code.

The arithmetic lives in ``mx_oracle.c`` (plain C, single thread, exact int64 and
fp64 after the fp32 quantization decisions).  This module only compiles it with
gcc and marshals numpy arrays through ctypes.  Every function cites the passage
of the MixLLM paper digest it follows (see the C file for the full list).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "mx_oracle.c")
_LIB = os.path.join(_HERE, "libmx_oracle.so")
_CFLAGS = ["-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared"]

_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (IEEE fp32/fp64, no contraction); return the .so path."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.run(["gcc", *_CFLAGS, "-o", tmp, _SRC, "-lm"], check=True)
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is not None:
        return _lib
    lib = ctypes.CDLL(build())
    P = ctypes.c_void_p
    I = ctypes.c_int
    lib.mxo_fp16_round.argtypes = [ctypes.c_double]
    lib.mxo_fp16_round.restype = ctypes.c_double
    lib.mxo_fp16_bits_of.argtypes = [ctypes.c_double]
    lib.mxo_fp16_bits_of.restype = ctypes.c_uint16
    lib.mxo_fp16_value.argtypes = [ctypes.c_uint16]
    lib.mxo_fp16_value.restype = ctypes.c_double
    lib.mxo_quant_sym8.argtypes = [P, I, P, P]
    lib.mxo_quant_sym8.restype = None
    lib.mxo_quant_asym4.argtypes = [P, I, P, P, P]
    lib.mxo_quant_asym4.restype = None
    lib.mxo_quant_act.argtypes = [P, I, I, I, I, P, P]
    lib.mxo_quant_act.restype = I
    lib.mxo_pack.argtypes = [P, I, I, I, I, P, P, P, P, P, P, P]
    lib.mxo_pack.restype = I
    lib.mxo_partials.argtypes = [P, I, I, I, I, P, I, P, P, P, P]
    lib.mxo_partials.restype = ctypes.c_int64
    lib.mxo_gemm.argtypes = [P, P, I, I, I, I, I, P, I, P, P, P, P, P, P, P, ctypes.c_long, P, P]
    lib.mxo_gemm.restype = I
    lib.mxo_saliency.argtypes = [P, I, P, I, I, I, I, P]
    lib.mxo_saliency.restype = I
    lib.mxo_quant_asym.argtypes = [P, I, I, P, P, P]
    lib.mxo_quant_asym.restype = I
    lib.mxo_pack_blockwise.argtypes = [P, I, I, I, P, P, P, P, P]
    lib.mxo_pack_blockwise.restype = I
    lib.mxo_gemm_blockwise.argtypes = [P, P, I, I, I, P, P, P, P, P, ctypes.c_long, P, P, P]
    lib.mxo_gemm_blockwise.restype = ctypes.c_int64
    _lib = lib
    return lib


def _p(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _f32(a) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=np.float32)


# ----------------------------------------------------------------- fp16 helpers
def fp16_round(v: float) -> float:
    """Nearest IEEE binary16 value (ties to even), overflow to inf."""
    return _load().mxo_fp16_round(float(v))


def fp16_bits(v: float) -> int:
    """Bit pattern of an exactly representable binary16 value."""
    return int(_load().mxo_fp16_bits_of(float(v)))


def fp16_value(bits: int) -> float:
    return _load().mxo_fp16_value(int(bits) & 0xFFFF)


def fp16_values(bits: np.ndarray) -> np.ndarray:
    """Vector form of fp16_value (loop over the C routine; for small arrays)."""
    lib = _load()
    flat = np.asarray(bits, dtype=np.uint16).ravel()
    out = np.array([lib.mxo_fp16_value(int(b)) for b in flat], dtype=np.float64)
    return out.reshape(np.shape(bits))


# ----------------------------------------------------------------- quantizers
def quant_sym8(x) -> tuple[np.ndarray, int]:
    """Symmetric 8-bit quantizer of one group (MixLLM section 2.1; range +-127)."""
    x = _f32(x).ravel()
    q = np.zeros(x.size, np.int8)
    s = np.zeros(1, np.uint16)
    _load().mxo_quant_sym8(_p(x), x.size, _p(q), _p(s))
    return q, int(s[0])


def quant_asym4(x) -> tuple[np.ndarray, int, int]:
    """Asymmetric 4-bit quantizer of one group (MixLLM section 2.1 affine form)."""
    x = _f32(x).ravel()
    q = np.zeros(x.size, np.uint8)
    z = np.zeros(1, np.uint8)
    s = np.zeros(1, np.uint16)
    _load().mxo_quant_asym4(_p(x), x.size, _p(q), _p(z), _p(s))
    return q, int(z[0]), int(s[0])


def quant_act(X, act_group: int = 0) -> tuple[np.ndarray, np.ndarray]:
    """8-bit symmetric activation quantization (MixLLM section 3.1.2).

    act_group == 0: one fp16 scale per token, s_a shape [M].
    act_group == g: one scale per (token, group of g columns), shape [M, K/g].
    Returns (Aq int8 [M, K], s_a fp16 bits uint16).
    """
    X = _f32(X)
    M, K = X.shape
    na = 1 if act_group == 0 else K // act_group
    Aq = np.zeros((M, K), np.int8)
    sa = np.zeros((M, na), np.uint16)
    rc = _load().mxo_quant_act(_p(X), M, K, K, act_group, _p(Aq), _p(sa))
    if rc != 0:
        raise ValueError("mxo_quant_act: bad arguments")
    return Aq, (sa[:, 0].copy() if act_group == 0 else sa)


@dataclass
class Canonical:
    """Canonical packed form: the compare target for the GPU blob."""
    N: int
    K: int
    group: int
    n8: int
    perm: np.ndarray      # int32 [N]: packed row -> original row
    codes8: np.ndarray    # int8  [n8, K]
    scales8: np.ndarray   # uint16 fp16 bits [n8, G]
    codes4: np.ndarray    # uint8 [N-n8, K], one code per byte
    zeros4: np.ndarray    # uint8 [N-n8, G]
    scales4: np.ndarray   # uint16 fp16 bits [N-n8, G]

    @property
    def G(self) -> int:
        return self.K // self.group


def pack(W, is8, group: int) -> Canonical:
    """Row split + permutation + per-group quantization (MixLLM sections 3.1.1, 2.1)."""
    W = _f32(W)
    N, K = W.shape
    is8 = np.ascontiguousarray(is8, dtype=np.uint8)
    assert is8.shape == (N,)
    G = K // group
    n8 = int((is8 != 0).sum())
    perm = np.zeros(N, np.int32)
    c8 = np.zeros((n8, K), np.int8)
    s8 = np.zeros((n8, G), np.uint16)
    c4 = np.zeros((N - n8, K), np.uint8)
    z4 = np.zeros((N - n8, G), np.uint8)
    s4 = np.zeros((N - n8, G), np.uint16)
    rc = _load().mxo_pack(_p(W), N, K, K, group, _p(is8), _p(perm), _p(c8), _p(s8),
                          _p(c4), _p(z4), _p(s4))
    if rc != n8:
        raise ValueError("mxo_pack: bad arguments")
    return Canonical(N, K, group, n8, perm, c8, s8, c4, z4, s4)


def partials(Aq: np.ndarray, c: Canonical) -> tuple[np.ndarray, int]:
    """int64 P[m, n, g] in original row order (MixLLM section 3.3 step one)."""
    Aq = np.ascontiguousarray(Aq, dtype=np.int8)
    M = Aq.shape[0]
    P = np.zeros((M, c.N, c.G), np.int64)
    pmax = _load().mxo_partials(_p(Aq), M, c.K, c.group, c.N, _p(c.perm), c.n8,
                                _p(c.codes8), _p(c.codes4), _p(c.zeros4), _p(P))
    if pmax < 0:
        raise ValueError("mxo_partials: bad arguments")
    return P, int(pmax)


def gemm(Aq: np.ndarray, s_a: np.ndarray, c: Canonical, act_group: int = 0,
         pairs: tuple[np.ndarray, np.ndarray] | None = None) -> tuple[np.ndarray, np.ndarray]:
    """fp64 Y two ways (plain definition, two-step form of MixLLM section 3.3).

    pairs=None: all outputs, shape [M, N].  pairs=(m_idx, n_idx): those entries only
    (n in original row order), shape [len(m_idx)].
    """
    Aq = np.ascontiguousarray(Aq, dtype=np.int8)
    s_a = np.ascontiguousarray(s_a, dtype=np.uint16)
    M = Aq.shape[0]
    if pairs is None:
        pm = pn = None
        cnt = M * c.N
        shape = (M, c.N)
    else:
        pm = np.ascontiguousarray(pairs[0], dtype=np.int32)
        pn = np.ascontiguousarray(pairs[1], dtype=np.int32)
        cnt = pm.size
        shape = (cnt,)
    yd = np.zeros(cnt, np.float64)
    yt = np.zeros(cnt, np.float64)
    rc = _load().mxo_gemm(_p(Aq), _p(s_a), act_group, M, c.K, c.group, c.N, _p(c.perm), c.n8,
                          _p(c.codes8), _p(c.scales8), _p(c.codes4), _p(c.zeros4), _p(c.scales4),
                          None if pm is None else _p(pm), None if pn is None else _p(pn),
                          cnt, _p(yd), _p(yt))
    if rc != 0:
        raise ValueError("mxo_gemm: bad arguments")
    return yd.reshape(shape), yt.reshape(shape)


def dequant_weights(c: Canonical) -> np.ndarray:
    """Dequantized W' [N, K] (fp64, original row order): (W_q - z) s_w (section 2.1)."""
    G, g = c.G, c.group
    W = np.zeros((c.N, c.K), np.float64)
    s8 = fp16_values(c.scales8) if c.n8 else np.zeros((0, G))
    s4 = fp16_values(c.scales4) if c.N - c.n8 else np.zeros((0, G))
    for j in range(c.N):
        n = int(c.perm[j])
        if j < c.n8:
            w = c.codes8[j].astype(np.float64)
            W[n] = w * np.repeat(s8[j], g)
        else:
            r = j - c.n8
            w = c.codes4[r].astype(np.float64) - np.repeat(c.zeros4[r].astype(np.float64), g)
            W[n] = w * np.repeat(s4[r], g)
    return W


def saliency(W, G, group: int) -> np.ndarray:
    """Channel saliency of the global precision search (MixLLM section 3.2, Eq. 4
    with one gradient batch, as Algorithm 1 scores a layer): per output row,
    S = |S1 + S1^2/2| with S1 = sum_k G * (dequant(quantize4(W)) - W), in fp64."""
    W = np.ascontiguousarray(_f32(W))
    G = np.ascontiguousarray(_f32(G))
    N, K = W.shape
    assert G.shape == (N, K)
    S = np.zeros(N, np.float64)
    if _load().mxo_saliency(_p(W), K, _p(G), K, N, K, group, _p(S)) != 0:
        raise ValueError("bad saliency arguments")
    return S


def select_top(scores, n_top: int) -> np.ndarray:
    """The global choice of Algorithm 1 over the scores of all layers concatenated: the
    n_top largest are the 8-bit channels (the paper leaves ties open: they go to the lower global
    index, i.e. the earlier layer, then the lower row).  Returns a uint8 mask."""
    scores = np.asarray(scores)
    order = np.lexsort((np.arange(scores.size), -scores.astype(np.float64)))
    mask = np.zeros(scores.size, np.uint8)
    mask[order[:max(0, min(n_top, scores.size))]] = 1
    return mask


# ----------------------------------------------------------------- block-wise bit widths
BLOCK_ROWS, BLOCK_COLS = 64, 128


def quant_asym(x, bits: int) -> tuple[np.ndarray, int, int]:
    """Asymmetric b-bit quantizer of one group, 1 <= b <= 7 (the 4-bit quantizer of
    MixLLM section 2.1 with 2^b - 1 levels; b = 4 is quant_asym4)."""
    x = _f32(x).ravel()
    q = np.zeros(x.size, np.uint8)
    z = np.zeros(1, np.uint8)
    s = np.zeros(1, np.uint16)
    if _load().mxo_quant_asym(_p(x), x.size, int(bits), _p(q), _p(z), _p(s)) != 0:
        raise ValueError("quant_asym: bad arguments")
    return q, int(z[0]), int(s[0])


def pack_block_codes(codes: np.ndarray) -> np.ndarray:
    """2-bit block codes [NB, KB] (values 0..3) packed four to a byte, block i (row-major)
    in bits 2 (i mod 4) of byte i / 4 (the ScaleBITS blog page's 2-bit metadata, section 3.2)."""
    flat = np.asarray(codes, dtype=np.uint8).ravel()
    assert flat.size == 0 or int(flat.max()) <= 3
    out = np.zeros((flat.size + 3) // 4, np.uint8)
    for i, c in enumerate(flat):
        out[i >> 2] |= np.uint8(int(c) << (2 * (i & 3)))
    return out


@dataclass
class Blockwise:
    """A layer with one bit width per 64 x 128 block, in original row order."""
    N: int
    K: int
    table: np.ndarray     # [4] uint8: the widths the 2-bit codes select
    codes: np.ndarray     # [NB, KB] uint8: each block's 2-bit code
    meta: np.ndarray      # packed codes (pack_block_codes)
    q: np.ndarray         # [N, K] int16: -127..127 in 8-bit blocks, else 0..2^b - 1
    zeros: np.ndarray     # [N, KB] uint8 (0 in 8-bit blocks)
    scales: np.ndarray    # [N, KB] uint16 fp16 bits

    @property
    def KB(self) -> int:
        return self.K // BLOCK_COLS

    def widths(self) -> np.ndarray:
        """[NB, KB] bit width of every block."""
        return self.table[self.codes]


def pack_blockwise(W, codes, table) -> Blockwise:
    """Quantize W block by block (ScaleBITS blog page, sections 1.2.2 and 3.2): each row's
    128 weights inside a block are one group, 8-bit blocks symmetric, narrower blocks
    asymmetric with 2^b levels."""
    W = _f32(W)
    N, K = W.shape
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    table = np.ascontiguousarray(table, dtype=np.uint8)
    assert table.shape == (4,)
    assert codes.shape == ((N + BLOCK_ROWS - 1) // BLOCK_ROWS, K // BLOCK_COLS)
    meta = pack_block_codes(codes)
    KB = K // BLOCK_COLS
    q = np.zeros((N, K), np.int16)
    zeros = np.zeros((N, KB), np.uint8)
    scales = np.zeros((N, KB), np.uint16)
    if _load().mxo_pack_blockwise(_p(W), N, K, K, _p(table), _p(meta), _p(q), _p(zeros), _p(scales)) != 0:
        raise ValueError("mxo_pack_blockwise: bad arguments")
    return Blockwise(N, K, table, codes, meta, q, zeros, scales)


def gemm_blockwise(Aq: np.ndarray, s_a: np.ndarray, b: Blockwise,
                   pairs: tuple[np.ndarray, np.ndarray] | None = None):
    """fp64 Y two ways (plain definition; two-step form of MixLLM section 3.3 over each
    block's groups) and the int64 partials P [.., KB].  Returns (Y_def, Y_two, P, max |P|)."""
    Aq = np.ascontiguousarray(Aq, dtype=np.int8)
    s_a = np.ascontiguousarray(s_a, dtype=np.uint16)
    M = Aq.shape[0]
    assert Aq.shape[1] == b.K and s_a.shape == (M,)
    if pairs is None:
        pm = pn = None
        cnt = M * b.N
        shape = (M, b.N)
    else:
        pm = np.ascontiguousarray(pairs[0], dtype=np.int32)
        pn = np.ascontiguousarray(pairs[1], dtype=np.int32)
        cnt = pm.size
        shape = (cnt,)
    yd = np.zeros(cnt, np.float64)
    yt = np.zeros(cnt, np.float64)
    P = np.zeros((cnt, b.KB), np.int64)
    pmax = _load().mxo_gemm_blockwise(_p(Aq), _p(s_a), M, b.K, b.N, _p(b.q), _p(b.zeros), _p(b.scales),
                                      None if pm is None else _p(pm), None if pn is None else _p(pn),
                                      cnt, _p(yd), _p(yt), _p(P))
    if pmax < 0:
        raise ValueError("mxo_gemm_blockwise: bad arguments")
    return yd.reshape(shape), yt.reshape(shape), P.reshape(shape + (b.KB,)), int(pmax)


def bits_per_weight(b: Blockwise) -> float:
    """Average stored bits per weight: each block's codes plus its 2-bit metadata (the
    per-row fp16 scales and zeros are counted separately by the layout)."""
    rows = np.minimum(BLOCK_ROWS, b.N - np.arange(b.codes.shape[0]) * BLOCK_ROWS)
    code_bits = float((b.widths().astype(np.int64) * rows[:, None] * BLOCK_COLS).sum())
    return (code_bits + 2.0 * b.codes.size) / (b.N * b.K)
