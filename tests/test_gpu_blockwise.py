"""Parity of the block-wise bit-width path (ScaleBITS blog page: section 1.2.2, one
width per 64 x 128 block; section 3.2, a block layout with 2-bit metadata; section
4.2, widths from {1, 2, 3, 4, 6, 8}) on MixLLM's two-step int8 dequantization
(section 3.3) with the oracle.

Packing is bit-exact: every block's codes (read back from the blob's bit strings by
an unpack written from the layout in mx_blockwise.h, not from the kernels), zero
points and scales against oracle.pack_blockwise; 8-bit blocks are compared as q - z
since the blob stores them in offset binary (code q + 128, zero 128).  The GEMM's
per-block int32 partials are bit-exact against the oracle's; Y is within the
tolerance of the other paths (gpu_helpers).
"""
import numpy as np
import pytest
import torch

from mixed_precision_quantized_mx_b200 import binding as mx
from mixed_precision_quantized_mx_b200 import inputs

from gpu_helpers import assert_y_close, dev, gpu_quant, to_dev

pytestmark = pytest.mark.gpu

MAGIC = 0x5742584D          # "MXBW"


def unpack_blocks(blob: np.ndarray, L, codes, table, blocks=None):
    """(q - z) int16 [N, K], zeros [N, KB], scale bits [N, KB] read from a packed blob.
    blocks: the (row block, column block) pairs to decode (default: all); the entries
    of other blocks stay zero."""
    h = blob[:24].view(np.uint32)
    assert h[0] == MAGIC and h[1] == 1 and h[2] == L.N and h[3] == L.K
    NB, KB = codes.shape
    offs = blob[L.off_offsets:L.off_offsets + 4 * (NB * KB + 1)].view(np.uint32)
    scales = blob[L.off_scales:L.off_scales + 2 * L.N * KB].view(np.uint16).reshape(L.N, KB)
    zeros = blob[L.off_zeros:L.off_zeros + L.N * KB].reshape(L.N, KB)
    assert int(offs[-1]) * 16 == L.code_bytes
    qz = np.zeros((L.N, L.K), np.int16)
    if blocks is None:
        blocks = [(rb, kb) for rb in range(NB) for kb in range(KB)]
    for rb, kb in blocks:
        b = int(table[codes[rb, kb]])
        rows = min(64, L.N - rb * 64)
        base = L.off_codes + 16 * int(offs[rb * KB + kb])
        # the block's rows, each 16 b bytes: code k in bits k b .. k b + b - 1
        raw = blob[base: base + rows * 16 * b].reshape(rows, 16 * b)
        bits = np.unpackbits(raw, axis=1, bitorder="little").reshape(rows, 128, b)
        u = (bits.astype(np.int32) << np.arange(b)).sum(2)
        n = slice(rb * 64, rb * 64 + rows)
        qz[n, kb * 128:(kb + 1) * 128] = u - zeros[n, kb].astype(np.int32)[:, None]
    # offsets are consecutive: each block takes its rows x 16 b bytes
    sizes = np.diff(offs.astype(np.int64)) * 16
    want = np.array([min(64, L.N - rb * 64) * 16 * int(table[codes[rb, kb]])
                     for rb in range(NB) for kb in range(KB)], np.int64)
    assert np.array_equal(sizes, want)
    return qz, zeros, scales


def gpu_bw_pack(orc, W, codes, table):
    meta = orc.pack_block_codes(codes)
    N, K = W.shape
    L = mx.mx_bw_layout_init(N, K, table, meta)
    blob = torch.empty(L.total_bytes, dtype=torch.uint8, device=dev())
    mx.mx_bw_pack(L, meta, to_dev(W), blob)
    torch.cuda.synchronize()
    return L, blob


def check_pack(orc, W, codes, table, blocks=None):
    L, blob = gpu_bw_pack(orc, W, codes, table)
    b = orc.pack_blockwise(W.astype(np.float32), codes, table)
    qz, zeros, scales = unpack_blocks(blob.cpu().numpy(), L, codes, np.asarray(table), blocks)
    want = b.q.astype(np.int16) - np.repeat(b.zeros.astype(np.int16), 128, 1)
    w8 = np.repeat(np.asarray(table)[codes], 64, 0)[:W.shape[0]] == 8
    if blocks is None:
        assert np.array_equal(qz, want)
        assert np.array_equal(scales, b.scales)
        assert np.array_equal(zeros[w8], np.full(int(w8.sum()), 128, np.uint8))
        assert np.array_equal(zeros[~w8], b.zeros[~w8])
    else:
        for rb, kb in blocks:
            n, k = slice(rb * 64, rb * 64 + 64), slice(kb * 128, kb * 128 + 128)
            assert np.array_equal(qz[n, k], want[n, k]), (rb, kb)
        assert np.array_equal(scales, b.scales)
        assert np.array_equal(zeros[~w8], b.zeros[~w8])
    return L, blob, b


@pytest.mark.parametrize("table", [[2, 3, 4, 8], [1, 5, 6, 7], [1, 2, 6, 8], [4, 4, 4, 4], [8, 8, 8, 8]])
@pytest.mark.parametrize("N,K", [(64, 128), (200, 512), (130, 1152)])
def test_pack_matches_oracle(orc, table, N, K):
    rng = np.random.default_rng(N + K + sum(table))
    W = inputs.weights(rng, N, K, outlier_frac=0.001)
    check_pack(orc, W, inputs.block_codes(rng, N, K), table)


def test_pack_fp16_weights(orc):
    rng = np.random.default_rng(3)
    W = inputs.weights(rng, 96, 384).astype(np.float16)
    check_pack(orc, W, inputs.block_codes(rng, 96, 384), [2, 4, 6, 8])


def test_pack_degenerate_groups(orc):
    # all-zero rows, constant rows, one outlier: scale 1 / zero 0 and saturation as the oracle
    rng = np.random.default_rng(4)
    W = inputs.weights(rng, 128, 256)
    W[3] = 0.0
    W[70] = 0.25
    W[100, 5] = 40.0
    check_pack(orc, W, inputs.block_codes(rng, 128, 256), [1, 3, 4, 8])


def run_gemm(orc, M, N, K, table, seed):
    rng = np.random.default_rng(seed)
    W = inputs.weights(rng, N, K, outlier_frac=0.001)
    codes = inputs.block_codes(rng, N, K)
    L, blob, b = check_pack(orc, W, codes, table)
    X = inputs.activations(rng, M, K, 3)
    Aq, sa = gpu_quant(X)
    Y = torch.full((M, N + 8), float("nan"), dtype=torch.float16, device=dev())
    P = torch.zeros((M, N, L.KB), dtype=torch.int32, device=dev())
    mx.mx_bw_gemm(L, blob, Aq, sa, Y, partials=P)
    torch.cuda.synchronize()
    Aq_o, sa_o = orc.quant_act(X.astype(np.float32))
    yd, yt, P_o, pmax = orc.gemm_blockwise(Aq_o, sa_o, b)
    assert np.array_equal(P.cpu().numpy().astype(np.int64), P_o)
    assert_y_close(Y[:, :N].cpu().numpy(), yt)
    assert torch.isnan(Y[:, N:]).all()                       # nothing past ldy's N columns
    Y2 = torch.empty((M, N), dtype=torch.float16, device=dev())
    mx.mx_bw_gemm(L, blob, Aq, sa, Y2)                        # without partials: the same Y
    torch.cuda.synchronize()
    assert torch.equal(Y2.view(torch.int16), Y[:, :N].contiguous().view(torch.int16))


@pytest.mark.parametrize("M", [1, 3, 4, 8, 9, 16, 17, 33])
@pytest.mark.parametrize("table", [[2, 3, 4, 8], [1, 5, 6, 7], [1, 2, 6, 8]])
def test_gemm_matches_oracle(orc, M, table):
    run_gemm(orc, M, 200, 640, table, M * 11 + table[0] + table[1])


def test_gemm_all_8bit_blocks(orc):
    run_gemm(orc, 5, 136, 384, [8, 8, 8, 8], 9)


def test_gemm_uniform_4bit_matches_mixllm_layer(orc):
    # all blocks 4-bit: the MixLLM layer with no 8-bit rows, through the MixLLM path
    from gpu_helpers import gpu_gemm, gpu_pack
    rng = np.random.default_rng(5)
    M, N, K = 4, 256, 1024
    W = inputs.weights(rng, N, K)
    L, blob, _ = check_pack(orc, W, np.zeros((N // 64, K // 128), np.uint8), [4, 4, 4, 4])
    X = inputs.activations(rng, M, K, 2)
    Aq, sa = gpu_quant(X)
    P = torch.zeros((M, N, K // 128), dtype=torch.int32, device=dev())
    Y = torch.empty((M, N), dtype=torch.float16, device=dev())
    mx.mx_bw_gemm(L, blob, Aq, sa, Y, partials=P)
    Lm, blobm = gpu_pack(W, np.zeros(N, np.uint8), 128)
    _, Pm, _ = gpu_gemm(Lm, blobm, Aq, sa, debug=True)
    torch.cuda.synchronize()
    assert torch.equal(P, Pm)


def test_llama3_8b_up_sampled(orc):
    """Full Llama-3-8B up shape (K 4096, N 14336) with the benchmark's width mix: the
    pack bit-exact on 64 sampled blocks (scales and zeros everywhere), the partials
    bit-exact and Y within tolerance on 1024 sampled (token, row) outputs and on a
    whole row of Y."""
    K, N = inputs.SHAPES["llama3-8b-up"]
    M = 4
    table = [2, 3, 4, 8]
    rng = np.random.default_rng(21)
    W = inputs.weights(rng, N, K, outlier_frac=0.001)
    codes = inputs.block_codes(rng, N, K, (0.25, 0.25, 0.40, 0.10))
    NB, KB = codes.shape
    blocks = list({(int(r), int(c)) for r, c in zip(rng.integers(0, NB, 64), rng.integers(0, KB, 64))})
    blocks.append((NB - 1, KB - 1))
    L, blob, b = check_pack(orc, W, codes, table, blocks)
    X = inputs.activations(rng, M, K, 41)
    Aq, sa = gpu_quant(X)
    Y = torch.empty((M, N), dtype=torch.float16, device=dev())
    P = torch.zeros((M, N, KB), dtype=torch.int32, device=dev())
    mx.mx_bw_gemm(L, blob, Aq, sa, Y, partials=P)
    torch.cuda.synchronize()
    Aq_o, sa_o = orc.quant_act(X.astype(np.float32))
    m = np.concatenate([rng.integers(0, M, 1024), np.full(N, 2)]).astype(np.int32)
    n = np.concatenate([rng.integers(0, N, 1024), np.arange(N)]).astype(np.int32)
    _, yt, P_o, _ = orc.gemm_blockwise(Aq_o, sa_o, b, pairs=(m, n))
    Pg = P.cpu().numpy()[m, n].astype(np.int64)
    assert np.array_equal(Pg, P_o)
    Yg = Y.cpu().numpy()
    assert_y_close(Yg[2][None, :], yt[1024:][None, :])
    rms = np.sqrt(np.mean(yt[1024:] ** 2))
    assert_y_close(Yg[m[:1024], n[:1024]], yt[:1024], rows_rms=np.full(1024, rms))
