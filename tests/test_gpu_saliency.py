"""Parity of the global precision search on the GPU (MixLLM section 3.2, Eq. 4 and
Algorithm 1) with the oracle: per-row saliency of each layer, then the global
choice of the 8-bit rows over all layers.

Saliency: both sides take the same fp32 quantizer decisions (the packer's) and
sum G * dW in fp64, in different orders; the GPU rounds S to fp32 once.  So S
matches the oracle's fp64 value to fp32 rounding: |S_gpu - S| <= 2^-23 |S| plus
the fp64 summation error (K 2^-52 of the sum of |G dW|), far below that.
Selection is integer work on the GPU's own fp32 scores: bit-exact against the
oracle's selection of the same scores, ties included.
"""
import numpy as np
import pytest
import torch

from mixed_precision_quantized_mx_b200 import binding as mx
from mixed_precision_quantized_mx_b200 import inputs

from gpu_helpers import dev, to_dev
from test_gpu_parity import check_pack, run_and_check

pytestmark = pytest.mark.gpu


def gpu_saliency(W, G, group):
    S = mx.mx_saliency(to_dev(W), to_dev(G), group)
    torch.cuda.synchronize()
    return S.cpu().numpy()


def assert_saliency_close(S_gpu, S_orc, G, W):
    assert S_gpu.dtype == np.float32 and S_gpu.shape == S_orc.shape
    # fp64 summation error bound, in units of the row's sum of |G| |W| (>= sum |G dW| / 1)
    slack = 64 * W.shape[1] * 2.0 ** -52 * (np.abs(G.astype(np.float64)) * (np.abs(W.astype(np.float64)) + 1)).sum(1)
    err = np.abs(S_gpu.astype(np.float64) - S_orc)
    assert (err <= 2.0 ** -23 * S_orc + slack).all(), float((err / np.maximum(S_orc, 1e-300)).max())


@pytest.mark.parametrize("g", [64, 128])
@pytest.mark.parametrize("wdt,gdt", [(np.float32, np.float32), (np.float16, np.float16),
                                     (np.float16, np.float32), (np.float32, np.float16)])
def test_saliency_matches_oracle(orc, g, wdt, gdt):
    rng = np.random.default_rng(g + 3 * (wdt == np.float16) + (gdt == np.float16))
    N, K = 301, 1024                       # a ragged last block of eight rows
    W = inputs.weights(rng, N, K, outlier_frac=0.001).astype(wdt)
    G = inputs.gradients(rng, N, K, dtype=gdt)
    S = gpu_saliency(W, G, g)
    S_o = orc.saliency(W.astype(np.float32), G.astype(np.float32), g)
    assert_saliency_close(S, S_o, G, W)
    assert (S > 0).all()


def test_saliency_strided_rows(orc):
    rng = np.random.default_rng(5)
    N, K = 70, 512
    Wb = inputs.weights(rng, N, K + 96)
    Gb = inputs.gradients(rng, N, K + 160)
    Wd, Gd = to_dev(Wb)[:, 32:32 + K], to_dev(Gb)[:, :K]
    S = mx.mx_saliency(Wd, Gd, 128).cpu().numpy()
    W, G = Wb[:, 32:32 + K], Gb[:, :K]
    assert_saliency_close(S, orc.saliency(W, G, 128), G, W)


def test_saliency_degenerate_rows(orc):
    # all-zero rows (scale 0 -> 1: dW = 0), constant rows, rows on the 4-bit grid,
    # zero gradients and very large gradients (the second-order term dominates)
    rng = np.random.default_rng(6)
    N, K = 16, 256
    W = inputs.weights(rng, N, K)
    G = inputs.gradients(rng, N, K)
    W[0] = 0.0
    W[1] = 0.37
    W[2] = (rng.integers(0, 16, K) - 7) * np.float32(0.0078125)    # exact on a 4-bit grid
    G[3] = 0.0
    G[4] *= 1e6
    W[5, :128] = 1e4                                                # one huge group
    S = gpu_saliency(W, G, 128)
    S_o = orc.saliency(W, G, 128)
    assert_saliency_close(S, S_o, G, W)
    assert S[0] == 0 and S[2] == 0 and S[3] == 0


@pytest.mark.parametrize("K,N", [(4096, 14336), (14336, 4096)])
def test_saliency_llama_shapes(orc, K, N):
    rng = np.random.default_rng(K + N)
    W = inputs.weights(rng, N, K, outlier_frac=0.001)
    G = inputs.gradients(rng, N, K)
    S = gpu_saliency(W, G, 128)
    assert_saliency_close(S, orc.saliency(W, G, 128), G, W)


def test_saliency_rejects_bad_arguments():
    lib = mx.lib()
    W = torch.zeros((4, 256), device=dev())
    S = torch.zeros(4, device=dev())
    P = W.data_ptr()
    assert lib.mx_saliency(P, 0, 256, P, 0, 256, 4, 256, 96, S.data_ptr(), None) != 0     # group 96
    assert lib.mx_saliency(P, 0, 256, P, 0, 256, 4, 200, 128, S.data_ptr(), None) != 0    # K % g
    assert lib.mx_saliency(P, 0, 100, P, 0, 256, 4, 256, 128, S.data_ptr(), None) != 0    # ldw < K
    host = torch.zeros((4, 256))
    assert lib.mx_saliency(host.data_ptr(), 0, 256, P, 0, 256, 4, 256, 128, S.data_ptr(), None) != 0
    assert lib.mx_saliency(P, 0, 256, P, 0, 256, 0, 256, 128, S.data_ptr(), None) == 0    # no rows


# ------------------------------------------------------------------ global selection
def gpu_select(S: np.ndarray, n_top: int) -> np.ndarray:
    m = mx.mx_select_top(to_dev(S.astype(np.float32)), n_top)
    torch.cuda.synchronize()
    return m.cpu().numpy()


@pytest.mark.parametrize("n", [1, 2, 255, 256, 257, 10007])
def test_select_counts(orc, n):
    rng = np.random.default_rng(n)
    S = np.abs(rng.standard_normal(n)).astype(np.float32)
    for n_top in sorted({0, 1, n // 10, n // 2, n - 1, n}):
        m = gpu_select(S, n_top)
        assert m.dtype == np.uint8 and int(m.sum()) == n_top
        assert np.array_equal(m, orc.select_top(S, n_top)), n_top


def test_select_ties_go_to_the_lower_index(orc):
    rng = np.random.default_rng(11)
    n = 50000
    S = rng.integers(0, 5, n).astype(np.float32) * np.float32(0.25)   # five values, many ties
    S[rng.integers(0, n, 500)] = 0.0
    for n_top in (1, 7, 9999, 10000, 10001, 25000, n - 3):
        assert np.array_equal(gpu_select(S, n_top), orc.select_top(S, n_top)), n_top
    same = np.full(1000, np.float32(3.5))          # all equal: the first n_top rows
    m = gpu_select(same, 123)
    assert m[:123].all() and not m[123:].any()


def test_select_wide_range_and_subnormals(orc):
    rng = np.random.default_rng(12)
    n = 4096
    S = (np.abs(rng.standard_normal(n)) * 10.0 ** rng.uniform(-44, 30, n)).astype(np.float32)
    S[:8] = np.float32(1e-45)                       # the smallest subnormal
    S[8:12] = np.inf
    for n_top in (3, 4, 5, 400, 4088, 4089):
        assert np.array_equal(gpu_select(S, n_top), orc.select_top(S, n_top)), n_top


def test_select_millions_of_rows(orc):
    # the row count of all linear layers of a 70B model is about 3.3 million
    rng = np.random.default_rng(13)
    n = 3_300_001
    S = np.abs(rng.standard_normal(n)).astype(np.float32)
    S[rng.integers(0, n, 100000)] = np.float32(0.5)    # a big tie group
    n_top = int(0.1 * n)
    assert np.array_equal(gpu_select(S, n_top), orc.select_top(S, n_top))


def test_select_rejects_bad_arguments():
    lib = mx.lib()
    S = torch.zeros(64, device=dev())
    m = torch.zeros(64, dtype=torch.uint8, device=dev())
    ws = torch.zeros(4096, dtype=torch.uint8, device=dev())
    assert lib.mx_select_top(S.data_ptr(), 64, 65, m.data_ptr(), ws.data_ptr(), 4096, None) == 1
    assert lib.mx_select_top(S.data_ptr(), 64, -1, m.data_ptr(), ws.data_ptr(), 4096, None) == 1
    assert lib.mx_select_top(S.data_ptr(), 64, 3, m.data_ptr(), ws.data_ptr(), 8, None) == 7   # workspace
    assert lib.mx_select_top(S.data_ptr(), 64, 3, m.data_ptr(), ws.data_ptr() + 4, 4000, None) != 0
    assert lib.mx_select_top(S.data_ptr(), 0, 0, m.data_ptr(), None, 0, None) == 0              # nothing
    torch.cuda.synchronize()
    assert not m.any()


# ------------------------------------------------------------------ the whole search, then the layer
def test_search_over_layers_then_pack_and_gemm(orc):
    # three layers of different shapes: saliency per layer, one global choice of 10%
    # of all rows, each layer packed with its slice of the mask, then a layer call
    rng = np.random.default_rng(21)
    shapes = [(384, 512), (256, 1024), (640, 512)]          # (N, K)
    Ws = [inputs.weights(rng, N, K, outlier_frac=0.001) for N, K in shapes]
    Gs = [inputs.gradients(rng, N, K) for N, K in shapes]
    S_gpu = [mx.mx_saliency(to_dev(W), to_dev(G), 128) for W, G in zip(Ws, Gs)]
    S_all = torch.cat(S_gpu)
    n_top = int(0.10 * S_all.numel())
    mask = mx.mx_select_top(S_all, n_top).cpu().numpy()
    S_np = S_all.cpu().numpy()
    # the scores against the oracle's, the choice against the oracle's choice on them
    S_o = [orc.saliency(W, G, 128) for W, G in zip(Ws, Gs)]
    for Sg, So, W, G in zip(S_gpu, S_o, Ws, Gs):
        assert_saliency_close(Sg.cpu().numpy(), So, G, W)
    S_o = np.concatenate(S_o)
    assert np.array_equal(mask, orc.select_top(S_np, n_top))
    if np.array_equal(S_np, S_o.astype(np.float32)):        # the usual case: same fp32 scores
        assert np.array_equal(mask, orc.select_top(S_o.astype(np.float32), n_top))
    # a layer's share of the 8-bit rows follows its scores, not a fixed fraction
    off = 0
    for (N, K), W in zip(shapes, Ws):
        is8 = mask[off:off + N]
        off += N
        check_pack(orc, W, is8, 128)
        X = inputs.activations(rng, 40, K, 4)
        run_and_check(orc, X, W, is8, 128)
