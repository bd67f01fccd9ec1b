"""Parity of the tensor-core path on CTA pairs (path 4: cta_group::2, 256 weight
rows x 128 tokens per tile) against the oracle.

Partials P[m, n, g] are compared bit for bit, Y within the tolerance of the
other paths.  Unsplit, the pair kernel does the same arithmetic in the same order
as the one-CTA tensor-core kernel, so their Y must be identical too.  Shapes cover
an odd number of row tiles (the last pair has a CTA without rows), token counts on
both sides of the 64-token halves and the 128-token tiles, both group sizes,
all-4-bit and all-8-bit layers, group-wise activation scales, splits of K (even and
uneven, through mx_gemm and mx_linear, and the workspace they need), and the
bounded waits.
"""
import numpy as np
import pytest
import torch

from mixed_precision_quantized_mx_b200 import binding as mx
from mixed_precision_quantized_mx_b200 import inputs

from gpu_helpers import assert_y_close, dev, gpu_gemm, gpu_pack, gpu_quant
from test_gpu_act_group import run_grouped
from test_gpu_parity import check_quant, run_and_check

pytestmark = pytest.mark.gpu


def _layer(rng, M, N, K, n8, outliers=4):
    X = inputs.activations(rng, M, K, outliers)
    W = inputs.weights(rng, N, K, outlier_frac=0.001)
    is8 = inputs.saliency_mask(np.abs(rng.standard_normal(N)), n8)
    return X, W, is8


@pytest.mark.parametrize("M", [1, 63, 64, 65, 127, 128, 129, 400])
@pytest.mark.parametrize("g", [64, 128])
def test_pair_token_counts(orc, M, g):
    # N = 430 with 37 8-bit rows: one 8-bit and four 4-bit row tiles, so the last
    # pair's odd CTA has no rows
    rng = np.random.default_rng(M * 7 + g)
    X, W, is8 = _layer(rng, M, 430, 512, 37)
    run_and_check(orc, X, W, is8, g, path=mx.PATH_PAIR)


@pytest.mark.parametrize("K", [128, 384, 1152])
def test_pair_kblock_counts(orc, K):
    rng = np.random.default_rng(K)
    X, W, is8 = _layer(rng, 250, 300, K, 30)
    run_and_check(orc, X, W, is8, 128, path=mx.PATH_PAIR)


@pytest.mark.parametrize("frac", [0.0, 1.0])
def test_pair_degenerate_fractions(orc, frac):
    rng = np.random.default_rng(int(frac * 10) + 5)
    M, N, K = 200, 384, 640
    X, W, _ = _layer(rng, M, N, K, 0)
    is8 = np.full(N, frac == 1.0)
    run_and_check(orc, X, W, is8, 128, path=mx.PATH_PAIR)


def test_pair_equals_one_cta_kernel(orc):
    # several units per pair of CTAs (the persistent walk wraps), mixed tile kinds
    rng = np.random.default_rng(77)
    M, N, K = 700, 2300, 1024
    X, W, is8 = _layer(rng, M, N, K, 230)
    Aq, sa = gpu_quant(X)
    L, blob = gpu_pack(W, is8, 128)
    Y2, P2, _ = gpu_gemm(L, blob, Aq, sa, path=mx.PATH_TENSOR, debug=True)
    Y4, P4, _ = gpu_gemm(L, blob, Aq, sa, path=mx.PATH_PAIR, split=1, debug=True)   # unsplit
    assert torch.equal(P2, P4)
    assert torch.equal(Y2.view(torch.int16), Y4.view(torch.int16))


@pytest.mark.parametrize("M", [17, 300])
@pytest.mark.parametrize("g", [64, 128])
def test_pair_group_wise_activations(orc, M, g):
    run_grouped(orc, M, 512, 430, g, path=mx.PATH_PAIR, seed=M + g + 1)


@pytest.mark.parametrize("M,K,N", [(2048, 4096, 14336), (4096, 8192, 28672)])
def test_pair_llama_shapes_sampled(orc, M, K, N):
    lay = inputs.llama_layer(M, K, N, seed=M + K + N + 1)
    Aq, sa, Aq_o, sa_o = check_quant(orc, lay.X)
    L, blob = gpu_pack(lay.W, lay.is8, 128)
    c = orc.pack(lay.W, lay.is8, 128)
    Y, _, _ = gpu_gemm(L, blob, Aq, sa, path=mx.PATH_PAIR)
    Yh = Y.cpu().numpy()
    rng = np.random.default_rng(2)
    y0 = orc.gemm(Aq_o, sa_o, c, pairs=(np.full(N, M - 1, np.int32), np.arange(N)))[1]
    assert_y_close(Yh[M - 1], y0)
    rows = rng.integers(0, N, 8)
    ym = orc.gemm(Aq_o, sa_o, c, pairs=(np.repeat(np.arange(M), 8), np.tile(rows, M)))[1]
    assert_y_close(Yh[:, rows].reshape(-1), ym, rows_rms=np.sqrt(np.mean(y0 ** 2)))
    pm = rng.integers(0, M, 1024)
    pn = rng.integers(0, N, 1024)
    yr = orc.gemm(Aq_o, sa_o, c, pairs=(pm, pn))[1]
    assert_y_close(Yh[pm, pn], yr, rows_rms=np.sqrt(np.mean(y0 ** 2)))


def test_pair_wait_timeout_sets_status_and_context_survives(orc):
    rng = np.random.default_rng(9)
    M, N, K = 160, 430, 512
    X, W, is8 = _layer(rng, M, N, K, 26)
    Aq, sa = gpu_quant(X)
    L, blob = gpu_pack(W, is8, 128)
    Y = torch.zeros((M, N), dtype=torch.float16, device=dev())
    status = torch.zeros(1, dtype=torch.int32, device=dev())
    mx.mx_gemm(L, blob, Aq, sa, Y, path=mx.PATH_PAIR, status=status, wait_timeout_us=20000, test_stall=1)
    torch.cuda.synchronize()
    assert int(status.item()) == 5             # MX_ERR_TIMEOUT
    status.zero_()
    Y2, _, _ = gpu_gemm(L, blob, Aq, sa, path=mx.PATH_PAIR)
    Aq_o, sa_o = orc.quant_act(X.astype(np.float32))
    c = orc.pack(W, is8, 128)
    assert_y_close(Y2.cpu().numpy(), orc.gemm(Aq_o, sa_o, c)[1])
    mx.mx_gemm(L, blob, Aq, sa, Y, path=mx.PATH_PAIR, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0


# ------------------------------------------------------------------ K split over CTA pairs
@pytest.mark.parametrize("M", [1, 100, 300])
@pytest.mark.parametrize("split", [2, 3, 5])
def test_pair_split_matches_oracle(orc, M, split):
    # K = 1152: nine k-blocks in five stages, so the splits are uneven
    rng = np.random.default_rng(M + 31 * split)
    X, W, is8 = _layer(rng, M, 430, 1152, 37)
    Y = run_and_check(orc, X, W, is8, 128, path=mx.PATH_PAIR, split=split)
    # the splits are added in a fixed order: the same Y every time
    Aq, sa = gpu_quant(X)
    L, blob = gpu_pack(W, is8, 128)
    Y2, _, _ = gpu_gemm(L, blob, Aq, sa, path=mx.PATH_PAIR, split=split)
    assert torch.equal(Y.view(torch.int16), Y2.view(torch.int16))


def test_pair_split_group_wise_and_g64(orc):
    run_grouped(orc, 40, 1024, 430, 64, path=mx.PATH_PAIR, split=3, seed=5)


def test_pair_split_workspace_rules(orc):
    rng = np.random.default_rng(4)
    M, N, K = 64, 430, 1024
    X, W, is8 = _layer(rng, M, N, K, 37)
    Aq, sa = gpu_quant(X)
    L, blob = gpu_pack(W, is8, 128)
    Y = torch.zeros((M, N), dtype=torch.float16, device=dev())
    with pytest.raises(mx.MXError) as e:            # an asked-for split needs its workspace
        mx.mx_gemm(L, blob, Aq, sa, Y, path=mx.PATH_PAIR, split=2)
    assert e.value.status == 7
    # an automatic split without a workspace runs unsplit: bit-identical to split=1
    assert mx.mx_gemm_workspace_size(L, M, path=mx.PATH_PAIR) > 0
    mx.mx_gemm(L, blob, Aq, sa, Y, path=mx.PATH_PAIR)
    Y1, _, _ = gpu_gemm(L, blob, Aq, sa, path=mx.PATH_PAIR, split=1)
    torch.cuda.synchronize()
    assert torch.equal(Y.view(torch.int16), Y1.view(torch.int16))
    # with it, the automatic split agrees with the oracle
    Ya, _, _ = gpu_gemm(L, blob, Aq, sa, path=mx.PATH_PAIR)
    Aq_o, sa_o = orc.quant_act(X.astype(np.float32))
    assert_y_close(Ya.cpu().numpy(), orc.gemm(Aq_o, sa_o, orc.pack(W, is8, 128))[1])


def test_pair_split_through_mx_linear(orc):
    # the layer call sizes its workspace with the split sums and gives the two-call result
    rng = np.random.default_rng(8)
    M, N, K = 48, 430, 2048
    X, W, is8 = _layer(rng, M, N, K, 37)
    L, blob = gpu_pack(W, is8, 128)
    Xd = torch.from_numpy(X).to(dev())
    n = mx.mx_linear_workspace_size(L, M, Xd.dtype)
    assert n > mx.mx_linear_workspace_size(L, M, Xd.dtype, split=1)
    ws = torch.empty(n, dtype=torch.uint8, device=dev())
    Y = torch.empty((M, N), dtype=torch.float16, device=dev())
    mx.mx_linear(L, blob, Xd, Y, workspace=ws)
    Aq, sa = gpu_quant(X)
    Y2, _, _ = gpu_gemm(L, blob, Aq, sa)
    torch.cuda.synchronize()
    assert torch.equal(Y.view(torch.int16), Y2.view(torch.int16))
