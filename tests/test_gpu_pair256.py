"""Parity of the tensor-core path on CTA pairs with 256-token tiles (path 5:
cta_group::2, M = N = 256 per MMA, two group accumulators of 256 TMEM columns)
against the oracle.

Partials P[m, n, g] are compared bit for bit, Y within the tolerance of the
other paths.  Path 5 does the same fp32 arithmetic in the same group order as the
unsplit 128-token pair kernel and the one-CTA kernel, so their Y must be identical
too.  Shapes cover an odd number of row tiles (the last pair has a CTA without
rows), token counts on both sides of the 128-token halves and the 256-token
tiles, both group sizes (g = 64 puts two groups in each k-block, so both
accumulators turn over inside one stage), one and many k-blocks, all-4-bit and
all-8-bit layers, group-wise activation scales, the full Llama-3 shapes on
sampled outputs, the automatic choice of this path, and the bounded waits.
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

P5 = mx.PATH_PAIR256


def _layer(rng, M, N, K, n8, outliers=4):
    X = inputs.activations(rng, M, K, outliers)
    W = inputs.weights(rng, N, K, outlier_frac=0.001)
    is8 = inputs.saliency_mask(np.abs(rng.standard_normal(N)), n8)
    return X, W, is8


@pytest.mark.parametrize("M", [1, 127, 128, 129, 255, 256, 257, 600])
@pytest.mark.parametrize("g", [64, 128])
def test_pair256_token_counts(orc, M, g):
    # N = 430 with 37 8-bit rows: one 8-bit and four 4-bit row tiles, so the last
    # pair's odd CTA has no rows
    rng = np.random.default_rng(M * 13 + g)
    X, W, is8 = _layer(rng, M, 430, 512, 37)
    run_and_check(orc, X, W, is8, g, path=P5)


@pytest.mark.parametrize("K", [128, 384, 1152, 2560])
def test_pair256_kblock_counts(orc, K):
    rng = np.random.default_rng(K + 1)
    X, W, is8 = _layer(rng, 300, 300, K, 30)
    run_and_check(orc, X, W, is8, 128, path=P5)


@pytest.mark.parametrize("frac", [0.0, 1.0])
def test_pair256_degenerate_fractions(orc, frac):
    rng = np.random.default_rng(int(frac * 10) + 15)
    M, N, K = 300, 384, 640
    X, W, _ = _layer(rng, M, N, K, 0)
    is8 = np.full(N, frac == 1.0)
    run_and_check(orc, X, W, is8, 128, path=P5)


@pytest.mark.parametrize("g", [64, 128])
def test_pair256_equals_other_tensor_core_kernels(orc, g):
    # several units per pair of CTAs (the persistent walk wraps), mixed tile kinds
    rng = np.random.default_rng(78 + g)
    M, N, K = 900, 2300, 1024
    X, W, is8 = _layer(rng, M, N, K, 230)
    Aq, sa = gpu_quant(X)
    L, blob = gpu_pack(W, is8, g)
    Y2, P2, _ = gpu_gemm(L, blob, Aq, sa, path=mx.PATH_TENSOR, debug=True)
    Y4, P4, _ = gpu_gemm(L, blob, Aq, sa, path=mx.PATH_PAIR, split=1, debug=True)
    Y5, P5_, _ = gpu_gemm(L, blob, Aq, sa, path=P5, debug=True)
    assert torch.equal(P2, P5_) and torch.equal(P4, P5_)
    assert torch.equal(Y2.view(torch.int16), Y5.view(torch.int16))
    assert torch.equal(Y4.view(torch.int16), Y5.view(torch.int16))
    # without the partials buffer: the same Y
    Y5b, _, _ = gpu_gemm(L, blob, Aq, sa, path=P5)
    assert torch.equal(Y5b.view(torch.int16), Y5.view(torch.int16))


@pytest.mark.parametrize("M", [17, 300])
@pytest.mark.parametrize("g", [64, 128])
def test_pair256_group_wise_activations(orc, M, g):
    run_grouped(orc, M, 512, 430, g, path=P5, seed=M + g + 3)


def test_pair256_strided_output(orc):
    rng = np.random.default_rng(21)
    M, N, K = 260, 430, 512
    X, W, is8 = _layer(rng, M, N, K, 37)
    Aq, sa = gpu_quant(X)
    L, blob = gpu_pack(W, is8, 128)
    Y, _, Yfull = gpu_gemm(L, blob, Aq, sa, path=P5, ldy=N + 24)
    assert torch.isnan(Yfull[:, N:]).all()          # nothing written past column N
    Aq_o, sa_o = orc.quant_act(X.astype(np.float32))
    assert_y_close(Y.cpu().numpy(), orc.gemm(Aq_o, sa_o, orc.pack(W, is8, 128))[1])


@pytest.mark.parametrize("M,K,N", [(2048, 4096, 14336), (2048, 14336, 4096), (4096, 8192, 28672)])
def test_pair256_llama_shapes_sampled(orc, M, K, N):
    lay = inputs.llama_layer(M, K, N, seed=M + K + N + 2)
    Aq, sa, Aq_o, sa_o = check_quant(orc, lay.X)
    L, blob = gpu_pack(lay.W, lay.is8, 128)
    c = orc.pack(lay.W, lay.is8, 128)
    assert mx.mx_gemm_select_path(L, M) == P5          # the automatic choice at prefill M
    Y, _, _ = gpu_gemm(L, blob, Aq, sa)
    Yh = Y.cpu().numpy()
    rng = np.random.default_rng(3)
    y0 = orc.gemm(Aq_o, sa_o, c, pairs=(np.full(N, M - 1, np.int32), np.arange(N)))[1]
    assert_y_close(Yh[M - 1], y0)
    rows = rng.integers(0, N, 8)
    ym = orc.gemm(Aq_o, sa_o, c, pairs=(np.repeat(np.arange(M), 8), np.tile(rows, M)))[1]
    assert_y_close(Yh[:, rows].reshape(-1), ym, rows_rms=np.sqrt(np.mean(y0 ** 2)))
    pm = rng.integers(0, M, 1024)
    pn = rng.integers(0, N, 1024)
    yr = orc.gemm(Aq_o, sa_o, c, pairs=(pm, pn))[1]
    assert_y_close(Yh[pm, pn], yr, rows_rms=np.sqrt(np.mean(y0 ** 2)))


def test_pair256_wait_timeout_sets_status_and_context_survives(orc):
    rng = np.random.default_rng(19)
    M, N, K = 300, 430, 512
    X, W, is8 = _layer(rng, M, N, K, 26)
    Aq, sa = gpu_quant(X)
    L, blob = gpu_pack(W, is8, 128)
    Y = torch.zeros((M, N), dtype=torch.float16, device=dev())
    status = torch.zeros(1, dtype=torch.int32, device=dev())
    mx.mx_gemm(L, blob, Aq, sa, Y, path=P5, status=status, wait_timeout_us=20000, test_stall=1)
    torch.cuda.synchronize()
    assert int(status.item()) == 5             # MX_ERR_TIMEOUT
    status.zero_()
    Y2, _, _ = gpu_gemm(L, blob, Aq, sa, path=P5)
    Aq_o, sa_o = orc.quant_act(X.astype(np.float32))
    c = orc.pack(W, is8, 128)
    assert_y_close(Y2.cpu().numpy(), orc.gemm(Aq_o, sa_o, c)[1])
    mx.mx_gemm(L, blob, Aq, sa, Y, path=P5, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0


def test_pair256_refuses_a_split(orc):
    rng = np.random.default_rng(23)
    X, W, is8 = _layer(rng, 300, 256, 256, 20)
    Aq, sa = gpu_quant(X)
    L, blob = gpu_pack(W, is8, 128)
    Y = torch.zeros((300, 256), dtype=torch.float16, device=dev())
    with pytest.raises(mx.MXError) as e:
        mx.mx_gemm(L, blob, Aq, sa, Y, path=P5, split=2)
    assert e.value.status == 2
