"""Parity of the decode-sized tensor-core path (path 6: tcgen05.mma.cta_group::1,
128 weight rows x the batch rounded up to 16 tokens per MMA, K split over units and
reduced in split order) against the oracle.

Partials P[m, n, g] are compared bit for bit and Y within the tolerance of the other
paths.  Unsplit, path 6 adds the same fp32 products in the same group order as the
one-CTA tensor-core kernel (path 2), so their Y must be identical.  Split, Y must
repeat bit for bit.  Cases cover the four token tiles (16, 32, 64, 128) and batches
on both sides of their edges, both group sizes, one and many k-blocks, all-4-bit and
all-8-bit layers, ragged row tiles, group-wise activation scales, splits (even,
uneven, automatic, through mx_linear), the Llama-3 decode shapes on sampled outputs,
and the bounded waits.
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

P6 = mx.PATH_TC_DECODE


def _layer(rng, M, N, K, n8, outliers=4):
    X = inputs.activations(rng, M, K, outliers)
    W = inputs.weights(rng, N, K, outlier_frac=0.001)
    is8 = inputs.saliency_mask(np.abs(rng.standard_normal(N)), n8)
    return X, W, is8


@pytest.mark.parametrize("M", [1, 5, 15, 16, 17, 32, 33, 63, 64, 65, 100, 128])
@pytest.mark.parametrize("g", [64, 128])
def test_tc_decode_token_counts(orc, M, g):
    # N = 430 with 37 8-bit rows: one 8-bit and four 4-bit row tiles, the last ragged
    rng = np.random.default_rng(M * 17 + g)
    X, W, is8 = _layer(rng, M, 430, 512, 37)
    run_and_check(orc, X, W, is8, g, path=P6, split=1)


@pytest.mark.parametrize("K", [128, 384, 2560])
@pytest.mark.parametrize("split", [1, 2, 3, 7])
def test_tc_decode_splits(orc, K, split):
    rng = np.random.default_rng(K + split)
    X, W, is8 = _layer(rng, 16, 300, K, 30)
    Y = run_and_check(orc, X, W, is8, 128, path=P6, split=split)
    # the splits are added in a fixed order: the same Y every time
    Aq, sa = gpu_quant(X)
    L, blob = gpu_pack(W, is8, 128)
    Y2, _, _ = gpu_gemm(L, blob, Aq, sa, path=P6, split=split)
    assert torch.equal(Y.view(torch.int16), Y2.view(torch.int16))


@pytest.mark.parametrize("frac", [0.0, 1.0])
def test_tc_decode_degenerate_fractions(orc, frac):
    rng = np.random.default_rng(int(frac * 10) + 25)
    M, N, K = 24, 384, 640
    X, W, _ = _layer(rng, M, N, K, 0)
    is8 = np.full(N, frac == 1.0)
    run_and_check(orc, X, W, is8, 128, path=P6, split=2)


@pytest.mark.parametrize("M", [8, 16, 48, 128])
def test_tc_decode_equals_one_cta_kernel(orc, M):
    rng = np.random.default_rng(90 + M)
    N, K = 2300, 1024
    X, W, is8 = _layer(rng, M, N, K, 230)
    Aq, sa = gpu_quant(X)
    L, blob = gpu_pack(W, is8, 128)
    Y2, P2, _ = gpu_gemm(L, blob, Aq, sa, path=mx.PATH_TENSOR, debug=True)
    Y6, P6_, _ = gpu_gemm(L, blob, Aq, sa, path=P6, split=1, debug=True)
    assert torch.equal(P2, P6_)
    assert torch.equal(Y2.view(torch.int16), Y6.view(torch.int16))


@pytest.mark.parametrize("M", [3, 16, 40])
@pytest.mark.parametrize("g", [64, 128])
def test_tc_decode_group_wise_activations(orc, M, g):
    run_grouped(orc, M, 512, 430, g, path=P6, split=1, seed=M + g + 7)
    run_grouped(orc, M, 1024, 430, g, path=P6, split=3, seed=M + g + 8)


def test_tc_decode_strided_output_and_auto_split(orc):
    rng = np.random.default_rng(31)
    M, N, K = 16, 430, 2048
    X, W, is8 = _layer(rng, M, N, K, 37)
    Aq, sa = gpu_quant(X)
    L, blob = gpu_pack(W, is8, 128)
    assert mx.mx_gemm_workspace_size(L, M, path=P6) > 0        # the automatic choice splits K
    Y, _, Yfull = gpu_gemm(L, blob, Aq, sa, path=P6, ldy=N + 24)
    assert torch.isnan(Yfull[:, N:]).all()
    Aq_o, sa_o = orc.quant_act(X.astype(np.float32))
    assert_y_close(Y.cpu().numpy(), orc.gemm(Aq_o, sa_o, orc.pack(W, is8, 128))[1])
    # without the workspace the automatic split runs unsplit: Y equals split=1
    Yn = torch.zeros((M, N), dtype=torch.float16, device=dev())
    mx.mx_gemm(L, blob, Aq, sa, Yn, path=P6)
    Y1, _, _ = gpu_gemm(L, blob, Aq, sa, path=P6, split=1)
    torch.cuda.synchronize()
    assert torch.equal(Yn.view(torch.int16), Y1.view(torch.int16))


def test_tc_decode_through_mx_linear(orc):
    rng = np.random.default_rng(33)
    M, N, K = 24, 430, 2048
    X, W, is8 = _layer(rng, M, N, K, 37)
    L, blob = gpu_pack(W, is8, 128)
    Xd = torch.from_numpy(X).to(dev())
    n = mx.mx_linear_workspace_size(L, M, Xd.dtype, path=P6)
    ws = torch.empty(n, dtype=torch.uint8, device=dev())
    Y = torch.empty((M, N), dtype=torch.float16, device=dev())
    mx.mx_linear(L, blob, Xd, Y, workspace=ws, path=P6)
    Aq, sa = gpu_quant(X)
    Y2, _, _ = gpu_gemm(L, blob, Aq, sa, path=P6)
    torch.cuda.synchronize()
    assert torch.equal(Y.view(torch.int16), Y2.view(torch.int16))


def test_tc_decode_refusals(orc):
    rng = np.random.default_rng(35)
    X, W, is8 = _layer(rng, 129, 256, 256, 20)
    Aq, sa = gpu_quant(X)
    L, blob = gpu_pack(W, is8, 128)
    Y = torch.zeros((129, 256), dtype=torch.float16, device=dev())
    with pytest.raises(mx.MXError) as e:                     # beyond 128 tokens
        mx.mx_gemm(L, blob, Aq, sa, Y, path=P6)
    assert e.value.status == 2
    with pytest.raises(mx.MXError) as e:                     # an asked-for split needs its workspace
        mx.mx_gemm(L, blob, Aq[:16], sa[:16], Y[:16], path=P6, split=2)
    assert e.value.status == 7


@pytest.mark.parametrize("M,K,N", [(16, 4096, 4096), (8, 14336, 4096), (64, 8192, 28672), (128, 4096, 14336)])
def test_tc_decode_llama_shapes_sampled(orc, M, K, N):
    lay = inputs.llama_layer(M, K, N, seed=M + K + N + 3)
    Aq, sa, Aq_o, sa_o = check_quant(orc, lay.X)
    L, blob = gpu_pack(lay.W, lay.is8, 128)
    c = orc.pack(lay.W, lay.is8, 128)
    Y, _, _ = gpu_gemm(L, blob, Aq, sa, path=P6)
    Yh = Y.cpu().numpy()
    y0 = orc.gemm(Aq_o, sa_o, c, pairs=(np.full(N, M - 1, np.int32), np.arange(N)))[1]
    assert_y_close(Yh[M - 1], y0)
    rng = np.random.default_rng(4)
    pm = rng.integers(0, M, 2048)
    pn = rng.integers(0, N, 2048)
    yr = orc.gemm(Aq_o, sa_o, c, pairs=(pm, pn))[1]
    assert_y_close(Yh[pm, pn], yr, rows_rms=np.sqrt(np.mean(y0 ** 2)))


def test_tc_decode_wait_timeout_sets_status_and_context_survives(orc):
    rng = np.random.default_rng(39)
    M, N, K = 16, 430, 512
    X, W, is8 = _layer(rng, M, N, K, 26)
    Aq, sa = gpu_quant(X)
    L, blob = gpu_pack(W, is8, 128)
    Y = torch.zeros((M, N), dtype=torch.float16, device=dev())
    status = torch.zeros(1, dtype=torch.int32, device=dev())
    mx.mx_gemm(L, blob, Aq, sa, Y, path=P6, split=1, status=status, wait_timeout_us=20000, test_stall=1)
    torch.cuda.synchronize()
    assert int(status.item()) == 5             # MX_ERR_TIMEOUT
    status.zero_()
    Y2, _, _ = gpu_gemm(L, blob, Aq, sa, path=P6)
    Aq_o, sa_o = orc.quant_act(X.astype(np.float32))
    assert_y_close(Y2.cpu().numpy(), orc.gemm(Aq_o, sa_o, orc.pack(W, is8, 128))[1])
