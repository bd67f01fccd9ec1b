"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle.

Bit-exact: activation codes and scales, the row permutation, every packed code,
zero point and scale (after the test-side unpack of the documented layout), and
every per-group int32 partial.  Y within the tolerance stated in gpu_helpers.
"""
import numpy as np
import pytest
import torch

from mixed_precision_quantized_mx_b200 import binding as mx
from mixed_precision_quantized_mx_b200 import inputs

from blob_unpack import unpack
from gpu_helpers import (assert_y_close, dev, f16bits, gpu_gemm, gpu_pack, gpu_quant, to_dev)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    from mixed_precision_quantized_mx_b200 import build
    build.build()
    assert torch.cuda.is_available()
    mx.lib()


def check_quant(orc, X):
    Aq, sa = gpu_quant(X)
    Aq_o, sa_o = orc.quant_act(X.astype(np.float32))
    assert np.array_equal(Aq.cpu().numpy(), Aq_o)
    assert np.array_equal(f16bits(sa), sa_o)
    return Aq, sa, Aq_o, sa_o


def check_pack(orc, W, is8, g):
    L, blob = gpu_pack(W, is8, g)
    u = unpack(blob.cpu().numpy(), L)
    c = orc.pack(W.astype(np.float32), is8, g)
    assert u["header"] == [0x4B50584D, 1, c.N, c.K, g, c.n8]
    assert np.array_equal(u["perm"], c.perm)
    assert (u["pad8"] == -1).all() and (u["pad4"] == -1).all()
    assert np.array_equal(u["codes8"], c.codes8)
    assert np.array_equal(u["scales8"], c.scales8)
    assert np.array_equal(u["codes4"], c.codes4)
    assert np.array_equal(u["zeros4"], c.zeros4)
    assert np.array_equal(u["scales4"], c.scales4)
    for k in ("pad_codes8", "pad_scales8", "pad_codes4", "pad_zeros4", "pad_scales4"):
        assert not u[k].any(), k
    return L, blob, c


# ------------------------------------------------------------------ activations
def test_quant_act_tiny(orc):
    check_quant(orc, inputs.tiny_layer(0).X)


@pytest.mark.parametrize("M,K", [(1, 4096), (3, 512), (64, 14336), (5, 296), (2, 28672)])
def test_quant_act_fp16_shapes(orc, M, K):
    rng = np.random.default_rng(M * 7 + K)
    check_quant(orc, inputs.activations(rng, M, K, max(1, K // 100)))


def test_quant_act_special_rows(orc):
    K = 256
    X = np.zeros((6, K), np.float32)
    X[1, :8] = [127, 2.5, 3.5, -2.5, 0.5, -0.5, 1.5, -127]            # ties with s = 1
    X[2] = np.linspace(-3e-9, 3e-9, K)                                  # fp16 scale underflows -> 1
    X[3] = np.linspace(-1e7, 2e7, K)                                    # fp16 scale saturates
    X[4] = 1.0
    X[5, 100] = -65504.0
    Aq, sa, Aq_o, sa_o = check_quant(orc, X)
    assert sa_o[0] == 0x3C00 and not Aq_o[0].any()
    assert Aq_o[1, :8].tolist() == [127, 2, 4, -2, 0, 0, 2, -127]
    check_quant(orc, X[[0, 1, 2, 4, 5]].astype(np.float16))       # rows that fp16 can hold


def test_quant_act_rounding_boundaries(orc):
    """Values at and one ulp either side of every half-integer multiple of the scale:
    the codes are decided by fl(x / s), the IEEE fp32 quotient, then round-half-even."""
    K = 1024
    rng = np.random.default_rng(21)
    rows = []
    for amax in (127.0, 100.0, 3.0, 0.37, 1.0e-3):
        s = np.float32(np.float16(np.float32(amax) / np.float32(127.0)))   # the fp16 scale
        k = rng.integers(-127, 127, K).astype(np.float32)
        x = (k + np.float32(0.5)) * s                                     # near ties
        nudge = rng.integers(-1, 2, K)                                    # -1, 0, +1 ulp
        x = np.where(nudge > 0, np.nextafter(x, np.float32(np.inf)),
                     np.where(nudge < 0, np.nextafter(x, np.float32(-np.inf)), x)).astype(np.float32)
        x = np.clip(x, -amax, amax)
        x[0] = amax                                                       # pins the scale
        rows.append(x)
    X = np.stack(rows).astype(np.float32)
    Aq, sa, Aq_o, sa_o = check_quant(orc, X)
    # the rows hit every kind of decision: exact ties and both neighbours
    q = Aq_o.astype(np.float64)
    assert (np.abs(q) == 127).any() and len(np.unique(q)) > 200


def test_quant_act_strided_rows(orc):
    rng = np.random.default_rng(3)
    Xbig = inputs.activations(rng, 9, 640, 6)
    Xd = to_dev(Xbig)[:, :512]                                           # ldx = 640 > K
    Aq = torch.empty((9, 512), dtype=torch.int8, device=dev())
    sa = torch.empty((9,), dtype=torch.float16, device=dev())
    mx.mx_quant_act(Xd, Aq, sa)
    Aq_o, sa_o = orc.quant_act(Xbig[:, :512].astype(np.float32))
    assert np.array_equal(Aq.cpu().numpy(), Aq_o) and np.array_equal(f16bits(sa), sa_o)


# ------------------------------------------------------------------ packing
def test_pack_tiny(orc):
    L = inputs.tiny_layer(0)
    check_pack(orc, L.W, L.is8, L.group)


@pytest.mark.parametrize("N,K,g,n8,dtype", [
    (300, 256, 64, 37, np.float32), (200, 384, 128, 0, np.float32),
    (130, 128, 128, 130, np.float32), (257, 512, 128, 129, np.float16),
    (64, 1024, 64, 1, np.float16)])
def test_pack_ragged_and_degenerate(orc, N, K, g, n8, dtype):
    rng = np.random.default_rng(N + K + n8)
    W = inputs.weights(rng, N, K, outlier_frac=0.01).astype(dtype)
    is8 = inputs.saliency_mask(np.abs(rng.standard_normal(N)), n8)
    if dtype == np.float16:
        W[0, :g] = 0.0                          # an all-zero group
        W[1, :g] = -0.01                        # an all-negative constant group
    check_pack(orc, W, is8, g)


def test_pack_strided_fp16_weights(orc):
    rng = np.random.default_rng(5)
    Wbig = inputs.weights(rng, 160, 384).astype(np.float16)
    is8 = inputs.saliency_mask(np.abs(rng.standard_normal(160)), 20)
    L = mx.mx_layout_init(160, 256, 128, 20)
    blob = torch.empty(L.total_bytes, dtype=torch.uint8, device=dev())
    mx.mx_pack_weights(L, to_dev(Wbig)[:, :256], to_dev(is8), blob)
    u = unpack(blob.cpu().numpy(), L)
    c = orc.pack(Wbig[:, :256].astype(np.float32), is8, 128)
    assert np.array_equal(u["codes4"], c.codes4) and np.array_equal(u["codes8"], c.codes8)
    assert np.array_equal(u["scales4"], c.scales4) and np.array_equal(u["zeros4"], c.zeros4)


def test_pack_mask_count_mismatch_reports_status(orc):
    rng = np.random.default_rng(6)
    W = inputs.weights(rng, 200, 128)
    is8 = np.zeros(200, np.uint8)
    is8[:30] = 1
    status = torch.zeros(1, dtype=torch.int32, device=dev())
    gpu_pack(W, is8, 128, n8=20, status=status)     # claims 20, mask has 30
    assert int(status.item()) == 1
    status.zero_()
    gpu_pack(W, is8, 128, n8=40, status=status)     # claims 40, mask has 30
    assert int(status.item()) == 1
    status.zero_()
    gpu_pack(W, is8, 128, n8=30, status=status)
    assert int(status.item()) == 0


# ------------------------------------------------------------------ GEMM
def run_and_check(orc, X, W, is8, g, path=0, split=0, check_partials=True):
    Aq, sa, Aq_o, sa_o = check_quant(orc, X)
    L, blob, c = check_pack(orc, W, is8, g)
    Y, P, Yfull = gpu_gemm(L, blob, Aq, sa, path=path, split=split, debug=check_partials)
    if check_partials:
        P_o, pmax = orc.partials(Aq_o, c)
        assert pmax < 2 ** 22
        assert np.array_equal(P.cpu().numpy().astype(np.int64), P_o)
    yd, yt = orc.gemm(Aq_o, sa_o, c)
    assert_y_close(Y.cpu().numpy(), yt)
    if Yfull.shape[1] > L.N:
        assert torch.isnan(Yfull[:, L.N:]).all()
    return Y


def test_gemm_tiny(orc):
    L = inputs.tiny_layer(0)
    run_and_check(orc, L.X, L.W, L.is8, L.group)


@pytest.mark.parametrize("M", [1, 2, 3, 5, 8, 16, 17, 33])
@pytest.mark.parametrize("g", [64, 128])
def test_gemm_token_counts(orc, M, g):
    rng = np.random.default_rng(M * 13 + g)
    N, K = 300, 512
    X = inputs.activations(rng, M, K, 5)
    W = inputs.weights(rng, N, K, outlier_frac=0.001)
    is8 = inputs.saliency_mask(np.abs(rng.standard_normal(N)), 37)
    run_and_check(orc, X, W, is8, g)


@pytest.mark.parametrize("split", [1, 2, 3, 7])
def test_gemm_split_factors(orc, split):
    rng = np.random.default_rng(split)
    M, N, K = 4, 260, 1024
    X = inputs.activations(rng, M, K, 10)
    W = inputs.weights(rng, N, K, outlier_frac=0.001)
    is8 = inputs.saliency_mask(np.abs(rng.standard_normal(N)), 26)
    run_and_check(orc, X, W, is8, 128, path=mx.PATH_SPLITK, split=split)


@pytest.mark.parametrize("frac", [0.0, 1.0])
def test_gemm_degenerate_fractions(orc, frac):
    rng = np.random.default_rng(int(frac * 10) + 1)
    M, N, K = 3, 256, 2048
    X = inputs.activations(rng, M, K, 20)
    W = inputs.weights(rng, N, K, outlier_frac=0.001)
    is8 = np.full(N, int(frac), np.uint8)
    run_and_check(orc, X, W, is8, 128)


def test_gemm_strided_output(orc):
    rng = np.random.default_rng(9)
    M, N, K = 2, 140, 256
    X = inputs.activations(rng, M, K, 3)
    W = inputs.weights(rng, N, K)
    is8 = inputs.saliency_mask(np.abs(rng.standard_normal(N)), 14)
    Aq, sa, Aq_o, sa_o = check_quant(orc, X)
    L, blob, c = check_pack(orc, W, is8, 128)
    Y, _, Yfull = gpu_gemm(L, blob, Aq, sa, ldy=200)
    assert torch.isnan(Yfull[:, N:]).all()
    assert_y_close(Y.cpu().numpy(), orc.gemm(Aq_o, sa_o, c)[1])


# ------------------------------------------------------------------ full sizes, sampled
@pytest.mark.parametrize("M,K,N", [(1, 4096, 4096), (16, 4096, 4096), (1, 8192, 28672),
                                   (4, 28672, 8192)])
def test_gemm_llama_shapes_sampled(orc, M, K, N):
    lay = inputs.llama_layer(M, K, N, seed=M + K)
    Aq, sa, Aq_o, sa_o = check_quant(orc, lay.X)
    L, blob = gpu_pack(lay.W, lay.is8, 128)
    c = orc.pack(lay.W, lay.is8, 128)
    u = unpack(blob.cpu().numpy(), L)
    assert np.array_equal(u["perm"], c.perm)
    assert np.array_equal(u["codes4"], c.codes4) and np.array_equal(u["codes8"], c.codes8)
    Y, _, _ = gpu_gemm(L, blob, Aq, sa)
    Yh = Y.cpu().numpy()
    rng = np.random.default_rng(0)
    # token 0 against every output row, plus random (token, row) pairs
    n_all = np.arange(N)
    y0 = orc.gemm(Aq_o, sa_o, c, pairs=(np.zeros(N, np.int32), n_all))[1]
    assert_y_close(Yh[0], y0)
    pm = rng.integers(0, M, 512)
    pn = rng.integers(0, N, 512)
    yr = orc.gemm(Aq_o, sa_o, c, pairs=(pm, pn))[1]
    assert_y_close(Yh[pm, pn], yr, rows_rms=np.sqrt(np.mean(y0 ** 2)))


# ------------------------------------------------------------------ errors
def test_gemm_rejects_bad_arguments(orc):
    rng = np.random.default_rng(11)
    X = inputs.activations(rng, 2, 256, 2)
    W = inputs.weights(rng, 140, 256)
    is8 = inputs.saliency_mask(np.abs(rng.standard_normal(140)), 14)
    Aq, sa = gpu_quant(X)
    L, blob = gpu_pack(W, is8, 128)
    Y = torch.empty((2, 140), dtype=torch.float16, device=dev())
    assert mx.mx_gemm_workspace_size(L, 2, path=mx.PATH_SPLITK) == 0
    ws = None
    with pytest.raises(mx.MXError) as e:                      # host memory is refused
        mx.mx_gemm(L, blob, Aq.cpu(), sa, Y, path=mx.PATH_SPLITK)
    assert e.value.status == 1
    with pytest.raises(mx.MXError) as e:                      # cluster split above 8
        mx.mx_gemm(L, blob, Aq, sa, Y, path=mx.PATH_SPLITK, split=9)
    assert e.value.status == 2
    raw = torch.empty(2 * 256 + 16, dtype=torch.uint8, device=dev())
    Aq_mis = raw[1:1 + 512].view(torch.int8).view(2, 256)
    with pytest.raises(mx.MXError) as e:
        mx.mx_gemm(L, blob, Aq_mis, sa, Y, path=mx.PATH_SPLITK)
    assert e.value.status == 3
    Xh = torch.from_numpy(X)
    with pytest.raises(mx.MXError) as e:
        mx.mx_quant_act(Xh, Aq, sa)
    assert e.value.status == 1


# ------------------------------------------------------------------ tensor-core path
@pytest.mark.parametrize("M", [1, 17, 128, 129, 300])
@pytest.mark.parametrize("g", [64, 128])
def test_gemm_tc_token_counts(orc, M, g):
    rng = np.random.default_rng(M * 31 + g)
    N, K = 300, 512
    X = inputs.activations(rng, M, K, 5)
    W = inputs.weights(rng, N, K, outlier_frac=0.001)
    is8 = inputs.saliency_mask(np.abs(rng.standard_normal(N)), 37)
    run_and_check(orc, X, W, is8, g, path=mx.PATH_TENSOR)


@pytest.mark.parametrize("frac", [0.0, 1.0])
def test_gemm_tc_degenerate_fractions(orc, frac):
    rng = np.random.default_rng(int(frac * 10) + 7)
    M, N, K = 130, 256, 2048
    X = inputs.activations(rng, M, K, 20)
    W = inputs.weights(rng, N, K, outlier_frac=0.001)
    is8 = np.full(N, int(frac), np.uint8)
    run_and_check(orc, X, W, is8, 128, path=mx.PATH_TENSOR)


# ------------------------------------------------------------------ row path (3)
@pytest.mark.parametrize("M", [1, 2, 3, 4])
@pytest.mark.parametrize("g", [64, 128])
def test_rows_path(orc, M, g):
    lay = inputs.llama_layer(M, 1024, 520, group=g, seed=40 + M + g)
    run_and_check(orc, lay.X, lay.W, lay.is8, g, path=mx.PATH_ROWS)


@pytest.mark.parametrize("N,K,n8", [(256, 512, 0), (256, 512, 256), (130, 384, 3), (4096, 4096, 410),
                                    (1000, 128, 100)])
def test_rows_path_shapes(orc, N, K, n8):
    rng = np.random.default_rng(N + K + n8)
    W = inputs.weights(rng, N, K, outlier_frac=0.001)
    is8 = inputs.saliency_mask(np.abs(rng.standard_normal(N)), n8)
    X = inputs.activations(rng, 2, K, max(1, K // 100))
    run_and_check(orc, X, W, is8, 128, path=mx.PATH_ROWS)


def test_rows_path_refuses_what_it_cannot_serve():
    rng = np.random.default_rng(5)
    for N, K, M in ((256, 8192, 1), (256, 512, 5)):
        L, blob = gpu_pack(inputs.weights(rng, N, K), inputs.saliency_mask(np.abs(rng.standard_normal(N)), 10), 128)
        Aq, sa = gpu_quant(inputs.activations(rng, M, K, 4))
        Y = torch.empty((M, N), dtype=torch.float16, device=dev())
        with pytest.raises(mx.MXError) as e:
            mx.mx_gemm(L, blob, Aq, sa, Y, path=mx.PATH_ROWS)
        assert e.value.status == 2


def test_paths_agree_bit_exact_partials(orc):
    rng = np.random.default_rng(21)
    M, N, K = 24, 400, 1024
    X = inputs.activations(rng, M, K, 10)
    W = inputs.weights(rng, N, K, outlier_frac=0.001)
    is8 = inputs.saliency_mask(np.abs(rng.standard_normal(N)), 40)
    Aq, sa = gpu_quant(X)
    L, blob = gpu_pack(W, is8, 128)
    Y1, P1, _ = gpu_gemm(L, blob, Aq, sa, path=mx.PATH_SPLITK, debug=True)
    Y2, P2, _ = gpu_gemm(L, blob, Aq, sa, path=mx.PATH_TENSOR, debug=True)
    assert torch.equal(P1, P2)
    y1, y2 = Y1.float().cpu().numpy(), Y2.float().cpu().numpy()
    assert np.abs(y1 - y2).max() <= 2 * 2e-3 * np.abs(y1).max()


@pytest.mark.parametrize("M,K,N", [(256, 4096, 14336), (2048, 4096, 14336), (2048, 14336, 4096),
                                   (4096, 8192, 28672)])
def test_gemm_tc_llama_shapes_sampled(orc, M, K, N):
    lay = inputs.llama_layer(M, K, N, seed=M + K + N)
    Aq, sa, Aq_o, sa_o = check_quant(orc, lay.X)
    L, blob = gpu_pack(lay.W, lay.is8, 128)
    c = orc.pack(lay.W, lay.is8, 128)
    Y, _, _ = gpu_gemm(L, blob, Aq, sa, path=mx.PATH_TENSOR)
    Yh = Y.cpu().numpy()
    rng = np.random.default_rng(1)
    y0 = orc.gemm(Aq_o, sa_o, c, pairs=(np.full(N, M - 1, np.int32), np.arange(N)))[1]
    assert_y_close(Yh[M - 1], y0)
    rows = rng.integers(0, N, 8)
    ym = orc.gemm(Aq_o, sa_o, c, pairs=(np.repeat(np.arange(M), 8), np.tile(rows, M)))[1]
    assert_y_close(Yh[:, rows].reshape(-1), ym, rows_rms=np.sqrt(np.mean(y0 ** 2)))
    pm = rng.integers(0, M, 1024)
    pn = rng.integers(0, N, 1024)
    yr = orc.gemm(Aq_o, sa_o, c, pairs=(pm, pn))[1]
    assert_y_close(Yh[pm, pn], yr, rows_rms=np.sqrt(np.mean(y0 ** 2)))


@pytest.mark.parametrize("K", [128, 384, 640])
@pytest.mark.parametrize("g", [64, 128])
def test_gemm_tc_odd_kblocks(orc, K, g):
    # an odd number of 128-column k-blocks leaves the last pipeline stage half filled
    rng = np.random.default_rng(K + g)
    M, N = 150, 260
    X = inputs.activations(rng, M, K, 3)
    W = inputs.weights(rng, N, K, outlier_frac=0.002)
    is8 = inputs.saliency_mask(np.abs(rng.standard_normal(N)), 30)
    run_and_check(orc, X, W, is8, g, path=mx.PATH_TENSOR)
