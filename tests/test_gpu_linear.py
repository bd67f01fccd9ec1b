"""GPU parity of mx_linear, the one-call layer (quantize X, then the mixed GEMM).

For decode-sized M one kernel quantizes and multiplies; its per-group int32
partials must equal the oracle's bit for bit (so the activation codes it made
in shared memory are the oracle's), its Y must be identical to mx_quant_act
followed by mx_gemm, and close to the oracle's Y.  Larger M runs the two kernels
through the caller's workspace and must give the same Y as the two calls.
"""
import numpy as np
import pytest
import torch

from mixed_precision_quantized_mx_b200 import binding as mx
from mixed_precision_quantized_mx_b200 import inputs

from gpu_helpers import assert_y_close, dev, gpu_gemm, gpu_pack, gpu_quant, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    from mixed_precision_quantized_mx_b200 import build
    build.build()
    assert torch.cuda.is_available()
    mx.lib()


def run_linear(L, blob, Xd, path=0, split=0, debug=False, ws_pad=0):
    M = Xd.shape[0]
    Y = torch.full((M, L.N), float("nan"), dtype=torch.float16, device=dev())
    n = mx.mx_linear_workspace_size(L, M, Xd.dtype, path=path, split=split)
    ws = torch.empty(n + ws_pad, dtype=torch.uint8, device=dev()) if n + ws_pad else None
    P = None
    if debug:                      # guard zones on both sides catch writes outside P
        pad = 64
        Pbig = torch.full((M * L.N * L.G + 2 * pad,), -12345, dtype=torch.int32, device=dev())
        P = Pbig[pad:pad + M * L.N * L.G].view(M, L.N, L.G)
        P.zero_()
    mx.mx_linear(L, blob, Xd, Y, workspace=ws, path=path, split=split, debug_partials=P)
    torch.cuda.synchronize()
    if debug:
        assert (Pbig[:pad] == -12345).all() and (Pbig[-pad:] == -12345).all()
    return Y, P, n


def check_linear(orc, X, W, is8, g, xdtype, path=0, split=0, expect_fused=None):
    L, blob = gpu_pack(W, is8, g)
    Xd = to_dev(X).to(xdtype)
    Y, P, n = run_linear(L, blob, Xd, path=path, split=split, debug=True)
    if expect_fused is not None:
        assert (n == 0) == expect_fused
    Xo = Xd.float().cpu().numpy()
    Aq_o, sa_o = orc.quant_act(Xo)
    c = orc.pack(W.astype(np.float32), is8, g)
    P_o, _ = orc.partials(Aq_o, c)
    assert np.array_equal(P.cpu().numpy().astype(np.int64), P_o)
    Yh, Yref = Y.cpu().numpy(), orc.gemm(Aq_o, sa_o, c)[1]
    big = np.abs(Yref) > 70000.0                  # beyond fp16: must round to inf of the same sign
    assert np.array_equal(Yh[big], np.sign(Yref[big]) * np.inf)
    fin = ~big.any(axis=1)
    assert_y_close(Yh[fin], Yref[fin])
    # the same codes, scales and GEMM as the two separate calls
    Aq, sa = gpu_quant(Xo.astype(np.float16) if xdtype == torch.float16 else Xo)
    Y2 = gpu_gemm(L, blob, Aq, sa, path=path, split=split)[0]
    assert torch.equal(Y, Y2)
    return Y


@pytest.mark.parametrize("M", [1, 2, 3, 4])
@pytest.mark.parametrize("xdtype", [torch.float16, torch.float32])
def test_fused_decode(orc, M, xdtype):
    lay = inputs.llama_layer(M, 2048, 520, seed=30 + M)
    check_linear(orc, lay.X, lay.W, lay.is8, 128, xdtype, expect_fused=True)


@pytest.mark.parametrize("split", [1, 2, 3, 8])
def test_fused_decode_cluster_sizes(orc, split):
    lay = inputs.llama_layer(2, 4096, 300, seed=split)
    check_linear(orc, lay.X, lay.W, lay.is8, 64, torch.float16, split=split, expect_fused=True)


@pytest.mark.parametrize("N,K,M", [(4096, 4096, 1), (1024, 14336, 2), (260, 128, 4), (128, 256, 1)])
def test_fused_decode_llama_shapes(orc, N, K, M):
    lay = inputs.llama_layer(M, K, N, seed=N + K)
    check_linear(orc, lay.X, lay.W, lay.is8, 128, torch.float16, expect_fused=True)


def test_fused_decode_all_8bit_and_all_4bit(orc):
    rng = np.random.default_rng(5)
    W = inputs.weights(rng, 256, 1024)
    X = inputs.activations(rng, 3, 1024, 10)
    for is8 in (np.ones(256, np.uint8), np.zeros(256, np.uint8)):
        check_linear(orc, X, W, is8, 128, torch.float16, expect_fused=True)


def test_fused_decode_special_rows(orc):
    rng = np.random.default_rng(9)
    lay = inputs.llama_layer(4, 1024, 300, seed=9)
    X = lay.X.copy()
    X[0] = 0.0                                     # all-zero token: scale 1, codes 0
    X[2, 17] = 60000.0                             # one huge outlier
    check_linear(orc, X, lay.W, lay.is8, 128, torch.float16, expect_fused=True)
    X32 = lay.X.astype(np.float32)
    X32[1] = np.linspace(-3e-9, 3e-9, 1024)        # fp16 scale underflows to 0 -> 1
    X32[3] = rng.standard_normal(1024) * 1e6       # fp16 scale saturates; Y overflows fp16
    check_linear(orc, X32, lay.W, lay.is8, 128, torch.float32, expect_fused=True)


def test_fused_decode_strided_rows(orc):
    lay = inputs.llama_layer(3, 1024, 400, seed=4)
    L, blob = gpu_pack(lay.W, lay.is8, 128)
    big = torch.zeros((3, 1024 + 64), dtype=torch.float16, device=dev())
    big[:, :1024] = to_dev(lay.X)
    Xv = big[:, :1024]
    Y, _, n = run_linear(L, blob, Xv)
    Y2, _, _ = run_linear(L, blob, Xv.contiguous())
    assert n == 0 and torch.equal(Y, Y2)


@pytest.mark.parametrize("M", [5, 17, 200])
def test_two_kernel_path_with_workspace(orc, M):
    lay = inputs.llama_layer(M, 1024, 300, seed=M)
    check_linear(orc, lay.X, lay.W, lay.is8, 128, torch.float16, expect_fused=False)


def test_forced_tensor_path_and_wide_fp32_rows(orc):
    lay = inputs.llama_layer(2, 512, 260, seed=11)
    check_linear(orc, lay.X, lay.W, lay.is8, 128, torch.float16, path=mx.PATH_TENSOR, expect_fused=False)
    # 4 fp32 rows of 20480 columns (320 KB) are too wide to stage: two kernels
    rng = np.random.default_rng(12)
    X = inputs.activations(rng, 4, 20480, 20)
    W = inputs.weights(rng, 130, 20480)
    is8 = inputs.saliency_mask(np.abs(rng.standard_normal(130)), 13)
    check_linear(orc, X, W, is8, 128, torch.float32, expect_fused=False)


def test_workspace_errors():
    lay = inputs.llama_layer(8, 512, 256, seed=2)
    L, blob = gpu_pack(lay.W, lay.is8, 128)
    Xd = to_dev(lay.X)
    Y = torch.empty((8, 256), dtype=torch.float16, device=dev())
    n = mx.mx_linear_workspace_size(L, 8, torch.float16)
    assert n == 8 * 512 + 16
    for ws in (None, torch.empty(n - 1, dtype=torch.uint8, device=dev())):
        with pytest.raises(mx.MXError) as e:
            mx.mx_linear(L, blob, Xd, Y, workspace=ws)
        assert e.value.status == 7
    with pytest.raises(mx.MXError) as e:              # workspace not 16-byte aligned
        mx.mx_linear(L, blob, Xd, Y, workspace=torch.empty(n + 16, dtype=torch.uint8, device=dev())[1:])
    assert e.value.status == 3
    # a larger workspace than needed is fine
    Y1, _, _ = run_linear(L, blob, Xd, ws_pad=4096)
    Y2, _, _ = run_linear(L, blob, Xd)
    assert torch.equal(Y1, Y2)
