"""GPU parity of group-wise activation scales (MixLLM section 3.1.2: activations
quantized group-wise, group 128 as the weights) against the oracle's act_group mode.

Bit-exact: codes and the [M][G] fp16 scales of the grouped quantizer, and every
per-group int32 partial.  Y within the tolerance of gpu_helpers; the fused and
two-kernel forms of mx_linear give identical Y.
"""
import numpy as np
import pytest
import torch

from mixed_precision_quantized_mx_b200 import binding as mx
from mixed_precision_quantized_mx_b200 import inputs

from gpu_helpers import assert_y_close, dev, f16bits, gpu_pack, gpu_quant_grouped, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    from mixed_precision_quantized_mx_b200 import build
    build.build()
    assert torch.cuda.is_available()
    mx.lib()


def check_quant_grouped(orc, X, g):
    Aq, sa = gpu_quant_grouped(X, g)
    Aq_o, sa_o = orc.quant_act(X.astype(np.float32), act_group=g)
    assert np.array_equal(Aq.cpu().numpy(), Aq_o)
    assert np.array_equal(f16bits(sa), sa_o)
    return Aq, sa, Aq_o, sa_o


@pytest.mark.parametrize("M,K,g", [(1, 512, 128), (5, 4096, 128), (3, 14336, 64), (7, 1024, 64), (2, 256, 128)])
@pytest.mark.parametrize("dtype", [np.float16, np.float32])
def test_quant_grouped(orc, M, K, g, dtype):
    rng = np.random.default_rng(M * K + g)
    check_quant_grouped(orc, inputs.activations(rng, M, K, max(1, K // 100), dtype=dtype), g)


def test_quant_grouped_special_groups(orc):
    K = 512
    X = np.random.default_rng(3).standard_normal((3, K)).astype(np.float32)
    X[0, :128] = 0.0                              # an all-zero group: scale 1, codes 0
    X[1, 128:256] = 1.0e-9                        # fp16 scale underflows -> 1
    X[2, 256:384] *= 1.0e6                        # fp16 scale saturates
    X[2, 384] = 127.0
    Aq, sa, Aq_o, sa_o = check_quant_grouped(orc, X, 128)
    assert sa_o[0, 0] == 0x3C00 and not Aq_o[0, :128].any()


def run_grouped(orc, M, K, N, g, path=0, split=0, seed=0):
    lay = inputs.llama_layer(M, K, N, group=g, seed=seed)
    L, blob = gpu_pack(lay.W, lay.is8, g)
    Aq, sa, Aq_o, sa_o = check_quant_grouped(orc, lay.X, g)
    Y = torch.full((M, N), float("nan"), dtype=torch.float16, device=dev())
    P = torch.zeros((M, N, L.G), dtype=torch.int32, device=dev())
    ws = torch.empty(max(16, mx.mx_gemm_workspace_size(L, M, path=path, split=split)), dtype=torch.uint8,
                     device=dev())
    mx.mx_gemm(L, blob, Aq, sa, Y, workspace=ws, path=path, split=split, debug_partials=P, act_group=g)
    torch.cuda.synchronize()
    c = orc.pack(lay.W, lay.is8, g)
    P_o, _ = orc.partials(Aq_o, c)
    assert np.array_equal(P.cpu().numpy().astype(np.int64), P_o)
    assert_y_close(Y.cpu().numpy(), orc.gemm(Aq_o, sa_o, c, act_group=g)[1])
    return lay, L, blob, Y


@pytest.mark.parametrize("M", [1, 3, 4])
@pytest.mark.parametrize("g", [64, 128])
def test_gemm_rows_path_grouped(orc, M, g):
    run_grouped(orc, M, 1024, 520, g, path=mx.PATH_ROWS, seed=M + g)


@pytest.mark.parametrize("M,split", [(1, 2), (5, 0), (16, 3), (9, 8)])
@pytest.mark.parametrize("g", [64, 128])
def test_gemm_splitk_path_grouped(orc, M, split, g):
    run_grouped(orc, M, 2048, 300, g, path=mx.PATH_SPLITK, split=split, seed=M + split + g)


@pytest.mark.parametrize("M", [17, 130])
@pytest.mark.parametrize("g", [64, 128])
def test_gemm_tensor_path_grouped(orc, M, g):
    run_grouped(orc, M, 512, 260, g, path=mx.PATH_TENSOR, seed=M + g)


@pytest.mark.parametrize("M,split", [(1, 0), (2, 0), (4, 0), (2, 2), (6, 0), (40, 0)])
@pytest.mark.parametrize("xdtype", [torch.float16, torch.float32])
def test_linear_grouped_matches_two_calls(orc, M, split, xdtype):
    lay = inputs.llama_layer(M, 1024, 300, seed=50 + M + split)
    L, blob = gpu_pack(lay.W, lay.is8, 128)
    Xd = to_dev(lay.X).to(xdtype)
    n = mx.mx_linear_workspace_size(L, M, xdtype, split=split, act_group=128)
    ws = torch.empty(n, dtype=torch.uint8, device=dev()) if n else None
    Y = torch.empty((M, 300), dtype=torch.float16, device=dev())
    P = torch.zeros((M, 300, L.G), dtype=torch.int32, device=dev())
    mx.mx_linear(L, blob, Xd, Y, workspace=ws, split=split, debug_partials=P, act_group=128)
    torch.cuda.synchronize()
    Xo = Xd.float().cpu().numpy()
    Aq_o, sa_o = orc.quant_act(Xo, act_group=128)
    c = orc.pack(lay.W, lay.is8, 128)
    assert np.array_equal(P.cpu().numpy().astype(np.int64), orc.partials(Aq_o, c)[0])
    assert_y_close(Y.cpu().numpy(), orc.gemm(Aq_o, sa_o, c, act_group=128)[1])
    Aq, sa = gpu_quant_grouped(Xo.astype(np.float16) if xdtype == torch.float16 else Xo, 128)
    Y2 = torch.empty_like(Y)
    # the GEMM's own workspace, as mx_linear gives it (a K split of the tensor cores)
    gws = torch.empty(max(16, mx.mx_gemm_workspace_size(L, M, split=split)), dtype=torch.uint8, device=dev())
    mx.mx_gemm(L, blob, Aq, sa, Y2, workspace=gws, split=split, act_group=128)
    torch.cuda.synchronize()
    assert torch.equal(Y, Y2)


def test_act_group_must_be_the_weight_group():
    lay = inputs.llama_layer(2, 512, 256, seed=1)
    L, blob = gpu_pack(lay.W, lay.is8, 128)
    Aq, sa = gpu_quant_grouped(lay.X, 64)
    Y = torch.empty((2, 256), dtype=torch.float16, device=dev())
    with pytest.raises(mx.MXError) as e:
        mx.mx_gemm(L, blob, Aq, sa, Y, act_group=64)
    assert e.value.status == 2
