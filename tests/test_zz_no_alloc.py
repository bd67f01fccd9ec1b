"""mx_linear_noalloc (scratch in a fixed device array) against mx_linear (scratch
in a caller workspace).  Collected last so that it also runs after every other
GPU test in the same process."""
import numpy as np
import pytest
import torch

from mixed_precision_quantized_mx_b200 import binding as mx
from mixed_precision_quantized_mx_b200 import inputs

from gpu_helpers import dev, gpu_pack, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    from mixed_precision_quantized_mx_b200 import build
    build.build()
    assert torch.cuda.is_available()
    mx.lib()


def with_workspace(L, blob, Xd):
    # a caller workspace of the fixed array's size: mx_linear then takes the same
    # decisions (a K split of the tensor cores only when its sums fit) as the array
    Y = torch.empty((Xd.shape[0], L.N), dtype=torch.float16, device=dev())
    n = mx.mx_linear_workspace_size(L, Xd.shape[0], Xd.dtype)
    ws = torch.empty(mx.NOALLOC_SCRATCH_BYTES, dtype=torch.uint8, device=dev()) if n else None
    mx.mx_linear(L, blob, Xd, Y, workspace=ws)
    return Y


def nan_out(L, M):
    return torch.full((M, L.N), float("nan"), dtype=torch.float16, device=dev())


def test_two_calls_in_a_row_match_mx_linear():
    lay = inputs.llama_layer(16, 4096, 1024, seed=101)
    L, blob = gpu_pack(lay.W, lay.is8, 128)
    rng = np.random.default_rng(102)
    Xa = to_dev(lay.X)                                         # 16 tokens: split-K path
    Xb = to_dev(inputs.activations(rng, 300, 4096, 41))        # 300 tokens: tensor cores
    assert mx.mx_linear_workspace_size(L, 16) > 0 and mx.mx_linear_workspace_size(L, 300) > 0
    Ya, Yb = nan_out(L, 16), nan_out(L, 300)
    mx.mx_linear_noalloc(L, blob, Xa, Ya)                      # both in one stream, no sync
    mx.mx_linear_noalloc(L, blob, Xb, Yb)
    torch.cuda.synchronize()
    assert torch.equal(Ya, with_workspace(L, blob, Xa))
    assert torch.equal(Yb, with_workspace(L, blob, Xb))
    # and again in the other order, with fp32 input
    Xa32 = Xa.float()
    mx.mx_linear_noalloc(L, blob, Xb, Yb)
    mx.mx_linear_noalloc(L, blob, Xa32, Ya)
    torch.cuda.synchronize()
    assert torch.equal(Yb, with_workspace(L, blob, Xb))
    assert torch.equal(Ya, with_workspace(L, blob, Xa32))


def test_fused_sizes_need_no_scratch():
    lay = inputs.llama_layer(3, 2048, 520, seed=103)
    L, blob = gpu_pack(lay.W, lay.is8, 128)
    Xd = to_dev(lay.X)
    assert mx.mx_linear_workspace_size(L, 3) == 0
    Y = nan_out(L, 3)
    mx.mx_linear_noalloc(L, blob, Xd, Y)
    torch.cuda.synchronize()
    assert torch.equal(Y, with_workspace(L, blob, Xd))


def test_largest_fit_and_first_refusal():
    K = 4096
    lay = inputs.llama_layer(1, K, 256, seed=104)
    L, blob = gpu_pack(lay.W, lay.is8, 128)
    cap = mx.NOALLOC_SCRATCH_BYTES
    # the limit is on Aq and s_a (the unsplit scratch)
    M_fit = max(m for m in range(cap // K - 2, cap // K + 1) if mx.mx_linear_workspace_size(L, m, split=1) <= cap)
    rng = np.random.default_rng(105)
    Xd = to_dev(inputs.activations(rng, M_fit + 1, K, 41))
    Y = nan_out(L, M_fit)
    mx.mx_linear_noalloc(L, blob, Xd[:M_fit], Y)
    torch.cuda.synchronize()
    assert torch.equal(Y, with_workspace(L, blob, Xd[:M_fit]))
    Y2 = nan_out(L, M_fit + 1)
    with pytest.raises(mx.MXError) as e:
        mx.mx_linear_noalloc(L, blob, Xd, Y2)
    assert e.value.status == 7
    torch.cuda.synchronize()
    assert torch.isnan(Y2).all()                               # nothing was launched


def test_group_wise_activation_scales():
    # act_group = g: s_a takes 2 M (K / g) bytes of the array, two calls in a row
    lay = inputs.llama_layer(40, 2048, 768, seed=106)
    L, blob = gpu_pack(lay.W, lay.is8, 128)
    Xd = to_dev(lay.X)
    n = mx.mx_linear_workspace_size(L, 40, act_group=128)
    assert n >= 40 * 2048 + 2 * 40 * (2048 // 128)
    ref = torch.empty((40, L.N), dtype=torch.float16, device=dev())
    ws = torch.empty(mx.NOALLOC_SCRATCH_BYTES, dtype=torch.uint8, device=dev())
    mx.mx_linear(L, blob, Xd, ref, workspace=ws, act_group=128)
    for _ in range(2):
        Y = nan_out(L, 40)
        mx.mx_linear_noalloc(L, blob, Xd, Y, act_group=128)
        torch.cuda.synchronize()
        assert torch.equal(Y, ref)
