"""Failure detection without a GPU fault.

The tensor-core kernel bounds every wait.  With the test hook `test_stall` its
loader issues no copies, so the consumers' waits run out after a short limit;
the kernel must record MX_ERR_TIMEOUT in the status word, release TMEM and
return, leaving the context usable for the next call.
"""
import numpy as np
import pytest
import torch

from mixed_precision_quantized_mx_b200 import binding as mx
from mixed_precision_quantized_mx_b200 import inputs

from gpu_helpers import assert_y_close, dev, gpu_gemm, gpu_pack, gpu_quant

pytestmark = pytest.mark.gpu


def test_tc_wait_timeout_sets_status_and_context_survives(orc):
    rng = np.random.default_rng(3)
    M, N, K = 160, 256, 512
    X = inputs.activations(rng, M, K, 4)
    W = inputs.weights(rng, N, K)
    is8 = inputs.saliency_mask(np.abs(rng.standard_normal(N)), 26)
    Aq, sa = gpu_quant(X)
    L, blob = gpu_pack(W, is8, 128)
    Y = torch.zeros((M, N), dtype=torch.float16, device=dev())
    status = torch.zeros(1, dtype=torch.int32, device=dev())
    with pytest.raises(mx.MXError):            # the hook needs a status word
        mx.mx_gemm(L, blob, Aq, sa, Y, path=mx.PATH_TENSOR, test_stall=1)
    mx.mx_gemm(L, blob, Aq, sa, Y, path=mx.PATH_TENSOR, status=status,
               wait_timeout_us=20000, test_stall=1)
    torch.cuda.synchronize()
    assert int(status.item()) == 5             # MX_ERR_TIMEOUT
    # the same context still runs the real thing correctly
    status.zero_()
    Y2, _, _ = gpu_gemm(L, blob, Aq, sa, path=mx.PATH_TENSOR)
    Aq_o, sa_o = orc.quant_act(X.astype(np.float32))
    c = orc.pack(W, is8, 128)
    assert_y_close(Y2.cpu().numpy(), orc.gemm(Aq_o, sa_o, c)[1])
    mx.mx_gemm(L, blob, Aq, sa, Y, path=mx.PATH_TENSOR, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
