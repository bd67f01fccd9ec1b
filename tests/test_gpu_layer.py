"""The user-facing layer object against the oracle: eager forward, a blob saved and
reopened from its header, and the graph-captured host-in / host-out runner."""
import numpy as np
import pytest
import torch

from mixed_precision_quantized_mx_b200 import binding as mx
from mixed_precision_quantized_mx_b200 import inputs
from mixed_precision_quantized_mx_b200.layer import MixedPrecisionLinear

from gpu_helpers import assert_y_close, dev

pytestmark = pytest.mark.gpu


def oracle_y(orc, X, W, is8, g):
    Aq, sa = orc.quant_act(X.astype(np.float32))
    return orc.gemm(Aq, sa, orc.pack(W, is8, g))[1]


@pytest.mark.parametrize("M", [1, 3, 40])
def test_forward_and_reopened_blob(orc, M, tmp_path):
    lay = inputs.llama_layer(M, 512, 300, seed=M)
    layer = MixedPrecisionLinear(torch.from_numpy(lay.W).to(dev()), torch.from_numpy(lay.is8).to(dev()))
    layer.check_pack_status()
    X = torch.from_numpy(lay.X).to(dev())
    ref = oracle_y(orc, lay.X, lay.W, lay.is8, 128)
    assert_y_close(layer(X).cpu().numpy(), ref)
    # the blob is position independent: save, reload, reopen from its header
    path = tmp_path / "layer.pt"
    torch.save(layer.blob.cpu(), path)
    again = MixedPrecisionLinear.from_blob(torch.load(path).to(dev()))
    assert (again.N, again.K) == (300, 512)
    assert torch.equal(again(X), layer(X))


@pytest.mark.parametrize("M", [1, 24])
def test_graphed_host_in_host_out(orc, M):
    lay = inputs.llama_layer(M, 1024, 260, seed=7 + M)
    layer = MixedPrecisionLinear(torch.from_numpy(lay.W).to(dev()), torch.from_numpy(lay.is8).to(dev()))
    x_host = torch.empty((M, 1024), dtype=torch.float16).pin_memory()
    runner = layer.graphed(x_host)
    for seed in (1, 2):                      # new input in the same pinned buffer each call
        X = inputs.activations(np.random.default_rng(seed), M, 1024, 10)
        x_host.copy_(torch.from_numpy(X))
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(runner.stream)
        runner.replay()                      # runs on runner.stream, whatever stream is current
        e1.record(runner.stream)
        runner.stream.synchronize()
        assert e0.elapsed_time(e1) > 0.001   # the copies and the kernel ran between the events
        assert_y_close(runner.y_host.numpy(), oracle_y(orc, X, lay.W, lay.is8, 128))


def test_graphed_rejects_pageable_input():
    lay = inputs.llama_layer(1, 256, 130, seed=3)
    layer = MixedPrecisionLinear(torch.from_numpy(lay.W).to(dev()), torch.from_numpy(lay.is8).to(dev()))
    with pytest.raises(ValueError):
        layer.graphed(torch.zeros((1, 256), dtype=torch.float16))


@pytest.mark.parametrize("M", [1, 40])
def test_forward_group_wise_activations(orc, M):
    lay = inputs.llama_layer(M, 1024, 300, seed=60 + M)
    layer = MixedPrecisionLinear(torch.from_numpy(lay.W).to(dev()), torch.from_numpy(lay.is8).to(dev()))
    Y = layer(torch.from_numpy(lay.X).to(dev()), act_group=128)
    Aq, sa = orc.quant_act(lay.X.astype(np.float32), act_group=128)
    ref = orc.gemm(Aq, sa, orc.pack(lay.W, lay.is8, 128), act_group=128)[1]
    assert_y_close(Y.cpu().numpy(), ref)


@pytest.mark.parametrize("M", [2, 40])
def test_sharded_linear_on_one_rank_equals_the_layer(orc, M):
    # output-feature sharding with a single rank: the shard is the whole layer
    from mixed_precision_quantized_mx_b200.tensor_parallel import ShardedLinear
    lay = inputs.llama_layer(M, 512, 300, seed=40 + M)
    sharded = ShardedLinear(torch.from_numpy(lay.W), torch.from_numpy(lay.is8), device=dev())
    assert (sharded.start, sharded.stop, sharded.world) == (0, 300, 1)
    X = torch.from_numpy(lay.X).to(dev())
    Y = sharded(X)
    assert_y_close(Y.cpu().numpy(), oracle_y(orc, lay.X, lay.W, lay.is8, 128))
    whole = MixedPrecisionLinear(torch.from_numpy(lay.W).to(dev()), torch.from_numpy(lay.is8).to(dev()))
    assert torch.equal(Y, whole(X))
