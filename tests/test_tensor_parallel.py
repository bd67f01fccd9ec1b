"""Output-feature sharding (tensor parallelism along N), exercised with two gloo ranks
on CPU: the row partition and the all-gather of Y.  Each rank stands its GPU call in
with the oracle on its own rows (packed with the slice of the layer's 8-bit mask,
under a permutation local to the rank); the gathered Y must equal the oracle's Y of
the whole layer exactly, since every column comes from the same row, codes and
scales (MixLLM section 3.1.1, Figure 1: output features are independent).
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


@pytest.mark.parametrize("N,world", [(0, 1), (1, 1), (130, 2), (131, 2), (7, 3), (28672, 8), (5, 8)])
def test_shard_range_covers_rows_once_balanced(N, world):
    import sys
    sys.path.insert(0, ROOT)
    from mixed_precision_quantized_mx_b200.tensor_parallel import shard_range
    ranges = [shard_range(N, world, r) for r in range(world)]
    assert ranges[0][0] == 0 and ranges[-1][1] == N
    for (a0, b0), (a1, b1) in zip(ranges, ranges[1:]):
        assert b0 == a1                                   # contiguous, disjoint
    sizes = [b - a for a, b in ranges]
    assert max(sizes) - min(sizes) <= 1                   # balanced
    assert sorted(sizes, reverse=True) == sizes           # the larger shards first


def test_shard_range_rejects_bad_arguments():
    import sys
    sys.path.insert(0, ROOT)
    from mixed_precision_quantized_mx_b200.tensor_parallel import shard_range
    for args in ((10, 0, 0), (10, 2, 2), (10, 2, -1), (-1, 2, 0)):
        with pytest.raises(ValueError):
            shard_range(*args)


def _worker(rank, world, port, N, out):
    import sys
    sys.path.insert(0, ROOT)
    import datetime
    import oracle
    from mixed_precision_quantized_mx_b200 import inputs
    from mixed_precision_quantized_mx_b200.tensor_parallel import gather_columns, shard_range
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        lay = inputs.llama_layer(5, 256, N, seed=11)      # the same layer and tokens on every rank
        a, b = shard_range(N, world, rank)
        Aq, sa = oracle.quant_act(lay.X.astype(np.float32))
        c = oracle.pack(lay.W[a:b], lay.is8[a:b], lay.group)
        y_local = torch.from_numpy(oracle.gemm(Aq, sa, c)[1])
        y = gather_columns(y_local, N, world)
        if rank == 0:
            full = oracle.gemm(Aq, sa, oracle.pack(lay.W, lay.is8, lay.group))[1]
            out["equal"] = bool(np.array_equal(y.numpy(), full))
            out["shape"] = tuple(y.shape)
            out["n8"] = (int(lay.is8[:shard_range(N, world, 0)[1]].sum()), int(lay.is8.sum()))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("N", [130, 131])
def test_two_gloo_ranks_shard_and_gather_equal_the_whole_layer(N):
    port = _free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_worker, args=(2, port, N, out), nprocs=2, join=True)
        res = dict(out)
    assert res["shape"] == (5, N)
    assert res["equal"]
    assert 0 < res["n8"][0] < res["n8"][1]               # both shards hold 8-bit rows


def test_gather_is_identity_on_one_rank():
    import sys
    sys.path.insert(0, ROOT)
    from mixed_precision_quantized_mx_b200.tensor_parallel import gather_columns
    y = torch.arange(12.0).reshape(3, 4)
    assert gather_columns(y, 4, 1) is y
