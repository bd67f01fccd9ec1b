"""Host-side logic of multi-GPU runs, exercised with two gloo ranks on CPU.

The layer shards by independent batches (weak scaling): every rank packs and runs
its own layer and tokens, and the only cross-rank traffic is the barrier and the
max-over-ranks reduction of the timed region.  Nothing here needs a GPU.
"""
import os
import socket

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out):
    import sys
    sys.path.insert(0, ROOT)
    import datetime
    import bench
    from mixed_precision_quantized_mx_b200 import inputs
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        t = bench.max_over_ranks(1.5 + rank)            # rank 1 is the slow one
        seed = bench.rank_seed(7, rank)
        lay = inputs.llama_layer(2, 256, 130, seed=seed)
        dist.barrier()
        out[rank] = (t, seed, float(lay.X[0, 0]), int(lay.is8.sum()))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_max_timing_and_distinct_batches():
    port = _free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_worker, args=(2, port, out), nprocs=2, join=True)
        res = dict(out)
    assert res[0][0] == res[1][0] == 2.5                 # both ranks report the slowest
    assert res[0][1] != res[1][1]                        # each rank its own seed
    assert res[0][2] != res[1][2]                        # ... and its own activations
    assert res[0][3] == res[1][3] == 13                  # same layer shape and 8-bit fraction


def test_single_process_max_is_identity():
    import sys
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.25) == 3.25
