"""World-size-2 checks of the multi-GPU host plumbing on CPU (gloo): ranks draw distinct
batches, rank 0 draws the 1-GPU inputs, and the timing reduction takes the max over ranks."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, out):
    os.environ.update({"MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port), "WORLD_SIZE": str(world),
                       "RANK": str(rank), "LOCAL_RANK": str(rank)})
    from kv_cache_compression_ua_b200 import dist
    from kv_cache_compression_ua_b200 import inputs as I
    w_, r_, _ = dist.init("gloo", timeout_s=60)
    assert (w_, r_) == (world, rank)
    w = I.WORKLOADS["prefill_1b"].resized(B=1, T=16)
    wr = w.resized(seed=dist.rank_seed(w.seed, rank))
    k = I.make_prefill_inputs(wr, names=["k"])["k"]
    dist.barrier(world)
    m = dist.max_over_ranks(10.0 + rank, world)
    out[rank] = (float(k.sum()), m)
    dist.finalize(world)


def test_two_rank_gloo_plumbing():
    world = 2
    port = _free_port()
    with mp.Manager() as mgr:
        out = mgr.dict()
        mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    assert res[0][1] == res[1][1] == 11.0          # max over ranks
    assert res[0][0] != res[1][0]                  # distinct batches per rank
    from kv_cache_compression_ua_b200 import inputs as I
    w = I.WORKLOADS["prefill_1b"].resized(B=1, T=16)
    k0 = I.make_prefill_inputs(w, names=["k"])["k"]
    assert abs(float(k0.sum()) - res[0][0]) < 1e-6  # rank 0 = the 1-GPU inputs
