"""World-size-2 checks of the multi-GPU host plumbing on CPU (gloo): ranks draw distinct
batches, rank 0 draws the 1-GPU inputs, the timing reduction takes the max over ranks, and
the data-parallel reduction of the decay parameters' gradients gives the gradient of the
whole batch (checked with the fp64 oracle's backward)."""
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


def _bwd_worker(rank, world, port, out):
    os.environ.update({"MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port), "WORLD_SIZE": str(world),
                       "RANK": str(rank), "LOCAL_RANK": str(rank)})
    import oracle
    from kv_cache_compression_ua_b200 import dist
    from kv_cache_compression_ua_b200 import inputs as I
    dist.init("gloo", timeout_s=60)
    x = _rank_batch(rank)
    g = oracle.prefill_bwd(**x, nthreads=1)
    da = torch.from_numpy(g["dalpha"].copy())
    db = torch.from_numpy(g["dbeta"].copy())
    dist.allreduce_decay_param_grads(da, db, world)
    out[rank] = (da.numpy().tolist(), db.numpy().tolist(), g["da_q"].tolist())
    dist.finalize(world)


def _rank_batch(rank):
    """Rank `rank`'s batch of a small problem: its own tokens, the model's shared alpha, beta."""
    from kv_cache_compression_ua_b200 import dist
    from kv_cache_compression_ua_b200 import inputs as I
    w = I.Workload("dp", 1, 10, 4, 2, 8, "f32", 77, with_grad=True)
    x = {k: v.astype(np.float64) for k, v in I.make_prefill_inputs(w.resized(seed=dist.rank_seed(w.seed, rank))).items()}
    shared = I.make_prefill_inputs(w, names=["alpha", "beta"])
    x["alpha"], x["beta"] = shared["alpha"].astype(np.float64), shared["beta"].astype(np.float64)
    return x


def test_two_rank_data_parallel_decay_grads():
    world = 2
    port = _free_port()
    with mp.Manager() as mgr:
        out = mgr.dict()
        mp.spawn(_bwd_worker, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    import oracle
    xs = [_rank_batch(r) for r in range(world)]
    whole = {k: (np.concatenate([x[k] for x in xs]) if k not in ("alpha", "beta") else xs[0][k]) for k in xs[0]}
    g = oracle.prefill_bwd(**whole, nthreads=1)
    for r in range(world):
        np.testing.assert_allclose(res[r][0], g["dalpha"], rtol=1e-12, atol=1e-14)
        np.testing.assert_allclose(res[r][1], g["dbeta"], rtol=1e-12, atol=1e-14)
        np.testing.assert_allclose(res[r][2], g["da_q"][r:r + 1], rtol=1e-12, atol=1e-14)  # per-token: not reduced
