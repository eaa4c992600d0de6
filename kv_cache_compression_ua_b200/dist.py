"""Host-side plumbing for running the UA hot path on several GPUs of one node.

The (batch, KV head) units are independent in prefill and decode, so ranks never exchange
data on the hot path (weak scaling: every rank runs its own batch).  The collectives are a
barrier around the timed region, the max of the per-rank times, and, for a data-parallel
backward, the sum of the decay parameters' gradients (the only gradients shared by the
ranks' batches).
"""
from __future__ import annotations

import datetime
import os

import torch


def env_world():
    """(world_size, rank, local_rank) from the torchrun environment (1, 0, 0 if absent)."""
    return (int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")),
            int(os.environ.get("LOCAL_RANK", "0")))


def init(backend: str = "nccl", timeout_s: int = 300):
    """Initialise the process group from the environment when WORLD_SIZE > 1; binds the rank
    to its local GPU for NCCL.  Returns (world, rank, local)."""
    world, rank, local = env_world()
    if world > 1 and not torch.distributed.is_initialized():
        kw = {}
        if backend == "nccl":
            torch.cuda.set_device(local)
            kw["device_id"] = torch.device("cuda", local)
        torch.distributed.init_process_group(backend, timeout=datetime.timedelta(seconds=timeout_s), **kw)
    elif backend == "nccl" and torch.cuda.is_available():
        torch.cuda.set_device(local)
    return world, rank, local


def rank_seed(seed: int, rank: int) -> int:
    """Seed of the batch a rank draws: rank 0 keeps the workload's own seed, so a 1-GPU run
    and rank 0 of an N-GPU run process identical inputs."""
    return seed + 7919 * rank


def barrier(world: int):
    if world > 1:
        torch.distributed.barrier()


def max_over_ranks(x: float, world: int) -> float:
    """Max of a per-rank scalar (device time) over all ranks."""
    if world == 1:
        return float(x)
    backend = torch.distributed.get_backend()
    dev = "cuda" if backend == "nccl" else "cpu"
    t = torch.tensor([float(x)], dtype=torch.float64, device=dev)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def allreduce_decay_param_grads(dalpha: torch.Tensor, dbeta: torch.Tensor, world: int):
    """Data-parallel backward: each rank's ua_prefill_bwd sums dalpha and dbeta [Hkv] over its
    own batch; the model's gradient is their sum over the ranks, taken in place with one
    all-reduce of 2*Hkv floats.  Every other gradient belongs to the rank's own tokens."""
    if world == 1:
        return
    buf = torch.cat([dalpha.reshape(-1), dbeta.reshape(-1)])
    torch.distributed.all_reduce(buf, op=torch.distributed.ReduceOp.SUM)
    n = dalpha.numel()
    dalpha.copy_(buf[:n].view_as(dalpha))
    dbeta.copy_(buf[n:].view_as(dbeta))


def finalize(world: int):
    if world > 1 and torch.distributed.is_initialized():
        torch.distributed.destroy_process_group()
