"""Multi-GPU execution of the block: independent replicas, one process per GPU.

The unit of work is one latent: a block (or a 50-block pass) needs nothing
from another latent, so N GPUs run N latents with no collective on the data
path. torch.distributed is used only for the host-side bookkeeping below: a
barrier around timed regions and the max / sum of per-rank figures. Tensors
for these reductions live on the GPU under NCCL and on the CPU under gloo (the
multi-process tests run the same code on CPU ranks).
"""
from __future__ import annotations

import datetime
import os
from typing import Tuple

import torch

from . import synth


def env_ranks() -> Tuple[int, int, int]:
    """(rank, world size, local rank) from the launcher's environment."""
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def init(backend: str = "nccl", timeout_s: int = 300) -> Tuple[int, int, int]:
    """Join the process group when WORLD_SIZE > 1 (rendezvous from MASTER_ADDR/PORT);
    under NCCL each rank binds the GPU of its local rank."""
    rank, world, local = env_ranks()
    if world > 1:
        import torch.distributed as dist
        kw = {}
        if backend == "nccl":
            torch.cuda.set_device(local)
            kw["device_id"] = torch.device("cuda", local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=timeout_s), **kw)
    elif backend == "nccl":
        torch.cuda.set_device(0)
    return rank, world, local


def _device():
    import torch.distributed as dist
    return torch.device("cuda", torch.cuda.current_device()) if dist.get_backend() == "nccl" else torch.device("cpu")


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def _reduce(v: float, world: int, op_name: str) -> float:
    if world == 1:
        return float(v)
    import torch.distributed as dist
    t = torch.tensor([float(v)], device=_device(), dtype=torch.float64)
    dist.all_reduce(t, op=getattr(dist.ReduceOp, op_name))
    return float(t.item())


def max_over_ranks(v: float, world: int) -> float:
    """The slowest rank's time (every rank receives it)."""
    return _reduce(v, world, "MAX")


def sum_over_ranks(v: float, world: int) -> float:
    return _reduce(v, world, "SUM")


def latent_seed(rank: int) -> int:
    """Each rank's latent is drawn from its own seed (independent replicas)."""
    return synth.BASE_SEED + rank


def throughput(tokens_this_rank: int, ms_this_rank: float, world: int) -> float:
    """Whole-job tokens/s: all ranks' tokens over the slowest rank's time."""
    tokens = sum_over_ranks(tokens_this_rank, world)
    ms = max_over_ranks(ms_this_rank, world)
    return tokens / (ms / 1e3)
