"""Multi-GPU plumbing: one process per GPU, each running its own replica of
the workload (independent batches; the attention of one batch needs nothing
from another), so no collective sits on the data path. The only
communication is control plane: a barrier around the timed region and the
max over ranks of the measured times."""
from __future__ import annotations

import datetime
import os
from typing import Sequence


def env_rank() -> tuple:
    """(rank, world_size, local_rank) from the torchrun environment."""
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def init(backend: str = "nccl", timeout_s: float = 120.0) -> None:
    """Initialise the default process group from the environment (no-op for
    a single process). MASTER_ADDR should be 127.0.0.1 on one node."""
    import torch.distributed as dist

    _, world, _ = env_rank()
    if world > 1 and not dist.is_initialized():
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=timeout_s))


def barrier() -> None:
    import torch
    import torch.distributed as dist

    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        if dist.get_backend() == "nccl":
            dist.barrier(device_ids=[torch.cuda.current_device()])  # the rank's own GPU, set by the caller
        else:
            dist.barrier()


def max_over_ranks(values: Sequence[float], device=None) -> list:
    """Element-wise max of per-rank values (times), identical on every rank."""
    import torch
    import torch.distributed as dist

    vals = [float(v) for v in values]
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return vals
    t = torch.tensor(vals, dtype=torch.float64, device=device if device is not None else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def replica_seed(base_seed: int, rank: int) -> int:
    """Seed of rank `rank`'s synthetic batch (distinct per replica)."""
    return int(base_seed) * 1000003 + int(rank)


def shutdown() -> None:
    import torch.distributed as dist

    if dist.is_available() and dist.is_initialized():
        barrier()
        dist.destroy_process_group()
