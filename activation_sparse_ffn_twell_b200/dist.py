"""Multi-GPU plumbing for the sparse FFN forward.

Tokens are independent in a feed-forward layer (upppp.jp 2026-05-11, section
「LLMフィードフォワード層の「無駄」とは何か」), so the layer shards over tokens
with the weights replicated and NO data-path collective: each rank runs the
whole hot path on its own token shard.  torch.distributed is used only for
launch plumbing (rank discovery, a barrier, and reducing the per-rank device
time with MAX so a multi-GPU number is the slowest rank's).
"""
from __future__ import annotations

import os
from typing import Tuple


def env_rank_world() -> Tuple[int, int, int]:
    """(rank, local_rank, world_size) from the torchrun environment (1 process if unset)."""
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("LOCAL_RANK", "0")),
            int(os.environ.get("WORLD_SIZE", "1")))


def token_shard(M_total: int, rank: int, world: int) -> Tuple[int, int]:
    """Contiguous [start, stop) token range of `rank` when M_total tokens are split
    over `world` ranks; the first M_total % world ranks take one extra token."""
    if world < 1 or not (0 <= rank < world) or M_total < 0:
        raise ValueError("bad shard request")
    base, extra = divmod(M_total, world)
    start = rank * base + min(rank, extra)
    return start, start + base + (1 if rank < extra else 0)


def init(backend: str = "nccl", timeout_s: float = 120.0):
    """Initialise the default process group when launched with WORLD_SIZE > 1."""
    import datetime
    import torch.distributed as dist
    rank, local, world = env_rank_world()
    if world > 1 and not dist.is_initialized():
        dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=timeout_s))
    return rank, local, world


def max_over_ranks(value: float, device=None) -> float:
    """MAX of a per-rank scalar over all ranks (identity on one process)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64,
                     device=device if device is not None else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(device=None):
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        if device is not None and dist.get_backend() == "nccl":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


def finish():
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized():
        dist.destroy_process_group()
