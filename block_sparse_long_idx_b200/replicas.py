"""Host logic of multi-GPU runs: one process per GPU, each on its own independent problem.

The MSA forward path partitions into independent sequences, so N GPUs run N replicas with no
data-path collective (weak scaling). The only collectives are the timing barrier and the max over
ranks of the measured device time.
"""
from __future__ import annotations

import datetime
import os


def rank_info():
    """(rank, world_size, local_rank) from the launcher's environment (torchrun)."""
    return int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("LOCAL_RANK", "0"))


def replica_seed(base_seed: int, rank: int) -> int:
    """Each rank draws an independent sequence."""
    return base_seed + 1000 * rank


def init(backend: str, timeout_s: int = 300):
    import torch.distributed as dist

    if not dist.is_initialized():
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=timeout_s))


def max_over_ranks(values, device=None):
    """Element-wise max of a list of floats over all ranks (identity when not distributed)."""
    import torch
    import torch.distributed as dist

    t = torch.tensor(list(values), dtype=torch.float64, device=device)
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def aggregate_rate(units_per_rank: float, world: int, slowest_seconds: float) -> float:
    """Whole-job throughput: all ranks' units over the slowest rank's time."""
    return units_per_rank * world / slowest_seconds
