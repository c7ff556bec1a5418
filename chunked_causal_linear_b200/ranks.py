"""One process per GPU: rank discovery, the per-rank share of independent problems, and
device-side timings reduced as the maximum over ranks.

The prefill has no exchange step between (b, h) pairs, so several GPUs run independent
problems (weak scaling) and the only collectives are the barrier around the timed region
and the max-reduction of the measured times.
"""

from __future__ import annotations

import os
from dataclasses import dataclass
from datetime import timedelta

import torch
import torch.distributed as dist


@dataclass(frozen=True)
class RankInfo:
    rank: int
    world: int
    local_rank: int

    @property
    def is_root(self) -> bool:
        return self.rank == 0


def rank_info() -> RankInfo:
    return RankInfo(int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
                    int(os.environ.get("LOCAL_RANK", "0")))


def init(backend: str = "nccl", timeout_s: float = 120.0) -> RankInfo:
    """Initialises the process group when launched with more than one rank."""
    info = rank_info()
    if info.world > 1 and not dist.is_initialized():
        if backend == "nccl":
            torch.cuda.set_device(info.local_rank)
        dist.init_process_group(backend=backend, timeout=timedelta(seconds=timeout_s))
    return info


def shard(n_units: int, info: RankInfo) -> range:
    """Contiguous share of `n_units` independent units for this rank (sizes differ by at
    most one; every unit is owned by exactly one rank)."""
    base, extra = divmod(n_units, info.world)
    start = info.rank * base + min(info.rank, extra)
    return range(start, start + base + (1 if info.rank < extra else 0))


def barrier(info: RankInfo) -> None:
    if info.world > 1:
        dist.barrier()


def max_over_ranks(x: float, info: RankInfo, device=None) -> float:
    if info.world == 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def any_over_ranks(flag: bool, info: RankInfo, device=None) -> bool:
    return max_over_ranks(1.0 if flag else 0.0, info, device) > 0.5


def finish(info: RankInfo) -> None:
    if info.world > 1 and dist.is_initialized():
        dist.barrier()
        dist.destroy_process_group()
