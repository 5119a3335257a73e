"""Host-side plumbing for running the decode path on several GPUs of one node.

The sparse decode path shards with no exchange step: every (sequence, KV
head, layer) is independent, so each rank owns its own batch (data-parallel,
weak scaling) and the only collectives are a barrier around the timed region
and a max-reduction of the elapsed time -- neither is on the data path.
"""
from __future__ import annotations

import datetime
import os
from dataclasses import dataclass

import torch


@dataclass
class RankInfo:
    world: int
    rank: int
    local_rank: int


def rank_info() -> RankInfo:
    """World size, rank and local rank from the torchrun environment."""
    return RankInfo(int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")),
                    int(os.environ.get("LOCAL_RANK", "0")))


def init(info: RankInfo, backend: str = "nccl", timeout_s: float = 120.0):
    """Join the process group (no-op for one rank).  A short timeout makes
    ranks that wait on a missing peer end with an error instead of hanging."""
    if info.world <= 1:
        return
    import torch.distributed as dist
    kwargs = {}
    if backend == "nccl":
        torch.cuda.set_device(info.local_rank)
        kwargs["device_id"] = torch.device("cuda", info.local_rank)
    dist.init_process_group(backend, timeout=datetime.timedelta(seconds=timeout_s), **kwargs)


def barrier(info: RankInfo):
    if info.world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, info: RankInfo, device="cpu") -> float:
    """The largest value of ``x`` over all ranks (every rank gets it)."""
    if info.world <= 1:
        return float(x)
    import torch.distributed as dist
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate_rate(units_per_rank: float, info: RankInfo, max_seconds: float) -> float:
    """Whole-job throughput: the units all ranks processed over the slowest
    rank's time."""
    return info.world * units_per_rank / max_seconds


def rank_seed(base: int, info: RankInfo) -> int:
    """Distinct input seed per rank (each rank owns different sequences)."""
    return base + 1000 * (info.rank + 1)


def shutdown(info: RankInfo):
    if info.world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
