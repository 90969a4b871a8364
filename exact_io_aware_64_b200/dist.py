"""Host-side plumbing for running the benchmark on several GPUs of one node.

The hot path has no exchange step: every (batch, head) is independent, so N GPUs run N
replicas of the workload on disjoint heads (weak scaling) and the only collectives are
for timing: a barrier around the timed region and the max of the per-rank times.  These
helpers take the backend as an argument so the same code runs over NCCL on GPUs and
over gloo on CPU in the tests.
"""
from __future__ import annotations

import datetime
import os
from dataclasses import dataclass

import torch


@dataclass(frozen=True)
class RankInfo:
    rank: int
    world: int
    local_rank: int


def rank_info() -> RankInfo:
    """RANK / WORLD_SIZE / LOCAL_RANK as set by torch.distributed.run (defaults: 1 rank)."""
    return RankInfo(int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
                    int(os.environ.get("LOCAL_RANK", "0")))


def init(info: RankInfo, backend: str, timeout_s: float = 120.0) -> None:
    """Join the process group when there is more than one rank (no-op otherwise)."""
    if info.world <= 1:
        return
    import torch.distributed as dist
    kwargs = {}
    if backend == "nccl":
        torch.cuda.set_device(info.local_rank)
        kwargs["device_id"] = torch.device("cuda", info.local_rank)
    dist.init_process_group(backend, timeout=datetime.timedelta(seconds=timeout_s), **kwargs)


def barrier(info: RankInfo) -> None:
    if info.world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, info: RankInfo, device: str = "cpu") -> float:
    """The largest of the ranks' values (every rank gets it)."""
    if info.world <= 1:
        return float(x)
    import torch.distributed as dist
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate_throughput(work_per_rank: float, seconds_max: float, info: RankInfo) -> float:
    """Whole-job throughput: every rank did `work_per_rank`, the job took the slowest
    rank's time."""
    return info.world * work_per_rank / seconds_max


def replica_seed(base_seed: int, info: RankInfo) -> int:
    """Each replica draws its own heads (disjoint inputs) from a rank-dependent seed."""
    return base_seed + 101 * info.rank


def shutdown(info: RankInfo) -> None:
    if info.world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
