"""Multi-process plumbing for running independent decode batches on several
GPUs (one process per GPU, launched by torchrun).

The decode path shards with no exchange: each rank owns its own pool, tables
and batch, so no collective touches the data.  The process group is used
only to line ranks up around a timed region and to take the slowest rank's
time (max over ranks), which is what a whole-job throughput must divide by.
"""
from __future__ import annotations

import datetime
import os
from dataclasses import dataclass
from typing import List, Sequence

import torch


@dataclass
class Ranks:
    world: int
    rank: int
    local: int


def env_ranks() -> Ranks:
    return Ranks(int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")),
                 int(os.environ.get("LOCAL_RANK", "0")))


def init(backend: str, timeout_s: float = 120.0) -> Ranks:
    """Join the process group when WORLD_SIZE > 1 (rendezvous on 127.0.0.1
    unless MASTER_ADDR is set).  A short timeout turns a missing rank into an
    error instead of a wait."""
    r = env_ranks()
    if r.world > 1:
        import torch.distributed as dist
        os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
        if backend == "nccl":
            torch.cuda.set_device(r.local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=timeout_s))
    return r


def barrier(r: Ranks) -> None:
    if r.world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(r: Ranks, values: Sequence[float], device=None) -> List[float]:
    """Element-wise max of per-rank values (times), identical on every rank."""
    t = torch.tensor(list(values), dtype=torch.float64, device=device)
    if r.world > 1:
        import torch.distributed as dist
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def batch_seed(base: int, r: Ranks) -> int:
    """Each rank decodes its own independent batch."""
    return base + r.rank


def finish(r: Ranks) -> None:
    if r.world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
