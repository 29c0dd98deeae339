"""Host-side helpers for running the gated layer as independent replicas, one
process per GPU (torchrun).  The path shards by prompt, so ranks exchange no
data: the only collectives are the timing barrier and the max over ranks of a
rank's device-timed interval."""
from __future__ import annotations

import dataclasses

import torch
import torch.distributed as dist


def rank_workload(w, rank: int):
    """Rank r processes its own prompt batch: same shapes, seed + 1000*r."""
    return dataclasses.replace(w, seed=w.seed + 1000 * rank)


def max_over_ranks(x: float, device=None) -> float:
    """Max of a per-rank float over the default process group (identity when not
    initialised)."""
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(device=None):
    if torch.cuda.is_available() and (device is None or torch.device(device).type == "cuda"):
        torch.cuda.synchronize()
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        dist.barrier()
    if torch.cuda.is_available() and (device is None or torch.device(device).type == "cuda"):
        torch.cuda.synchronize()


def aggregate_throughput(tokens_per_rank: int, steps: int, max_ms: float, world: int) -> float:
    """Whole-job tokens per second: every rank processed `tokens_per_rank` per
    step; the job took the slowest rank's time."""
    return world * tokens_per_rank * steps / (max_ms / 1e3)
