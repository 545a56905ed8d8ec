"""Host logic of multi-GPU runs: one process per GPU, each decoding its own
batch (sequences are independent, so the decode path shards by batch with no
data-path collective).

* ``rank_workload`` gives every rank its own seeded batch of the workload.
* ``slowest`` reduces per-rank device timings to the maximum over ranks (the
  job takes as long as its slowest rank).
* ``aggregate_rate`` turns that into the whole-job rate: the units all ranks
  processed divided by the slowest rank's time (weak scaling).

Only timings cross ranks; with the NCCL backend the tensors live on the
rank's GPU, with gloo (CPU tests) on the host.
"""
from __future__ import annotations

from typing import Sequence

import torch
import torch.distributed as dist

from . import synth


def rank_workload(w: synth.Workload, rank: int, world: int) -> synth.Workload:
    """The workload of one rank: same shapes, seed offset by the rank so every
    rank decodes different sequences."""
    if world <= 1:
        return w
    return synth.scaled(w, seed=w.seed + 1000 * rank)


def slowest(values: Sequence[float], device=None) -> list:
    """Element-wise maximum over ranks of per-rank timings (no-op on one rank)."""
    vals = [float(v) for v in values]
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return vals
    t = torch.tensor(vals, dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t.cpu()]


def aggregate_rate(units_per_rank: float, world: int, slowest_ms: float) -> float:
    """Whole-job units per second: every rank processes units_per_rank in the
    timed region, which lasts slowest_ms (per step)."""
    return world * units_per_rank / (slowest_ms / 1e3)
