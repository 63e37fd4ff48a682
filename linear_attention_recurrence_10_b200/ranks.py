"""Rank plumbing for running the mixer on several GPUs, one process per GPU.

The gated delta rule exchanges nothing between sequences or value heads:
each (sequence, value head) pair carries its own state through the
recurrence (Gated DeltaNet, "Gated Delta Rule" section).  Work is therefore
split across ranks by sequence, with no collective on the data path.  The
only collectives are the barriers around a timed region and the maximum of
the per-rank times.  This module holds that host-side logic and nothing of
the method's arithmetic.
"""
from __future__ import annotations

import heapq
import os
from dataclasses import dataclass

import torch


@dataclass(frozen=True)
class RankEnv:
    rank: int
    world: int
    local: int


def rank_env(environ=None) -> RankEnv:
    """RANK / WORLD_SIZE / LOCAL_RANK as set by torchrun (defaults: one rank)."""
    env = os.environ if environ is None else environ
    world = int(env.get("WORLD_SIZE", "1"))
    rank = int(env.get("RANK", "0"))
    local = int(env.get("LOCAL_RANK", str(rank)))
    if world < 1 or not 0 <= rank < world or local < 0:
        raise ValueError(f"bad rank environment: rank={rank} world={world} local={local}")
    return RankEnv(rank, world, local)


def batch_slice(global_batch: int, rank: int, world: int) -> range:
    """The contiguous block of a batch that ``rank`` owns.  Block sizes differ
    by at most one, the first ``global_batch % world`` ranks taking the larger."""
    if global_batch < 0 or world < 1 or not 0 <= rank < world:
        raise ValueError("bad batch split")
    base, extra = divmod(global_batch, world)
    start = rank * base + min(rank, extra)
    return range(start, start + base + (1 if rank < extra else 0))


def partition_by_tokens(lengths, world: int) -> list[list[int]]:
    """Split variable-length sequences over ``world`` ranks by token count.

    Longest-processing-time-first: sequences in order of decreasing length
    (ties by index) each go to the rank with the fewest tokens so far (ties by
    rank).  The heaviest rank then holds at most the mean load plus one
    sequence.  Each rank's list is returned in increasing sequence order."""
    if world < 1:
        raise ValueError("world must be >= 1")
    order = sorted(range(len(lengths)), key=lambda i: (-int(lengths[i]), i))
    heap = [(0, r) for r in range(world)]
    parts: list[list[int]] = [[] for _ in range(world)]
    for i in order:
        load, r = heapq.heappop(heap)
        parts[r].append(i)
        heapq.heappush(heap, (load + int(lengths[i]), r))
    return [sorted(p) for p in parts]


def max_over_ranks(value: float, world: int, device=None) -> float:
    """Maximum of a per-rank float over the default process group (a no-op on
    one rank).  ``device`` is where the collective's buffer lives: a CUDA
    device under NCCL, the CPU under gloo."""
    if world <= 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def weak_scaling_rate(units_per_rank: float, world: int, ms_max: float) -> float:
    """Whole-job rate when every rank processes ``units_per_rank`` units and the
    slowest rank took ``ms_max`` milliseconds."""
    if ms_max <= 0:
        raise ValueError("time must be positive")
    return units_per_rank * world / (ms_max * 1e-3)


def shard_inputs(inp, seqs):
    """The packed sub-problem holding sequences ``seqs`` (in that order) of a
    packed problem from ``synth.make_inputs``."""
    from . import synth
    cu = inp.cu_seqlens
    spans = [(cu[s], cu[s + 1]) for s in seqs]
    take = lambda t: torch.cat([t[a:b] for a, b in spans]) if spans else t[:0]
    new_cu = [0]
    for a, b in spans:
        new_cu.append(new_cu[-1] + (b - a))
    s0 = None if inp.s0 is None else inp.s0[list(seqs)]
    return synth.Inputs(take(inp.q), take(inp.k), take(inp.v), take(inp.z), take(inp.g),
                        take(inp.beta), s0, inp.w, new_cu, inp.H_k, inp.H_v, inp.d, inp.seed,
                        dict(inp.meta, shard=list(seqs)))
