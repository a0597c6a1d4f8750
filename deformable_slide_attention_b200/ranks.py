"""Host-side logic of multi-GPU runs (one process per GPU).

3D Deformable Slide Attention (MegaSlide-DiT, arXiv 2607.22696, Eq. 1) is computed independently
per head and per clip, so the operator has no exchange step: a multi-GPU run gives each rank its
own clip (weak scaling), or its own heads of one clip, and the only collectives are the run's
barriers and the max-reduction of the timing.  These helpers hold that logic so it can be tested
with the gloo backend on CPU.
"""
from __future__ import annotations

import dataclasses
import os

CLIP_SEED_STRIDE = 1000  # rank r draws its clip with seed base + 1000 r


@dataclasses.dataclass(frozen=True)
class RankInfo:
    rank: int
    world: int
    local: int


def rank_info(env=None) -> RankInfo:
    """RANK / WORLD_SIZE / LOCAL_RANK as set by torch.distributed.run (defaults: one process)."""
    env = os.environ if env is None else env
    return RankInfo(int(env.get("RANK", "0")), int(env.get("WORLD_SIZE", "1")),
                    int(env.get("LOCAL_RANK", "0")))


def clip_workload(base, rank: int):
    """The workload rank `rank` processes: the same shapes and recipe, its own seeded clip."""
    return dataclasses.replace(base, seed=base.seed + CLIP_SEED_STRIDE * rank)


def head_range(heads: int, rank: int, world: int) -> tuple[int, int]:
    """Contiguous heads [h0, h1) of rank `rank` when one clip's heads are split over `world`
    ranks (sizes differ by at most one, lower ranks first)."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError("rank outside the world")
    base, extra = divmod(heads, world)
    h0 = rank * base + min(rank, extra)
    return h0, h0 + base + (1 if rank < extra else 0)


def max_over_ranks(value: float, device=None) -> float:
    """The largest `value` over all ranks (the whole job ends when its slowest rank does); the
    value itself when no process group is running."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_rate(tokens_per_rank: int, world: int, ms_per_step: float) -> float:
    """Whole-job tokens per second: every rank's tokens over the (max-over-ranks) step time."""
    if ms_per_step <= 0:
        raise ValueError("step time must be positive")
    return tokens_per_rank * world / (ms_per_step / 1000.0)
