"""Multi-process host logic (one process per GPU in a real run) on CPU with the gloo backend:
per-rank clips and head ranges, the max-over-ranks step time and the whole-job rate, and the
rank gate of the reference arm.  No GPU is involved."""
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

from deformable_slide_attention_b200 import inputs, ranks

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, values, out_q):
    import datetime

    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        info = ranks.rank_info()
        ms = ranks.max_over_ranks(values[rank])
        dist.barrier()
        out_q.put((rank, info.rank, info.world, ms, ranks.job_rate(1000, world, ms),
                   ranks.clip_workload(inputs.BY_NAME["small-bf16"], rank).seed))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_max_over_ranks_and_job_rate_gloo(world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    values = [10.0 + 7.5 * ((r * 5) % world) for r in range(world)]  # the slowest rank is not rank 0
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, values, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    slowest = max(values)
    seeds = set()
    for rank, info_rank, info_world, ms, rate, seed in res:
        assert (info_rank, info_world) == (rank, world)
        assert ms == slowest                                  # every rank reports the max
        assert rate == pytest.approx(1000 * world / (slowest / 1000.0))
        seeds.add(seed)
    assert len(seeds) == world                                # each rank draws its own clip


def test_single_process_needs_no_group():
    assert ranks.max_over_ranks(3.25) == 3.25
    assert ranks.rank_info({}) == ranks.RankInfo(0, 1, 0)
    assert ranks.job_rate(2_088_960, 1, 1000.0) == 2_088_960
    with pytest.raises(ValueError):
        ranks.job_rate(1, 1, 0.0)


@pytest.mark.parametrize("heads,world", [(32, 1), (32, 2), (32, 8), (30, 4), (5, 8)])
def test_head_ranges_partition_the_heads(heads, world):
    spans = [ranks.head_range(heads, r, world) for r in range(world)]
    assert spans[0][0] == 0 and spans[-1][1] == heads
    for (a0, a1), (b0, b1) in zip(spans, spans[1:]):
        assert a1 == b0
    sizes = [b - a for a, b in spans]
    assert max(sizes) - min(sizes) <= 1
    with pytest.raises(ValueError):
        ranks.head_range(heads, world, world)


def test_reference_arm_runs_on_rank_zero_only():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--gpus", "2", "--steps", "1", "--warmup", "0"],
                       env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0
    assert r.stdout.strip() == ""  # no JSON line from a non-zero rank
