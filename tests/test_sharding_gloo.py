"""Head-sharded 3D-DSA (deformable_slide_attention_b200.sharding) on CPU with the gloo backend.

Each rank holds one token shard of a clip; HeadShardedDSA moves it to head shards with an
all-to-all, runs the per-rank operator and moves the results back.  The operator here is a
stand-in that, like 3D-DSA, works head by head and needs tokens from every shard of a head (its
first and last tokens, a shift along the tokens, a running sum over them), so a result on the
wrong rank, head or token shows up.  Its arithmetic does not depend on how many heads a tensor
holds, so the comparisons are exact.
Every rank compares its token shard with the stand-in applied to the whole, unsharded clip.
"""
import math
import os
import socket

import pytest
import torch
import torch.multiprocessing as mp

from deformable_slide_attention_b200 import ranks, sharding


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _ends(k):
    kf = k.float()
    return kf[:1] + kf[-1:]


def fake_forward(q, k, v, off, dims, window):
    """Per head: out = q * (k[first token] + k[last token]) + v shifted by one token + the sum of
    the token's offsets; lse = sum(q) + the first offset component."""
    H, N = off.shape[0], off.shape[1]
    of = off.float().reshape(H, N, -1)
    out = q.float() * _ends(k) + torch.roll(v.float(), 1, 0)
    out = out + of.sum(-1).T[:, :, None]
    lse = q.float().sum(-1).T + of[..., 0]
    return out.to(q.dtype), lse


def fake_backward(q, k, v, off, lse, dout, dims, window):
    d = dout.float()
    dq = d * 2 + lse.T[:, :, None]
    dk = torch.flip(d, [0]) * _ends(k)
    dv = d.cumsum(0)
    doff = off.float() * lse.reshape(lse.shape + (1,) * (off.dim() - 2))
    return dq.to(q.dtype), dk.to(q.dtype), dv.to(q.dtype), doff


def _problem(dims, heads, dh, window, dtype, per_tap, seed=0):
    g = torch.Generator().manual_seed(seed)
    N, K = math.prod(dims), math.prod(window)
    q, k, v, dout = (torch.randn(N, heads, dh, generator=g).to(dtype) for _ in range(4))
    off = torch.randn((heads, N, K, 3) if per_tap else (heads, N, 3), generator=g)
    return q, k, v, off, dout


CASES = [((3, 5, 7), 5, 8, (3, 3, 3), torch.bfloat16, False),
         ((2, 4, 5), 4, 4, (1, 3, 3), torch.float32, True),
         ((4, 3, 3), 6, 4, (3, 1, 1), torch.float32, False)]


def _worker(rank, world, port, out_q):
    import datetime

    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        for ci, (dims, heads, dh, window, dtype, per_tap) in enumerate(CASES):
            q, k, v, off, dout = _problem(dims, heads, dh, window, dtype, per_tap, seed=ci)
            ref_out, ref_lse = fake_forward(q, k, v, off, dims, window)
            ref = fake_backward(q, k, v, off, ref_lse, dout, dims, window)
            op = sharding.HeadShardedDSA(dims, window, heads, per_tap=per_tap,
                                         forward_fn=fake_forward, backward_fn=fake_backward)
            n0, n1 = sharding.token_range(math.prod(dims), rank, world)
            assert (op.n0, op.n1) == (n0, n1)
            assert (op.h0, op.h1) == ranks.head_range(heads, rank, world)
            shard = lambda t: t[n0:n1]
            oshard = lambda t: t[:, n0:n1]
            out, lse, ctx = op.forward(shard(q), shard(k), shard(v), oshard(off))
            assert ctx[0].shape == (math.prod(dims), op.h1 - op.h0, dh)  # the head shard
            assert torch.equal(out, shard(ref_out)), (rank, ci, "out")
            assert torch.equal(lse, oshard(ref_lse)), (rank, ci, "lse")
            dq, dk, dv, doff = op.backward(ctx, shard(dout))
            for name, got, want in (("dq", dq, shard(ref[0])), ("dk", dk, shard(ref[1])),
                                    ("dv", dv, shard(ref[2])), ("doff", doff, oshard(ref[3]))):
                assert got.dtype == want.dtype and torch.equal(got, want), (rank, ci, name)
        out_q.put((rank, "ok"))
    except BaseException as e:  # report the failure to the parent instead of hanging it
        out_q.put((rank, repr(e)))
        raise
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_head_sharded_resharding_gloo(world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=180) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
    assert res == [(r, "ok") for r in range(world)], res
    assert all(p.exitcode == 0 for p in procs)


def test_single_process_is_the_operator_itself():
    dims, heads, dh, window, dtype, per_tap = CASES[0]
    q, k, v, off, dout = _problem(dims, heads, dh, window, dtype, per_tap)
    op = sharding.HeadShardedDSA(dims, window, heads, forward_fn=fake_forward,
                                 backward_fn=fake_backward)
    out, lse, ctx = op.forward(q, k, v, off)
    ref_out, ref_lse = fake_forward(q, k, v, off, dims, window)
    assert torch.equal(out, ref_out) and torch.equal(lse, ref_lse)
    for got, want in zip(op.backward(ctx, dout), fake_backward(q, k, v, off, ref_lse, dout, dims, window)):
        assert torch.equal(got, want)


def test_rejects_wrong_shards():
    dims, heads, dh, window, dtype, per_tap = CASES[0]
    q, k, v, off, _ = _problem(dims, heads, dh, window, dtype, per_tap)
    op = sharding.HeadShardedDSA(dims, window, heads, forward_fn=fake_forward,
                                 backward_fn=fake_backward)
    with pytest.raises(ValueError):
        op.forward(q[:-1], k, v, off)
    with pytest.raises(ValueError):
        op.forward(q, k, v, off[:, :, None].expand(-1, -1, 27, -1))  # per-tap offsets, per-token op
    with pytest.raises(ValueError):
        sharding.HeadShardedDSA(dims, window, 0, forward_fn=fake_forward, backward_fn=fake_backward)


def test_default_operator_is_the_library():
    """Without stand-ins the per-rank calls are the library's entry points (per token or per tap);
    their signatures are the ones the wrapper calls."""
    import inspect

    from deformable_slide_attention_b200 import abi
    op = sharding.HeadShardedDSA((2, 3, 4), (1, 3, 3), 2)
    assert op.forward_fn is abi.forward and op.backward_fn is abi.backward
    op = sharding.HeadShardedDSA((2, 3, 4), (1, 3, 3), 2, per_tap=True)
    assert op.forward_fn is abi.forward_taps and op.backward_fn is abi.backward_taps
    for fn, names in ((abi.forward, ["q", "k", "v", "offsets", "dims", "window"]),
                      (abi.forward_taps, ["q", "k", "v", "offsets", "dims", "window"]),
                      (abi.backward, ["q", "k", "v", "offsets", "lse", "dout", "dims", "window"]),
                      (abi.backward_taps, ["q", "k", "v", "offsets", "lse", "dout", "dims", "window"])):
        assert list(inspect.signature(fn).parameters)[:len(names)] == names
