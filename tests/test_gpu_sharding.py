"""Head-sharded 3D-DSA around the library's CUDA operator, checked against the oracle.

Two processes share the one GPU of the test machine.  Each holds one token shard of a clip
(sequence-parallel layout); HeadShardedDSA moves the shards to head shards with gloo all-to-alls
on host-staged tensors, each rank runs dsa3d_forward / dsa3d_backward (per token) or the per-tap
entry points on cuda:0 for its heads, and the results come back to the token shards.  Every rank
compares its shards element by element with the oracle on the whole clip.  The ranks' kernels
never wait on one another: the only exchanges are gloo's, on the host.
"""
import math
import os
import socket

import pytest
import torch
import torch.multiprocessing as mp

pytestmark = [pytest.mark.gpu, pytest.mark.usefixtures("gpu_lib", "oracle_lib")]

CASES = [((4, 12, 20), 5, 64, (3, 5, 5), False),   # 5 heads over 2 ranks: 3 + 2
         ((3, 6, 7), 3, 64, (3, 3, 3), True)]      # per-tap offsets


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out_q):
    import datetime

    import numpy as np
    import torch.distributed as dist

    import oracle
    from deformable_slide_attention_b200 import abi, inputs, sharding

    def on_gpu(fn):
        def run(*args):
            dims, window = args[-2], args[-1]
            res = fn(*(a.cuda() for a in args[:-2]), dims, window)
            torch.cuda.synchronize()
            return tuple(r.cpu() for r in res)
        return run

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=120))
    try:
        for ci, (dims, heads, dh, window, per_tap) in enumerate(CASES):
            _, inp = inputs.custom(*dims, heads, dh, window, "bf16", seed=300 + ci, scale=2.0,
                                   per_tap=per_tap)
            fwd, bwd = (abi.forward_taps, abi.backward_taps) if per_tap else (abi.forward, abi.backward)
            op = sharding.HeadShardedDSA(dims, window, heads, per_tap=per_tap,
                                         forward_fn=on_gpu(fwd), backward_fn=on_gpu(bwd))
            n0, n1 = op.n0, op.n1
            tok = lambda t: t[n0:n1].contiguous()
            hm = lambda t: t[:, n0:n1].contiguous()
            out, lse, ctx = op.forward(tok(inp["q"]), tok(inp["k"]), tok(inp["v"]), hm(inp["offsets"]))
            dq, dk, dv, doff = op.backward(ctx, tok(inp["dout"]))
            r_out, r_lse = oracle.full_forward(inp["q"], inp["k"], inp["v"], inp["offsets"], dims,
                                               window, per_tap=per_tap)
            r_dq, r_doff, r_dk, r_dv = oracle.full_backward(inp["q"], inp["k"], inp["v"],
                                                            inp["offsets"], inp["dout"], dims,
                                                            window, per_tap=per_tap)
            for name, got, ref in (("out", out, r_out[n0:n1]), ("lse", lse, r_lse[:, n0:n1]),
                                   ("dq", dq, r_dq[n0:n1]), ("dk", dk, r_dk[n0:n1]),
                                   ("dv", dv, r_dv[n0:n1]), ("doffsets", doff, r_doff[:, n0:n1])):
                g = got.double().numpy()
                fin = np.isfinite(ref)
                assert got.shape == ref.shape, (rank, ci, name, tuple(got.shape), ref.shape)
                assert np.array_equal(np.isfinite(g), fin), (rank, ci, name, "finiteness")
                err = np.abs(g[fin] - ref[fin]).max(initial=0.0)
                assert err <= 2e-2, (rank, ci, name, err)
        out_q.put((rank, "ok"))
    except BaseException as e:  # report the failure to the parent instead of hanging it
        out_q.put((rank, repr(e)))
        raise
    finally:
        dist.destroy_process_group()


def test_head_sharded_library_operator_two_ranks():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=600) for _ in range(world))
    for p in procs:
        p.join(timeout=120)
    assert res == [(r, "ok") for r in range(world)], res
    assert all(p.exitcode == 0 for p in procs)
