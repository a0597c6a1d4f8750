"""Time the oracle on the workloads: the CPU baseline of the performance table.

TEST INFRASTRUCTURE ONLY (like the rest of this package): it measures the plain fp64 C oracle as
it stands, on seeded synthetic inputs from ``deformable_slide_attention_b200.inputs``.

    python -m oracle.time_oracle [--budget SECONDS] [--json OUT]

Per workload and thread count (all host threads, then one) it times the three parts of a step:
the forward, the query side of the backward (dq, doffsets) and the key side (dK, dV).  The tiny
workload runs in full, and so does the small one on all threads; the rest run on a seeded sample
of head 0 -- query items drawn at random, key items a block of whole frames -- and the full step
is extrapolated from the measured rates (the work per item is the same throughout a workload).

The oracle's key side runs one thread per head and, for the keys asked of a head, redoes the
query-side work of every query whose taps touch them: a sampled block of F_s frames costs the
queries of about F_s + k_t frames.  So a sampled key-side rate is a lower bound, and the
extrapolation to all heads multiplies it by min(threads, heads), the heads the oracle runs at
once.
"""
from __future__ import annotations

import argparse
import json
import os
import time

import numpy as np

import oracle
from deformable_slide_attention_b200 import inputs

FULL = ("tiny-f32", "small-bf16")
SAMPLED = ("720p-bf16", "720p-train-bf16", "1080p-long-bf16")


def _heads(w, inp, heads):
    """The named heads' inputs as CPU tensors ([N][h][dh], [h][N][3])."""
    import torch
    idx = torch.tensor(heads)
    pick = lambda t: t.index_select(1, idx.to(t.device)).contiguous().cpu()
    out = {k: pick(inp[k]) for k in ("q", "k", "v") if k in inp}
    if inp.get("dout") is not None:
        out["dout"] = pick(inp["dout"])
    out["offsets"] = inp["offsets"].index_select(0, idx.to(inp["offsets"].device)).contiguous().cpu()
    return out


def _rate(fn, items):
    t0 = time.perf_counter()
    fn()
    dt = time.perf_counter() - t0
    return items / dt, dt


def time_workload(name, threads, budget):
    full = name == "tiny-f32" or (name in FULL and threads > 1)
    import torch
    w = inputs.BY_NAME[name]
    train = name.endswith("train-bf16") or name in FULL or name.startswith("1080p")
    dev = "cuda" if (w.device_generated and torch.cuda.is_available()) else "cpu"
    if w.device_generated and dev == "cpu":
        import dataclasses
        w = dataclasses.replace(w, device_generated=False)
    inp = inputs.make(w, dev, with_dout=train)
    heads = list(range(w.heads)) if full else [0]
    d = _heads(w, inp, heads)
    del inp
    H, N = len(heads), w.N
    res = {"workload": name, "threads": threads, "heads_timed": H, "tokens": N, "heads": w.heads}
    rng = np.random.default_rng(4321)
    if full:
        q_items = None
        nq = N * H
    else:
        # about a quarter of the budget per part, calibrated on a small first sample
        probe = np.sort(rng.choice(N, size=min(N, 8 * threads), replace=False)).astype(np.int64)
        r, _ = _rate(lambda: oracle.forward(d["q"], d["k"], d["v"], d["offsets"], w.dims, w.window, probe,
                                            threads), len(probe))
        nq = int(min(N, max(threads, r * budget / 4)))
        q_items = np.sort(rng.choice(N, size=nq, replace=False)).astype(np.int64)
    fr, ft = _rate(lambda: oracle.forward(d["q"], d["k"], d["v"], d["offsets"], w.dims, w.window, q_items,
                                          threads), nq)
    res["forward_items_per_s"] = fr
    res["forward_s"] = ft
    if train:
        qr, qt = _rate(lambda: oracle.backward(d["q"], d["k"], d["v"], d["offsets"], d["dout"], w.dims,
                                               w.window, q_items, [], threads), nq)
        res["bwd_query_items_per_s"] = qr
        res["bwd_query_s"] = qt
        F, Hp, Wp = w.dims
        if full:
            k_items = None
            nk = N * H
        else:
            # a block of whole frames of head 0, sized from the query-side rate
            frames = int(max(1, min(F, (qr * budget / 2) // (Hp * Wp))))
            k_items = np.arange(frames * Hp * Wp, dtype=np.int64)
            nk = len(k_items)
        kr, kt_ = _rate(lambda: oracle.backward(d["q"], d["k"], d["v"], d["offsets"], d["dout"], w.dims,
                                                w.window, [], k_items, threads), nk)
        res["bwd_key_items_per_s"] = kr
        res["bwd_key_s"] = kt_
        if not full:
            res["bwd_key_frames_sampled"] = nk // (Hp * Wp)
            kr = kr * min(threads, w.heads)  # one thread per head: the heads run side by side
        res["bwd_key_items_per_s_all_heads"] = kr
    total_items = N * w.heads
    step = total_items / res["forward_items_per_s"]
    if train:
        step += total_items / res["bwd_query_items_per_s"] + total_items / res["bwd_key_items_per_s_all_heads"]
    res["step_s" if full else "step_s_extrapolated"] = step
    res["full"] = full
    res["tokens_per_s"] = N / step
    return res


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    ap.add_argument("--budget", type=float, default=10.0, help="seconds per sampled workload and thread count")
    ap.add_argument("--json", default=None)
    ap.add_argument("--workloads", default=",".join(FULL + SAMPLED))
    args = ap.parse_args(argv)
    oracle.build()
    out = []
    for name in args.workloads.split(","):
        for threads in (os.cpu_count() or 1, 1):
            r = time_workload(name, threads, args.budget)
            out.append(r)
            print(json.dumps(r), flush=True)
    if args.json:
        with open(args.json, "w") as f:
            json.dump(out, f, indent=1)


if __name__ == "__main__":
    main()
