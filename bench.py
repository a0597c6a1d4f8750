#!/usr/bin/env python
"""Benchmark: 3D-DSA forward + backward throughput on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

One step is one pass of the whole path over one batch: the forward (saving lse) and the backward
(dq, dk, dv, doffsets) of 3D Deformable Slide Attention on the named synthetic workload (default:
the 1080p long-video workload, 256 frames x 68 x 120 tokens, 32 heads x 128, window 3x9x9, bf16).
Inputs are resident in HBM when the timed region starts; every input tensor is larger than L2,
so no extra L2 flush is needed between steps.  Multi-GPU runs (torchrun) are weak scaling: each
rank processes its own independent clip (seed + rank); 3D-DSA has no exchange step.

``--impl reference`` times the CPU oracle (the only other implementation) on a bounded sample.
``--workload 720p-train-taps-bf16`` measures the per-tap offset entry points (one offset 3-vector
per window tap) on the 720p training shapes instead.  Prints one JSON line (rank 0).
"""
from __future__ import annotations

import argparse
import dataclasses
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "3D-DSA fwd+bwd tokens/s at N≈2.1M (1 B200) and % of HBM roofline"
DEFAULT_WORKLOAD = "1080p-long-bf16"


def metric_of(w):
    """The headline metric on the default workload; other workloads name themselves."""
    if w.name.startswith(DEFAULT_WORKLOAD):
        return METRIC
    kind = "per-tap offsets, " if w.per_tap else ""
    return f"3D-DSA fwd+bwd tokens/s ({kind}{w.name}, N={w.N}, 1 B200) and % of HBM roofline"
UNIT = "tokens/s"
FALLBACK_HBM_GBS = 6650.0
FP32_LANES_PER_SM = 128


def parse_args(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-e2e", action="store_true", help="skip the host-buffer end-to-end leg")
    ap.add_argument("--e2e-groups", type=int, default=0,
                    help="head groups of the end-to-end leg (a divisor of the heads; 0: the default choice)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=15.0, help="CPU-baseline sample budget")
    ap.add_argument("--part", choices=["attention", "dwconv"], default="attention",
                    help="attention: the operator's forward + backward (the default); dwconv: the "
                         "DWConv3D term of Eq. 1 alone (forward with the fused add, backward) at "
                         "the workload's shapes")
    ap.add_argument("--heads", type=int, default=0,
                    help="run only this many of the workload's heads (small profiling captures); "
                         "0 = all")
    return ap.parse_args(argv)


# DRAM traffic per (token, head) of each kernel, dram__bytes_read.sum + dram__bytes_write.sum
# from ncu captures (the file named by "capture" gives the command and workload), valid while the
# files that define those kernels and their launches ("files", under the package's csrc/) hash to
# "sources"; the traffic of a launch is this times the (token, head) items it processes (the
# kernels' traffic grows in proportion to the items).
TENSOR_CORE_FILES = ["dsa3d.cu", "dsa3d_common.cuh", "dsa3d_tc.cuh", "dsa3d_sort.cuh", "dsa3d_fwd_tc.cuh",
                     "dsa3d_fwd_mma.cuh", "dsa3d_bwd_mma.cuh", "dsa3d_bwd_dq_tc.cuh", "dsa3d_bwd_kv_tc.cuh"]
PER_TAP_FILES = ["dsa3d.cu", "dsa3d_common.cuh", "dsa3d_taps.cuh", "dsa3d_bwd.cuh", "dsa3d_fwd.cuh"]
NCU_TRAFFIC = [
    {"files": TENSOR_CORE_FILES, "sources": "415297fb73f643fa",
     "capture": "profiles/tensor_core_kernels_720p-train-bf16.md",
     "bytes_per_item": {
         "dsa3d_fwd_tc_kernel": 1020.1,
         "dsa3d_bwd_q_kernel": 2256.4,
         "dsa3d_bwd_dq_tc_kernel": 1701.6,
         "dsa3d_bwd_kv_tc_kernel": 2136.1,
     }},
    {"files": PER_TAP_FILES, "sources": "df10cf32e12d6270",
     "capture": "profiles/per_tap_kernels_720p-train-taps-bf16.md",
     "bytes_per_item": {
         "dsa3d_fwd_taps_kernel": 18471.7,
         "dsa3d_bwd_taps_kernel": 191471.2,
     }},
]


def traffic_per_item(kernel):
    """(DRAM bytes per item, capture file) of a kernel from a capture of the current sources, or
    (None, None)."""
    for cap in NCU_TRAFFIC:
        if kernel in cap["bytes_per_item"] and cap["sources"] == sources_digest(cap["files"]):
            return cap["bytes_per_item"][kernel], cap["capture"]
    return None, None


def sources_digest(names=None):
    """Digest of the named csrc files (all of csrc/ and include/ when names is None)."""
    import glob
    import hashlib
    csrc = os.path.join(ROOT, "deformable_slide_attention_b200", "csrc")
    if names is None:
        files = sorted(glob.glob(os.path.join(csrc, "*")) +
                       glob.glob(os.path.join(ROOT, "include", "*.h")))
    else:
        files = sorted(os.path.join(csrc, n) for n in names)
    h = hashlib.sha256()
    for f in files:
        h.update(os.path.basename(f).encode())
        with open(f, "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            return json.load(f), "measured"
    except (OSError, ValueError):
        return {"hbm_gbs": FALLBACK_HBM_GBS, "sm_max_mhz": 1965.0}, "fallback"


# --- algorithmic units -------------------------------------------------------------------------
# Per (token, head), each tensor the kernel must touch read or written once; s = element size.
# Whole path: forward 4 dh s + 16, backward 8 dh s + 28 (q, k, v, dO read; dq, dk, dv written;
# offsets, lse read; doffsets written).  Per kernel, the backward's three passes each re-read
# some inputs, so their sum (10 dh s + 28) exceeds the backward's figure.  With per-tap offsets
# the offsets and their gradient are K 3-vectors per (token, head): 12 K bytes each.
def alg_bytes_per_item(w, kernel):
    s = 4 if w.dtype == "f32" else 2
    if w.per_tap:
        ob = 12 * w.K
        return {"dsa3d_fwd_taps_kernel": 4 * w.dh * s + ob + 4,     # q, k, v, offsets -> out, lse
                "dsa3d_bwd_taps_kernel": 8 * w.dh * s + 2 * ob + 4,  # + dO, lse -> dq, dk, dv, doffsets
                "fwd": 4 * w.dh * s + ob + 4,
                "bwd": 8 * w.dh * s + 2 * ob + 4}.get(kernel, 0)
    table = {
        "dsa3d_fwd_kernel": 4 * w.dh * s + 16,        # q, k, v -> out; offsets, lse
        "dsa3d_fwd_mma_kernel": 4 * w.dh * s + 16,
        "dsa3d_fwd_tc_kernel": 4 * w.dh * s + 16,
        "dsa3d_bwd_kernel": 8 * w.dh * s + 28,        # the CUDA-core backward does it all
        "dsa3d_bwd_q_kernel": 4 * w.dh * s + 28,      # q, k, v, dO; offsets, lse -> doffsets
        "dsa3d_bwd_dq_kernel": 2 * w.dh * s,          # k -> dq
        "dsa3d_bwd_dq_tc_kernel": 2 * w.dh * s,       # the same on tcgen05
        "dsa3d_bwd_kv_kernel": 4 * w.dh * s,          # q, dO -> dk, dv
        "dsa3d_bwd_kv_tc_kernel": 4 * w.dh * s,       # the same on tcgen05
        "dsa3d_pair_v_kernel": 2 * w.dh * s,          # v -> paired value rows (workspace)
        "fwd": 4 * w.dh * s + 16,
        "bwd": 8 * w.dh * s + 28,
    }
    return table.get(kernel, 0)


def alg_flop_per_item(w, kernel):
    """Factorised fp32 work per (token, head): dots and axpys of length dh over the B box tokens.
    Per-tap offsets have no shared box: 8 corners per tap, 36 dh K forward (sampling k~ and v~,
    one dot, one axpy) and 64 dh K backward (per-corner dots with q and dO, then dq and the dK/dV
    scatter)."""
    if w.per_tap:
        return {"dsa3d_fwd_taps_kernel": 36, "dsa3d_bwd_taps_kernel": 64,
                "fwd": 36, "bwd": 64}.get(kernel, 0) * w.dh * w.K
    B = (w.window[0] + 1) * (w.window[1] + 1) * (w.window[2] + 1)
    per = {"dsa3d_fwd_kernel": 4, "dsa3d_fwd_mma_kernel": 4, "dsa3d_fwd_tc_kernel": 4, "dsa3d_bwd_kernel": 10,
           "dsa3d_bwd_q_kernel": 4, "dsa3d_bwd_dq_kernel": 2, "dsa3d_bwd_kv_kernel": 4,
           "dsa3d_bwd_kv_tc_kernel": 4, "dsa3d_bwd_dq_tc_kernel": 2,
           "fwd": 4, "bwd": 10}
    return per.get(kernel, 0) * w.dh * B


# --- clocks ------------------------------------------------------------------------------------
class ClockSampler:
    FIELDS = ("uuid,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, uuid):
        self.uuid = uuid
        self.rows = []
        self.proc = None
        self.thread = None

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) >= 9 and (not self.uuid or self.uuid in parts[0]):
                self.rows.append(parts)

    def stop(self):
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
        if self.thread:
            self.thread.join(timeout=5)
        sm = [float(r[1]) for r in self.rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in self.rows if r[2].replace(".", "").isdigit()]
        names = ["active", "hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = set()
        for r in self.rows:
            for i, n in enumerate(names[1:], start=5):
                if r[i].lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None,
                "reasons": sorted(reasons), "samples": len(self.rows)}


# --- CPU oracle leg ----------------------------------------------------------------------------
def oracle_sample(w, head_inputs, n_items, seed, threads):
    """Time the oracle on n_items seeded (token) queries of one head of workload w: its forward
    and the query side of its backward (dq, doffsets).  Returns seconds."""
    import numpy as np
    import oracle
    rng = np.random.default_rng(seed)
    items = np.sort(rng.choice(w.N, size=n_items, replace=False)).astype(np.int64)
    q, k, v, off, do = head_inputs
    t0 = time.perf_counter()
    oracle.forward(q, k, v, off, w.dims, w.window, items, threads, per_tap=w.per_tap)
    oracle.backward(q, k, v, off, do, w.dims, w.window, items, [], threads, per_tap=w.per_tap)
    return time.perf_counter() - t0


def head_inputs_for_oracle(w, inp, head=0):
    """One head's inputs as contiguous CPU tensors ([N][1][dh] and [1][N][3] or [1][N][K][3])."""
    pick = lambda t: t[:, head:head + 1, :].contiguous().cpu()
    return (pick(inp["q"]), pick(inp["k"]), pick(inp["v"]),
            inp["offsets"][head:head + 1].contiguous().cpu(), pick(inp["dout"]))


def calibrated_items(w, hin, threads, budget_s):
    """Items (a multiple of the thread count) that take about budget_s: time growing samples until
    one lasts half a second, so the per-call overhead does not distort the estimate."""
    threads = max(threads, 1)
    oracle_sample(w, hin, min(w.N, threads), 12344, threads)  # warm the inputs' pages
    rounds = 4
    while True:
        t = oracle_sample(w, hin, min(w.N, rounds * threads), 12345, threads)
        if t >= 0.5 or rounds >= (1 << 20) or rounds * threads >= w.N:
            break
        rounds *= 4
    rounds = min(rounds * threads, w.N) / threads
    per_round = t / rounds  # one item per thread
    # at most one head's queries (a sample is drawn without replacement from them)
    return min(w.N, max(1, int(budget_s / max(per_round, 1e-9))) * threads)


def cpu_baseline(w, inp, budget_s):
    import oracle
    oracle.build()
    threads = os.cpu_count() or 1
    hin = head_inputs_for_oracle(w, inp)
    n_items = calibrated_items(w, hin, threads, budget_s)
    secs = oracle_sample(w, hin, n_items, 777, threads)
    tokens = n_items / w.heads  # one token = all heads
    return {"value": tokens / secs, "unit": UNIT, "cores": threads, "kind": "oracle",
            "sample": (f"{n_items} seeded query tokens of head 0 of the {w.name} workload: oracle "
                       f"forward + query-side backward (dq, doffsets; dk/dv excluded), "
                       f"{secs:.1f} s on {threads} threads; tokens = items / {w.heads} heads")}


def run_reference(args):
    """--impl reference: the CPU oracle, K timed steps of a bounded sample each."""
    from deformable_slide_attention_b200 import ranks
    if ranks.rank_info().rank != 0:
        return 0  # rank 0 alone times the oracle; the other ranks exit without work
    import torch
    from deformable_slide_attention_b200 import inputs
    import oracle
    oracle.build()
    w = inputs.BY_NAME[args.workload]
    dev = "cuda" if (w.device_generated and torch.cuda.is_available()) else "cpu"
    if w.device_generated and dev == "cpu":
        # the 1080p workload is drawn on the device; without one, draw the same recipe on the CPU
        w = dataclasses.replace(w, device_generated=False)
    inp = inputs.make(w, dev, with_dout=True)
    hin = head_inputs_for_oracle(w, inp)
    del inp
    threads = os.cpu_count() or 1
    per_step = max(2.0, 150.0 / max(1, args.steps + args.warmup))
    n_items = calibrated_items(w, hin, threads, per_step)
    for i in range(args.warmup):
        oracle_sample(w, hin, n_items, 1000 + i, threads)
    secs = [oracle_sample(w, hin, n_items, 2000 + i, threads) for i in range(args.steps)]
    total = sum(secs)
    tokens_per_step = n_items / w.heads
    value = tokens_per_step * args.steps / total
    line = {
        "impl": "reference", "metric": metric_of(w), "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1000 * total / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": {"workload": w.name, "tokens": w.N, "heads": w.heads, "dh": w.dh,
                   "window": list(w.window)},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle",
                         "sample": f"per step {n_items} seeded query tokens of head 0: oracle forward "
                                   f"+ query-side backward (dq, doffsets); tokens = items / {w.heads}"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# --- GPU leg -----------------------------------------------------------------------------------
def path_of(w, abi):
    """The public forward and backward calls of the workload: per-token or per-tap offsets."""
    if not w.per_tap:
        return abi.forward, abi.backward

    def fwd(q, k, v, off, dims, window, out=None, lse=None, workspace=None):
        return abi.forward_taps(q, k, v, off, dims, window, out=out, lse=lse)
    return fwd, abi.backward_taps


def dwconv_units(w):
    """Per token, the DWConv3D term over C = heads * dh channels with the window's kernel:
    bytes: forward reads x and the attention output and writes the sum (3 C s), backward reads x
    and dy and writes dx (3 C s); flop: 2 C K each for the forward and dX, 2 C K for dW."""
    s = 4 if w.dtype == "f32" else 2
    C, K = w.heads * w.dh, w.K
    return {"fwd_bytes": 3 * C * s, "bwd_bytes": 3 * C * s,
            "fwd_flop": 2 * C * K, "bwd_flop": 4 * C * K}


def run_dwconv(args):
    """--part dwconv: the DWConv3D term's forward (fused into an attention-shaped output) and
    backward on one GPU, timed like the attention step; one JSON line."""
    import torch
    from deformable_slide_attention_b200 import abi, build, inputs
    build.build()
    w = inputs.BY_NAME[args.workload]
    if args.heads:
        w = dataclasses.replace(w, heads=args.heads)
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    C, N = w.heads * w.dh, w.N
    gen = torch.Generator(device=dev)
    gen.manual_seed(w.seed)
    td = w.torch_dtype
    x, y, dy = (torch.empty((N, C), dtype=td, device=dev) for _ in range(3))
    for t in (x, y, dy):
        inputs._fill_normal_chunked(t, gen)
    weight = torch.empty((C, *w.window), dtype=torch.float32, device=dev)
    weight.normal_(0.0, 1.0 / math.sqrt(w.K), generator=gen)
    bias = torch.empty(C, dtype=torch.float32, device=dev)
    bias.normal_(0.0, 1.0, generator=gen)
    stream = torch.cuda.current_stream(dev)

    def step():
        abi.dwconv3d(x, weight, bias, w.dims, add=y, out=y)  # y += conv(x): the layer's sum
        abi.dwconv3d_backward(x, weight, dy, w.dims)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    props = torch.cuda.get_device_properties(dev)
    sampler = ClockSampler(str(getattr(props, "uuid", "") or ""))
    sampler.start()
    time.sleep(0.5)
    abi.dsa3d_timing_reset()
    abi.dsa3d_timing_enable(True)
    torch.cuda.synchronize(dev)
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for _ in range(args.steps):
        step()
    t1.record(stream)
    torch.cuda.synchronize(dev)
    abi.dsa3d_timing_enable(False)
    ktimes = abi.dsa3d_timing_read()
    clocks = sampler.stop()
    ms = t0.elapsed_time(t1) / args.steps
    u = dwconv_units(w)
    peaks, peak_src = measured_peaks()
    mhz = clocks["sm_mhz"] or float(peaks.get("sm_max_mhz", 1965.0))
    fp32_peak = props.multi_processor_count * FP32_LANES_PER_SM * 2 * mhz * 1e6 / 1e12
    flop = N * (u["fwd_flop"] + u["bwd_flop"])
    tflops = flop / (ms / 1000.0) / 1e12
    line = {
        "metric": f"3D-DSA DWConv3D term fwd+bwd tokens/s ({w.name} shapes, C={C}, 1 B200)",
        "value": N / (ms / 1000.0), "unit": UNIT, "n_gpus": 1, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": w.dtype, "data": "synthetic",
        "config": {"workload": w.name, "part": "dwconv", "tokens": N, "channels": C,
                   "kernel": list(w.window), "l2": "inputs larger than L2; no flush"},
        "roofline": {"bound": "alu", "achieved": tflops, "peak": fp32_peak, "unit": "TFLOP/s",
                     "frac": tflops / fp32_peak, "traffic": None,
                     "peak_basis": f"{props.multi_processor_count} SMs x 128 fp32 lanes x 2 x {mhz:.0f} MHz"},
        "hbm": {"alg_bytes_per_step": N * (u["fwd_bytes"] + u["bwd_bytes"]),
                "frac_of_hbm": N * (u["fwd_bytes"] + u["bwd_bytes"]) / (ms / 1000.0) / 1e9
                               / float(peaks.get("hbm_gbs", FALLBACK_HBM_GBS))},
        "kernels": {k: {"launches": n, "avg_ms": tot / n} for k, (n, tot) in ktimes.items()},
        "gpu_launches": sum(n for n, _ in ktimes.values()), "clocks": clocks,
        "e2e": None, "cpu_baseline": None,
    }
    print(json.dumps(line), flush=True)
    return 0


def main(argv=None):
    args = parse_args(argv)
    if args.impl == "reference":
        return run_reference(args)
    if args.part == "dwconv":
        return run_dwconv(args)
    import torch
    import torch.distributed as dist
    from deformable_slide_attention_b200 import abi, build, inputs, ranks

    ri = ranks.rank_info()
    world, rank, local = ri.world, ri.rank, ri.local
    if world != args.gpus:
        print(f"warning: --gpus {args.gpus} but WORLD_SIZE {world}", file=sys.stderr)
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=600), device_id=dev)
    build.build()

    base = inputs.BY_NAME[args.workload]
    if args.heads:
        base = dataclasses.replace(base, heads=args.heads)
    w = ranks.clip_workload(base, rank)
    inp = inputs.make(w, dev, with_dout=True)
    code = abi.DSA3D_BF16 if w.dtype == "bf16" else abi.DSA3D_F32
    q, k, v, off, do = (inp[n] for n in ("q", "k", "v", "offsets", "dout"))
    out = torch.empty_like(q)
    lse = torch.empty((w.heads, w.N), dtype=torch.float32, device=dev)
    dq, dk, dv, doff = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v), torch.empty_like(off)
    # one workspace serves the forward and the backward (they run one after the other on the
    # stream): all heads at once when that fits in free memory minus a margin, else head groups
    if w.per_tap:  # the per-tap forward takes no workspace
        fws_bytes = 0
        full_ws = abi.dsa3d_backward_taps_workspace_bytes(*w.dims, w.heads, w.dh, *w.window, code)
    else:
        fws_bytes = abi.dsa3d_forward_workspace_bytes(*w.dims, w.heads, w.dh, *w.window, code)
        full_ws = abi.dsa3d_backward_workspace_bytes(*w.dims, w.heads, w.dh, *w.window, code)
    per_head = full_ws // w.heads if full_ws else 0
    free, _ = torch.cuda.mem_get_info(dev)
    margin = 6 << 30
    ws_bytes = max(16, min(max(fws_bytes, full_ws), free - margin))
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    heads_per_pass = w.heads if not per_head else max(1, min(w.heads, ws_bytes // per_head))
    fwd_heads = w.heads
    while not w.per_tap and fwd_heads > 1 and abi.dsa3d_forward_workspace_bytes(
            *w.dims, fwd_heads, w.dh, *w.window, code) > ws_bytes:
        fwd_heads = (fwd_heads + 1) // 2
    stream = torch.cuda.current_stream(dev)
    fwd_fn, bwd_fn = path_of(w, abi)

    def step():
        fwd_fn(q, k, v, off, w.dims, w.window, out=out, lse=lse, workspace=ws)
        bwd_fn(q, k, v, off, lse, do, w.dims, w.window, workspace=ws, grads=(dq, dk, dv, doff))

    def barrier():
        if world > 1:
            dist.barrier()

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)

    props = torch.cuda.get_device_properties(dev)
    uuid = str(getattr(props, "uuid", "") or "")
    sampler = ClockSampler(uuid)
    sampler.start()
    time.sleep(0.5)
    abi.dsa3d_timing_reset()
    abi.dsa3d_timing_enable(True)
    barrier()
    torch.cuda.synchronize(dev)
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for _ in range(args.steps):
        step()
    t1.record(stream)
    torch.cuda.synchronize(dev)
    barrier()
    abi.dsa3d_timing_enable(False)
    ktimes = abi.dsa3d_timing_read()
    clocks = sampler.stop()
    ms = ranks.max_over_ranks(t0.elapsed_time(t1) / args.steps, dev)
    value = ranks.job_rate(w.N, world, ms)
    launches = sum(n for n, _ in ktimes.values())

    peaks, peak_src = measured_peaks()
    hbm = float(peaks.get("hbm_gbs", FALLBACK_HBM_GBS))
    dominant = max(ktimes.items(), key=lambda kv: kv[1][1]) if ktimes else None
    roof = None
    alu = None
    kernel_table = {kname: {"launches": n, "avg_ms": tot / n, "share": tot / sum(x[1] for x in ktimes.values())}
                    for kname, (n, tot) in ktimes.items()}
    if dominant:
        kname, (n, tot) = dominant
        avg_ms = tot / n
        launches_per_step = n / args.steps
        items_per_launch = w.heads * w.N / launches_per_step
        alg = alg_bytes_per_item(w, kname) * items_per_launch
        achieved = alg / (avg_ms / 1000.0) / 1e9
        per_item, capture = traffic_per_item(kname)
        traffic = per_item * items_per_launch if per_item is not None else None
        roof = {"bound": "hbm", "achieved": achieved, "peak": hbm, "unit": "GB/s",
                "frac": achieved / hbm, "traffic": traffic, "traffic_unit": "bytes per launch",
                "traffic_source": capture,
                "kernel": kname,
                "peak_source": f"{peak_src} hbm_gbs (MEASURED_PEAKS.json)"
                               if peak_src == "measured" else "fallback 6.65 TB/s"}
        mhz = clocks["sm_mhz"] or float(peaks.get("sm_max_mhz", 1965.0))
        fp32_peak = props.multi_processor_count * FP32_LANES_PER_SM * 2 * mhz * 1e6 / 1e12
        flops = alg_flop_per_item(w, kname) * items_per_launch
        alu = {"bound": "alu", "achieved": flops / (avg_ms / 1000.0) / 1e12, "unit": "TFLOP/s",
               "peak": fp32_peak, "frac": flops / (avg_ms / 1000.0) / 1e12 / fp32_peak,
               "peak_basis": f"{props.multi_processor_count} SMs x 128 fp32 lanes x 2 x {mhz:.0f} MHz"}
    step_bytes = w.heads * w.N * (alg_bytes_per_item(w, "fwd") + alg_bytes_per_item(w, "bwd"))
    step_roof = {"alg_bytes_per_step": step_bytes,
                 "achieved_gbs": step_bytes / (ms / 1000.0) / 1e9,
                 "frac_of_hbm": step_bytes / (ms / 1000.0) / 1e9 / hbm}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(w, inp, args.cpu_seconds)

    # end to end through the public API with pinned host buffers: the host copies are taken from
    # the device inputs, then the device leg's tensors are released for the leg's own buffers
    e2e = None
    if not args.no_e2e:
        host, why = e2e_host(w, inp, torch, dev, world)
        del step
        inp = q = k = v = off = do = out = lse = dq = dk = dv = doff = ws = None
        torch.cuda.empty_cache()
        if host is None:
            e2e = {"value": None, "unit": UNIT, "skipped": why}
        else:
            e2e = e2e_leg(args, w, host, abi, torch, dev, world, code)
            host.clear()

    line = {
        "metric": metric_of(w), "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": w.dtype, "data": "synthetic",
        "config": {"workload": w.name, "frames": w.F, "grid": [w.Hp, w.Wp], "tokens": w.N,
                   "heads": w.heads, "dh": w.dh, "window": list(w.window),
                   "offsets": "per tap [heads][N][K][3]" if w.per_tap else "per token [heads][N][3]",
                   "heads_per_forward_pass": fwd_heads,
                   "heads_per_backward_pass": heads_per_pass,
                   "l2": "inputs larger than L2 (each tensor > 126 MB); no flush",
                   "parallelism": f"independent clip per GPU x{world}"},
        "roofline": roof, "alu_roofline": alu, "step_roofline": step_roof,
        "kernels": kernel_table, "gpu_launches": launches, "clocks": clocks,
        "e2e": e2e, "cpu_baseline": cpu,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def _cudart():
    """The CUDA runtime library torch has loaded (for 2-D copies between pitched host and device
    rows, which torch's copy_ does not issue)."""
    import ctypes
    lib = None
    with open("/proc/self/maps") as f:
        for line in f:
            if "libcudart.so" in line:
                lib = line.split()[-1]
                break
    rt = ctypes.CDLL(lib or "libcudart.so.12")
    rt.cudaMemcpy2DAsync.argtypes = [ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p, ctypes.c_size_t,
                                     ctypes.c_size_t, ctypes.c_size_t, ctypes.c_int, ctypes.c_void_p]
    rt.cudaMemcpy2DAsync.restype = ctypes.c_int
    return rt


def e2e_host(w, inp, torch, dev, world):
    """Pinned host copies of the step's inputs and a pinned read-back area, or (None, reason)."""
    names_in = ("q", "k", "v", "offsets", "dout")
    in_bytes = sum(inp[n].numel() * inp[n].element_size() for n in names_in)
    row_bytes = inp["q"].numel() * inp["q"].element_size()
    host_out_bytes = row_bytes + w.heads * w.N * 4 + inp["offsets"].numel() * 4
    try:
        import psutil
        avail = psutil.virtual_memory().available
    except ImportError:
        avail = 0
    # every rank on this node pins its own buffers at about the same time: each may use its share
    # of the free RAM only
    local_ranks = max(1, int(os.environ.get("LOCAL_WORLD_SIZE", str(world))))
    avail //= local_ranks
    skip = in_bytes + host_out_bytes > 0.75 * avail
    if world > 1:
        # the ranks must agree on running the leg (it contains collectives)
        from deformable_slide_attention_b200 import ranks
        skip = ranks.max_over_ranks(1.0 if skip else 0.0, dev) > 0.5
    if skip:
        return None, (f"host RAM share {avail >> 30} GiB per rank too small for "
                      f"{(in_bytes + host_out_bytes) >> 30} GiB")
    host = {}
    try:
        for n in names_in:
            host[n] = torch.empty(inp[n].shape, dtype=inp[n].dtype, pin_memory=True)
            host[n].copy_(inp[n])
        host["rows"] = torch.empty(inp["q"].shape, dtype=inp["q"].dtype, pin_memory=True)
        host["lse"] = torch.empty((w.heads, w.N), dtype=torch.float32, pin_memory=True)
        host["doff"] = torch.empty(inp["offsets"].shape, dtype=torch.float32, pin_memory=True)
    except RuntimeError as e:
        err = str(e)
    else:
        err = None
    failed = err is not None
    if world > 1:  # every rank runs the leg or none does
        from deformable_slide_attention_b200 import ranks
        failed = ranks.max_over_ranks(1.0 if failed else 0.0, dev) > 0.5
    if failed:
        host.clear()
        return None, f"pinned host buffers unavailable: {err or 'on another rank'}"[:200]
    return host, None


def e2e_leg(args, w, host, abi, torch, dev, world, code):
    """The step through the public API with host inputs and results: every step copies all inputs
    host->device from pinned buffers and reads every output (out, lse, dq, dk, dv, doffsets) back
    device->host.  The step runs as G head groups (heads are independent), each a forward and a
    backward call on [N][g][dh] tensors, through two slots of device buffers: group i+1's inputs
    cross on their own stream (pitched 2-D copies out of the [N][heads][dh] host arrays) while
    group i computes, and group i-1's outputs come back on a third stream, so both directions of
    the link and the compute overlap.  Host RAM holds the pinned inputs and a read-back area: lse
    and doffsets each their own, one [N][heads][dh] buffer that out, dq, dk and dv pass through in
    turn."""
    from deformable_slide_attention_b200 import ranks
    s = 4 if w.dtype == "f32" else 2
    H, N, dh = w.heads, w.N, w.dh
    off_per_head = host["offsets"][0].numel()  # N*3, or N*K*3 with per-tap offsets

    def ws_bytes(g):
        if w.per_tap:
            return abi.dsa3d_backward_taps_workspace_bytes(*w.dims, g, dh, *w.window, code)
        return max(abi.dsa3d_forward_workspace_bytes(*w.dims, g, dh, *w.window, code),
                   abi.dsa3d_backward_workspace_bytes(*w.dims, g, dh, *w.window, code))

    def slot_bytes(g):
        return 8 * N * g * dh * s + 2 * g * off_per_head * 4 + g * N * 4

    free, _ = torch.cuda.mem_get_info(dev)
    budget = free - (6 << 30)
    # the largest group that fits, with four groups or more where the heads allow it (the first
    # group's inputs and the last one's outputs are the pipeline's fill and drain)
    g = 1
    if args.e2e_groups > 0:
        if H % args.e2e_groups:
            raise SystemExit(f"--e2e-groups {args.e2e_groups} does not divide the {H} heads")
        g = H // args.e2e_groups
        if 2 * slot_bytes(g) + ws_bytes(g) > budget:
            raise SystemExit(f"--e2e-groups {args.e2e_groups}: the group's device buffers do not fit")
    else:
        for cand in list(range(H // 4, 0, -1)) + list(range(H // 2, H // 4, -1)):
            if cand >= 1 and H % cand == 0 and 2 * slot_bytes(cand) + ws_bytes(cand) <= budget:
                g = cand
                break
    G = H // g
    slots = []
    for _ in range(2):
        t = {n: torch.empty((N, g, dh), dtype=host["q"].dtype, device=dev)
             for n in ("q", "k", "v", "dout", "out", "dq", "dk", "dv")}
        t["offsets"] = torch.empty((g,) + tuple(host["offsets"].shape[1:]), dtype=torch.float32, device=dev)
        t["doff"] = torch.empty_like(t["offsets"])
        t["lse"] = torch.empty((g, N), dtype=torch.float32, device=dev)
        slots.append(t)
    ws = torch.empty(max(16, ws_bytes(g)), dtype=torch.uint8, device=dev)
    rt = _cudart()
    row_src, row_dst = H * dh * s, g * dh * s  # bytes per token row: host arrays, group slices
    compute = torch.cuda.current_stream(dev)
    s_h2d, s_d2h = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    fwd_fn, bwd_fn = path_of(w, abi)
    ev = {"comp": [None, None], "out": [None, None]}
    state = {"k": 0, "start": None, "last": None}
    nbytes = {"h2d": 0, "d2h": 0}

    def copy2d(dst, dpitch, src, spitch, width, stream, kind):
        rc = rt.cudaMemcpy2DAsync(dst, dpitch, src, spitch, width, N, kind, stream.cuda_stream)
        if rc != 0:
            raise RuntimeError(f"cudaMemcpy2DAsync failed ({rc})")

    def group(h0):
        sl = state["k"] % 2
        state["k"] += 1
        t = slots[sl]
        # inputs: the slot's previous group must have finished reading them
        if ev["comp"][sl] is not None:
            s_h2d.wait_event(ev["comp"][sl])
        elif state["start"] is not None:
            s_h2d.wait_event(state["start"])
        for n in ("q", "k", "v", "dout"):
            copy2d(t[n].data_ptr(), row_dst, host[n].data_ptr() + h0 * dh * s, row_src, row_dst, s_h2d, 1)
            nbytes["h2d"] += N * row_dst
        with torch.cuda.stream(s_h2d):
            t["offsets"].copy_(host["offsets"][h0:h0 + g], non_blocking=True)
        nbytes["h2d"] += t["offsets"].numel() * 4
        arrived = torch.cuda.Event()
        arrived.record(s_h2d)
        compute.wait_event(arrived)
        if ev["out"][sl] is not None:  # the slot's outputs have been read back
            compute.wait_event(ev["out"][sl])
        fwd_fn(t["q"], t["k"], t["v"], t["offsets"], w.dims, w.window, out=t["out"], lse=t["lse"], workspace=ws)
        bwd_fn(t["q"], t["k"], t["v"], t["offsets"], t["lse"], t["dout"], w.dims, w.window, workspace=ws,
               grads=(t["dq"], t["dk"], t["dv"], t["doff"]))
        done = torch.cuda.Event()
        done.record(compute)
        ev["comp"][sl] = done
        s_d2h.wait_event(done)
        for n in ("out", "dq", "dk", "dv"):
            copy2d(host["rows"].data_ptr() + h0 * dh * s, row_src, t[n].data_ptr(), row_dst, row_dst, s_d2h, 2)
            nbytes["d2h"] += N * row_dst
        with torch.cuda.stream(s_d2h):
            host["lse"][h0:h0 + g].copy_(t["lse"], non_blocking=True)
            host["doff"][h0:h0 + g].copy_(t["doff"], non_blocking=True)
        nbytes["d2h"] += t["lse"].numel() * 4 + t["doff"].numel() * 4
        read = torch.cuda.Event()
        read.record(s_d2h)
        ev["out"][sl] = read
        state["last"] = read

    def step():
        for gi in range(G):
            group(gi * g)

    step()
    torch.cuda.synchronize(dev)
    steps = max(1, min(args.steps, 3))
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(compute)
    begin = torch.cuda.Event()
    begin.record(compute)
    ev["comp"] = [begin, begin]  # the first timed copies start after t0
    nbytes["h2d"] = nbytes["d2h"] = 0
    for _ in range(steps):
        step()
    compute.wait_event(state["last"])  # the last read-back is inside the timed region
    t1.record(compute)
    torch.cuda.synchronize(dev)
    ms = ranks.max_over_ranks(t0.elapsed_time(t1) / steps, dev)
    return {"value": ranks.job_rate(w.N, world, ms), "unit": UNIT, "ms_per_step": ms, "steps": steps,
            "h2d_bytes_per_step": nbytes["h2d"] // steps, "d2h_bytes_per_step": nbytes["d2h"] // steps,
            "read_back": ["dk", "doffsets", "dq", "dv", "lse", "out"],
            "head_groups": G, "heads_per_group": g,
            "overlap": "per head group: inputs of group i+1 and outputs of group i-1 (own streams) "
                       "while group i computes"}


if __name__ == "__main__":
    sys.exit(main())
