"""Parity at the full 1080p long-video size (F=256, 68x120, 32 heads x 128, window 3x9x9, bf16),
in the launch configuration bench.py times (forward workspace for all heads, backward workspace
sized from free device memory).  The oracle computes a seeded sample of outputs one by one on two
heads; invariants that hold at any size are checked on every head:
  sum_j dV[j, h] = sum over queries with a valid tap of dO[q, h]  (the value weights sum to 1)
  sum_j dK[j, h] = 0                                               (the dS of a query sum to 0)
"""
import numpy as np
import pytest
import torch

import oracle
from deformable_slide_attention_b200 import abi, inputs
from tests.gpu_helpers import TOL, assert_close, edge_keys, items_of

pytestmark = [pytest.mark.gpu, pytest.mark.usefixtures("gpu_lib", "oracle_lib")]


def test_1080p_workload_full_size():
    w = inputs.BY_NAME["1080p-long-bf16"]
    dev = torch.device("cuda", 0)
    free0, _ = torch.cuda.mem_get_info(dev)
    if free0 < 160 << 30:
        pytest.fail(f"the 1080p workload needs ~150 GB of device memory; {free0 >> 30} GiB free")
    inp = inputs.make(w, dev, with_dout=True)
    q, k, v, off, do = (inp[n] for n in ("q", "k", "v", "offsets", "dout"))
    code = abi.DSA3D_BF16
    out, lse = torch.empty_like(q), torch.empty((w.heads, w.N), dtype=torch.float32, device=dev)
    grads = (torch.empty_like(q), torch.empty_like(k), torch.empty_like(v), torch.empty_like(off))
    # one workspace for both calls, sized as bench.py sizes it
    fws = abi.dsa3d_forward_workspace_bytes(*w.dims, w.heads, w.dh, *w.window, code)
    full_ws = abi.dsa3d_backward_workspace_bytes(*w.dims, w.heads, w.dh, *w.window, code)
    free, _ = torch.cuda.mem_get_info(dev)
    ws = torch.empty(max(16, min(max(fws, full_ws), free - (6 << 30))), dtype=torch.uint8, device=dev)
    out, lse = abi.forward(q, k, v, off, w.dims, w.window, out=out, lse=lse, workspace=ws)
    dq, dk, dv, doff = abi.backward(q, k, v, off, lse, do, w.dims, w.window, workspace=ws, grads=grads)
    torch.cuda.synchronize()
    del ws

    # invariants on every head
    valid = torch.isfinite(lse).t()  # [N][heads]
    for h in range(w.heads):
        sdv = dv[:, h].double().sum(0)
        sdo = (do[:, h].double() * valid[:, h, None]).sum(0)
        assert torch.allclose(sdv, sdo, atol=2e-3 * w.N ** 0.5, rtol=0), h
        sdk = dk[:, h].double().sum(0)
        assert float(sdk.abs().max()) <= 1e-3 * float(dk[:, h].double().abs().sum(0).max()), h

    # sampled parity on two heads against the oracle (one head's tensors copied to the host)
    tol = TOL["bf16"]
    for h in (0, w.heads - 1):
        pick = lambda t: t[:, h:h + 1].contiguous().cpu()
        hq, hk, hv, hdo = pick(q), pick(k), pick(v), pick(do)
        hoff = off[h:h + 1].contiguous().cpu()
        qi = items_of(1, w.N, 96, seed=40 + h)           # query tokens (head index 0 of the slice)
        # key tokens: the key tiles' frame, row and segment edges, and a few at random
        ki = edge_keys(w.dims, (0,), seed=50 + h, n_random=8)
        r_out, r_lse = oracle.forward(hq, hk, hv, hoff, w.dims, w.window, qi)
        assert_close("out", out[qi, h].float().cpu().double().numpy(), r_out, tol)
        assert_close("lse", lse[h, qi].cpu().double().numpy(), r_lse, tol)
        r_dq, r_doff, r_dk, r_dv = oracle.backward(hq, hk, hv, hoff, hdo, w.dims, w.window, qi, ki)
        assert_close("dq", dq[qi, h].float().cpu().double().numpy(), r_dq, tol)
        assert_close("doff", doff[h, qi].cpu().double().numpy(), r_doff, tol)
        assert_close("dk", dk[ki, h].float().cpu().double().numpy(), r_dk, tol)
        assert_close("dv", dv[ki, h].float().cpu().double().numpy(), r_dv, tol)
