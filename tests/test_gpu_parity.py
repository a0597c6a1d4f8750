"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle on the same seeded inputs.

Tolerances (max-abs): 1e-5 for fp32 I/O, 2e-2 for bf16 I/O with fp32 accumulation.  Small cases
compare every output element; the 720p workloads compare a seeded sample of queries (out, lse,
dq, doffsets) and of keys (dk, dv), which the oracle computes one by one.
"""
import dataclasses
import math

import numpy as np
import pytest
import torch

import oracle
from deformable_slide_attention_b200 import abi, inputs
from tests.gpu_helpers import (TOL, assert_close, edge_keys, f64, full_parity, gather_rows,
                               gpu_backward, gpu_forward, items_of, to_cuda)

pytestmark = [pytest.mark.gpu, pytest.mark.usefixtures("gpu_lib", "oracle_lib")]


def test_tiny_f32_workload_forward_and_backward():
    w = inputs.BY_NAME["tiny-f32"]
    inp = inputs.make(w, "cpu", with_dout=True)
    full_parity(inp, w.dims, w.window, "f32", backward=True)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("dh", [32, 64, 128])
def test_ragged_multi_tile(dtype, dh):
    # 3 x 7 x 9 tokens (not a multiple of any warp or tile size), 3 heads, 3x5x5 window
    _, inp = inputs.custom(3, 7, 9, 3, dh, (3, 5, 5), dtype, seed=100 + dh, scale=2.5)
    full_parity(inp, (3, 7, 9), (3, 5, 5), dtype)


@pytest.mark.parametrize("window", [(1, 1, 1), (1, 3, 3), (3, 1, 5), (5, 5, 3), (3, 9, 9)])
def test_windows(window):
    dims = (5, 10, 11)
    _, inp = inputs.custom(*dims, 2, 64, window, "bf16", seed=200 + sum(window), scale=2.0)
    full_parity(inp, dims, window, "bf16")


def test_single_frame_and_thin_volumes():
    for dims, window in (((1, 6, 7), (1, 3, 5)), ((4, 1, 9), (3, 1, 3)), ((2, 3, 1), (3, 5, 1))):
        _, inp = inputs.custom(*dims, 2, 32, window, "f32", seed=7, scale=1.2)
        full_parity(inp, dims, window, "f32")


def test_full_volume_window_zero_offsets():
    dims = (2, 3, 4)
    window = (3, 5, 7)
    _, inp = inputs.custom(*dims, 2, 32, window, "f32", seed=8)
    inp["offsets"].zero_()
    full_parity(inp, dims, window, "f32")


def test_integer_and_zero_offsets():
    dims, window = (4, 8, 8), (3, 5, 5)
    _, inp = inputs.custom(*dims, 2, 64, window, "bf16", seed=9)
    g = torch.Generator().manual_seed(1)
    off = torch.randint(-3, 4, inp["offsets"].shape, generator=g).float()
    off[0, :100] = 0.0
    inp["offsets"] = off
    full_parity(inp, dims, window, "bf16")


def test_many_queries_without_valid_taps():
    dims, window = (3, 6, 6), (1, 3, 3)
    _, inp = inputs.custom(*dims, 2, 32, window, "f32", seed=10, offsets="normal", scale=6.0)
    r_lse = oracle.full_forward(inp["q"], inp["k"], inp["v"], inp["offsets"], dims, window)[1]
    assert (~np.isfinite(r_lse)).sum() > 20
    full_parity(inp, dims, window, "f32")


def test_invalid_offsets_and_carry():
    dims, window = (3, 5, 6), (3, 3, 3)
    _, inp = inputs.custom(*dims, 2, 32, window, "f32", seed=11)
    off = inp["offsets"]
    off[0, 0, 0] = float("nan")
    off[0, 1, 1] = float("inf")
    off[1, 2, 2] = -float("inf")
    off[1, 3, 0] = 2.0 ** 25
    off[0, 4, 2] = -2.0 ** -30   # fraction rounds to 1 and carries
    off[1, 5, 1] = 1.0 - 2.0 ** -24
    full_parity(inp, dims, window, "f32")


@pytest.mark.parametrize("window,dh", [((3, 3, 15), 128), ((1, 1, 13), 128), ((5, 3, 11), 128),
                                       ((3, 5, 15), 64), ((3, 3, 11), 64)])
def test_widest_tensor_core_windows(window, dh):
    # k_w > 9 selects the forward's longer tap runs; k_w = 15 is the widest window of the path
    dims = (6, 9, 37)
    _, inp = inputs.custom(*dims, 2, dh, window, "bf16", seed=300 + window[2] + dh, scale=3.0)
    full_parity(inp, dims, window, "bf16")


def test_tall_windows_many_bucket_rows_per_key_tile():
    # a key tile of the key-side pass is covered by (k_t + 1) x (rows + k_h) bucket rows of queries:
    # 10 x 18 = 180 here, more than one batch of the per-tile range list
    dims, window = (6, 12, 10), (9, 17, 5)
    _, inp = inputs.custom(*dims, 2, 64, window, "bf16", seed=17, scale=2.5)
    full_parity(inp, dims, window, "bf16")


def test_tensor_core_path_sparse_and_invalid_queries():
    # large offsets: many queries leave the volume, bucket rows are sparse and ragged
    dims, window = (4, 7, 9), (3, 3, 3)
    _, inp = inputs.custom(*dims, 3, 64, window, "bf16", seed=13, offsets="normal", scale=5.0)
    inp["offsets"][0, 5, 1] = float("nan")
    inp["offsets"][2, 9, 2] = 2.0 ** 30
    full_parity(inp, dims, window, "bf16")


def test_tensor_core_path_dense_buckets():
    # all queries of a head share one origin (many queries per bucket, long chunks of equal x)
    dims, window = (3, 6, 20), (3, 5, 7)
    _, inp = inputs.custom(*dims, 2, 128, window, "bf16", seed=14)
    t, y, x = [torch.arange(math.prod(dims)) // (6 * 20), (torch.arange(math.prod(dims)) // 20) % 6,
               torch.arange(math.prod(dims)) % 20]
    inp["offsets"][0] = torch.stack([1.25 - t, 2.5 - y, 7.75 - x], -1).float()
    full_parity(inp, dims, window, "bf16")


def test_forward_workspace_head_groups():
    dims, window = (4, 6, 7), (3, 3, 5)
    _, inp = inputs.custom(*dims, 5, 64, window, "bf16", seed=15, with_dout=False)
    d = to_cuda(inp)
    full, _ = abi.forward(d["q"], d["k"], d["v"], d["offsets"], dims, window)
    one = abi.dsa3d_forward_workspace_bytes(*dims, 1, 64, *window, abi.DSA3D_BF16)
    ws = torch.empty(one + 100, dtype=torch.uint8, device="cuda")
    part, _ = abi.forward(d["q"], d["k"], d["v"], d["offsets"], dims, window, workspace=ws)
    torch.cuda.synchronize()
    assert torch.equal(full, part)


def test_small_bf16_workload_forward_full():
    w = inputs.BY_NAME["small-bf16"]
    inp = inputs.make(w, "cpu", with_dout=False)
    zero_frac = float((inp["offsets"] == 0).all(-1).float().mean())
    assert zero_frac >= 0.25
    full_parity(inp, w.dims, w.window, "bf16", backward=False)


def _sampled(w, n_q, n_k, seed, backward, key_edges=False):
    inp = inputs.make(w, "cpu", with_dout=backward)
    d = to_cuda(inp)
    out, lse = gpu_forward(d, w.dims, w.window)
    N = w.N
    tol = TOL[w.dtype]
    qi = items_of(w.heads, N, n_q, seed)
    r_out, r_lse = oracle.forward(inp["q"], inp["k"], inp["v"], inp["offsets"], w.dims, w.window, qi)
    assert_close("out", gather_rows(out, qi, N), r_out, tol)
    assert_close("lse", f64(lse).reshape(-1)[qi], r_lse, tol)
    if not backward:
        return
    dq, dk, dv, doff = gpu_backward(d, lse, w.dims, w.window)
    ki = items_of(w.heads, N, n_k, seed + 1)
    if key_edges:  # the key tiles' frame, row and segment edges on the first and last heads
        ki = np.union1d(ki, edge_keys(w.dims, (0, w.heads - 1), seed + 2))
    r_dq, r_doff, r_dk, r_dv = oracle.backward(inp["q"], inp["k"], inp["v"], inp["offsets"],
                                               inp["dout"], w.dims, w.window, qi, ki)
    assert_close("dq", gather_rows(dq, qi, N), r_dq, tol)
    assert_close("doff", f64(doff).reshape(-1, 3)[qi], r_doff, tol)
    assert_close("dk", gather_rows(dk, ki, N), r_dk, tol)
    assert_close("dv", gather_rows(dv, ki, N), r_dv, tol)


def test_small_bf16_workload_backward_sampled():
    w = dataclasses.replace(inputs.BY_NAME["small-bf16"], backward=True)
    _sampled(w, 256, 48, 31, True)


def test_720p_workload_forward_sampled():
    _sampled(inputs.BY_NAME["720p-bf16"], 512, 0, 32, False)


def test_720p_train_workload_sampled():
    _sampled(inputs.BY_NAME["720p-train-bf16"], 256, 24, 33, True, key_edges=True)


def test_forward_without_lse_matches():
    w = inputs.BY_NAME["tiny-f32"]
    d = to_cuda(inputs.make(w, "cpu", with_dout=False))
    out1, _ = gpu_forward(d, w.dims, w.window)
    out2, lse2 = abi.forward(d["q"], d["k"], d["v"], d["offsets"], w.dims, w.window, want_lse=False)
    torch.cuda.synchronize()
    assert lse2 is None and torch.equal(out1, out2)


def test_workspace_smaller_than_all_heads():
    """A workspace for one head processes the heads one group at a time with the same result."""
    dims, window = (3, 6, 7), (3, 3, 3)
    _, inp = inputs.custom(*dims, 4, 64, window, "bf16", seed=12)
    d = to_cuda(inp)
    out, lse = gpu_forward(d, dims, window)
    full = gpu_backward(d, lse, dims, window)
    one = abi.dsa3d_backward_workspace_bytes(*dims, 1, 64, *window, abi.DSA3D_BF16)
    ws = torch.empty(one, dtype=torch.uint8, device="cuda")
    part = abi.backward(d["q"], d["k"], d["v"], d["offsets"], lse, d["dout"], dims, window,
                        workspace=ws)
    torch.cuda.synchronize()
    for a, b in zip(full, part):
        assert torch.allclose(a.float(), b.float(), atol=TOL["bf16"], rtol=0)


def test_device_check_clean():
    assert abi.dsa3d_check_device(torch.cuda.current_stream().cuda_stream) == 0


def test_cuda_core_backward_when_workspace_only_fits_its_accumulators():
    """bf16 shapes with a tensor-core backward fall back to the CUDA-core backward when the
    workspace holds one head's fp32 dK/dV accumulators but not the tensor-core pass's splats."""
    dims, window, heads, dh = (4, 9, 10), (3, 9, 9), 2, 64
    _, inp = inputs.custom(*dims, heads, dh, window, "bf16", seed=16, scale=2.0)
    d = to_cuda(inp)
    out, lse = gpu_forward(d, dims, window)
    N = math.prod(dims)
    acc_one = 2 * N * dh * 4
    mma_one = abi.dsa3d_backward_workspace_bytes(*dims, 1, dh, *window, abi.DSA3D_BF16)
    assert mma_one > acc_one
    ws = torch.empty(acc_one, dtype=torch.uint8, device="cuda")
    abi.dsa3d_timing_reset()
    abi.dsa3d_timing_enable(True)
    grads = abi.backward(d["q"], d["k"], d["v"], d["offsets"], lse, d["dout"], dims, window, workspace=ws)
    torch.cuda.synchronize()
    abi.dsa3d_timing_enable(False)
    launched = abi.dsa3d_timing_read()
    assert "dsa3d_bwd_kernel" in launched and "dsa3d_bwd_q_kernel" not in launched
    r = oracle.full_backward(inp["q"], inp["k"], inp["v"], inp["offsets"], inp["dout"], dims, window)
    for name, got, ref in (("dq", grads[0], r[0]), ("doff", grads[3], r[1]), ("dk", grads[1], r[2]),
                           ("dv", grads[2], r[3])):
        assert_close(name, f64(got), ref, TOL["bf16"])
