"""GPU parity of the per-tap offset entry points (dsa3d_forward_taps / dsa3d_backward_taps) against
the CPU oracle's per-tap mode, on the same seeded inputs.

Per-tap offsets are the offset tensor of the 3D-DSA definition (MegaSlide-DiT, Eq. 1) with one
3-vector per window tap: [heads][N][K][3].  Tolerances as in the per-token parity tests: max-abs
1e-5 for fp32 I/O, 2e-2 for bf16 I/O with fp32 accumulation.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from deformable_slide_attention_b200 import abi, inputs
from tests.gpu_helpers import TOL, assert_close, f64, gather_rows, items_of, to_cuda

pytestmark = [pytest.mark.gpu, pytest.mark.usefixtures("gpu_lib", "oracle_lib")]


def _gpu(d, dims, window, backward=True):
    out, lse = abi.forward_taps(d["q"], d["k"], d["v"], d["offsets"], dims, window)
    grads = None
    if backward:
        grads = abi.backward_taps(d["q"], d["k"], d["v"], d["offsets"], lse, d["dout"], dims, window)
    torch.cuda.synchronize()
    assert abi.dsa3d_check_device(torch.cuda.current_stream().cuda_stream) == 0
    return out, lse, grads


def parity_taps(inp, dims, window, dtype, backward=True):
    tol = TOL[dtype]
    d = to_cuda(inp)
    out, lse, grads = _gpu(d, dims, window, backward)
    r_out, r_lse = oracle.full_forward(inp["q"], inp["k"], inp["v"], inp["offsets"], dims, window,
                                       per_tap=True)
    assert_close("out", f64(out), r_out, tol)
    assert_close("lse", f64(lse), r_lse, max(tol, 1e-5))
    if not backward:
        return out, lse, None
    dq, dk, dv, doff = grads
    r_dq, r_doff, r_dk, r_dv = oracle.full_backward(inp["q"], inp["k"], inp["v"], inp["offsets"],
                                                    inp["dout"], dims, window, per_tap=True)
    assert tuple(doff.shape) == r_doff.shape
    for name, got, ref in (("dq", dq, r_dq), ("doff", doff, r_doff), ("dk", dk, r_dk), ("dv", dv, r_dv)):
        assert_close(name, f64(got), ref, tol)
    return out, lse, grads


def test_tiny_f32_per_tap():
    _, inp = inputs.custom(4, 8, 8, 2, 32, (3, 3, 3), "f32", seed=40, per_tap=True)
    parity_taps(inp, (4, 8, 8), (3, 3, 3), "f32")


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("dh", [32, 64, 128])
def test_ragged_blocks(dtype, dh):
    # 75 taps: two full blocks of 32 and a ragged one of 11; 3 x 7 x 9 tokens, 3 heads
    _, inp = inputs.custom(3, 7, 9, 3, dh, (3, 5, 5), dtype, seed=41 + dh, scale=2.0, per_tap=True)
    parity_taps(inp, (3, 7, 9), (3, 5, 5), dtype)


@pytest.mark.parametrize("window", [(1, 1, 1), (1, 3, 3), (3, 1, 5), (1, 5, 7), (3, 9, 9)])
def test_windows(window):
    dims = (4, 10, 11)
    _, inp = inputs.custom(*dims, 2, 64, window, "bf16", seed=50 + sum(window), offsets="normal",
                           scale=2.0, per_tap=True)
    parity_taps(inp, dims, window, "bf16")


def test_per_tap_equals_per_token_when_taps_share_the_offset():
    """Every tap carrying the query's per-token offset gives the per-token operator (R1 is R8 with
    one offset repeated); compared with the per-token general CUDA-core kernels and the oracle."""
    dims, window = (4, 7, 8), (3, 3, 5)
    K = math.prod(window)
    _, inp = inputs.custom(*dims, 2, 64, window, "f32", seed=60, scale=2.5)
    tok = {k: v for k, v in inp.items()}
    taps = dict(tok, offsets=tok["offsets"][:, :, None, :].expand(-1, -1, K, -1).contiguous())
    out_t, lse_t, g_t = parity_taps(taps, dims, window, "f32")
    d = to_cuda(tok)
    out, lse = abi.forward(d["q"], d["k"], d["v"], d["offsets"], dims, window, workspace=None)
    dq, dk, dv, doff = abi.backward(d["q"], d["k"], d["v"], d["offsets"], lse, d["dout"], dims, window)
    torch.cuda.synchronize()
    tol = TOL["f32"]
    assert_close("out", f64(out_t), f64(out), tol)
    assert_close("lse", f64(lse_t), f64(lse), tol)
    for name, a, b in (("dq", g_t[0], dq), ("dk", g_t[1], dk), ("dv", g_t[2], dv)):
        assert_close(name, f64(a), f64(b), tol)
    # the per-token offset gradient is the sum of the per-tap gradients over the taps
    assert_close("doff", f64(g_t[3]).sum(axis=2), f64(doff), 1e-4)


def test_non_finite_and_large_tap_offsets_mask_only_their_tap():
    dims, window = (3, 6, 7), (3, 3, 3)
    _, inp = inputs.custom(*dims, 2, 32, window, "f32", seed=61, per_tap=True)
    off = inp["offsets"]
    off[0, 5, 0, 0] = float("nan")
    off[0, 5, 13, 1] = float("inf")
    off[1, 9, 26, 2] = -float("inf")
    off[1, 10, 4, 0] = 2.0 ** 25
    off[0, 11, 7, 2] = -2.0 ** -30          # the fraction rounds to 1 and carries
    off[1, 12, 8, 1] = 1.0 - 2.0 ** -24
    off[0, 20, :, :] = float("nan")         # every tap masked: out 0, lse -inf, zero gradients
    out, lse, grads = parity_taps(inp, dims, window, "f32")
    assert np.isfinite(f64(lse)[0, 5]) and f64(lse)[0, 20] == -np.inf
    assert not f64(out)[20, 0].any() and not f64(grads[3])[0, 20].any()


def test_queries_outside_the_volume_and_integer_offsets():
    dims, window = (3, 6, 6), (1, 3, 3)
    _, inp = inputs.custom(*dims, 2, 64, window, "bf16", seed=62, offsets="normal", scale=5.0,
                           per_tap=True)
    g = torch.Generator().manual_seed(3)
    ints = torch.randint(-2, 3, inp["offsets"][1].shape, generator=g).float()
    inp["offsets"][1] = ints  # head 1: integer offsets (zero fractions: single-corner taps)
    r_lse = oracle.full_forward(inp["q"], inp["k"], inp["v"], inp["offsets"], dims, window,
                                per_tap=True)[1]
    assert (~np.isfinite(r_lse[0])).sum() > 0
    parity_taps(inp, dims, window, "bf16")


def test_backward_workspace_head_groups():
    dims, window = (3, 6, 7), (3, 3, 3)
    _, inp = inputs.custom(*dims, 5, 64, window, "bf16", seed=63, per_tap=True)
    d = to_cuda(inp)
    out, lse, full = _gpu(d, dims, window)
    one = abi.dsa3d_backward_taps_workspace_bytes(*dims, 1, 64, *window, abi.DSA3D_BF16)
    ws = torch.empty(2 * one + 64, dtype=torch.uint8, device="cuda")
    part = abi.backward_taps(d["q"], d["k"], d["v"], d["offsets"], lse, d["dout"], dims, window,
                             workspace=ws)
    torch.cuda.synchronize()
    for a, b in zip(full, part):
        assert torch.allclose(a.float(), b.float(), atol=TOL["bf16"], rtol=0)


def test_720p_per_tap_training_sampled():
    """The 720p per-tap training workload at full size (the benchmark's per-tap case): sampled
    queries (out, lse, dq, per-tap doff) and keys (dk, dv) against the oracle."""
    w = inputs.BY_NAME["720p-train-taps-bf16"]
    d = inputs.make(w, "cuda", with_dout=True)
    out, lse, (dq, dk, dv, doff) = _gpu(d, w.dims, w.window)
    cpu = {k: v.cpu() for k, v in d.items()}
    N, tol = w.N, TOL["bf16"]
    qi = items_of(w.heads, N, 96, 70)
    ki = items_of(w.heads, N, 12, 71)
    r_out, r_lse = oracle.forward(cpu["q"], cpu["k"], cpu["v"], cpu["offsets"], w.dims, w.window, qi,
                                  per_tap=True)
    assert_close("out", gather_rows(out, qi, N), r_out, tol)
    assert_close("lse", f64(lse).reshape(-1)[qi], r_lse, tol)
    r_dq, r_doff, r_dk, r_dv = oracle.backward(cpu["q"], cpu["k"], cpu["v"], cpu["offsets"], cpu["dout"],
                                               w.dims, w.window, qi, ki, per_tap=True)
    assert_close("dq", gather_rows(dq, qi, N), r_dq, tol)
    rows = torch.from_numpy(qi).to(doff.device)
    assert_close("doff", f64(doff.reshape(-1, w.K, 3)[rows]), r_doff, tol)
    assert_close("dk", gather_rows(dk, ki, N), r_dk, tol)
    assert_close("dv", gather_rows(dv, ki, N), r_dv, tol)
