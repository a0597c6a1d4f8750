"""GPU parity of the DWConv3D term of Eq. 1 (dsa3d_dwconv3d / dsa3d_dwconv3d_backward) against
the oracle's depthwise convolution (reading R9), through the C ABI.

Weights are scaled by 1/sqrt(kt kh kw) so outputs are O(1); tolerances max-abs 1e-5 (fp32) and
2e-2 (bf16 I/O, fp32 accumulation); dweight and dbias (fp32 sums over every token) relative 1e-4.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from deformable_slide_attention_b200 import abi
from tests.gpu_helpers import TOL, assert_close, f64

pytestmark = [pytest.mark.gpu, pytest.mark.usefixtures("gpu_lib", "oracle_lib")]

CASES = [((3, 5, 6), 4, (3, 3, 3)), ((2, 7, 19), 6, (3, 5, 9)), ((4, 3, 11), 2, (1, 1, 15)),
         ((1, 4, 9), 8, (1, 3, 1)), ((5, 2, 17), 4, (5, 3, 7)), ((4, 9, 16), 64, (3, 9, 9)),
         # the forward's staged kernel over two runs of units with a last channel group of one pair,
         # the strip-pair kernel (C a multiple of 32) over five groups, with a ragged last strip pair
         # and at k_w = 15, and a 405-tap kernel past the staged limit (global kernel)
         ((4, 7, 40), 66, (3, 5, 9)), ((3, 5, 6), 160, (3, 3, 3)), ((4, 9, 21), 64, (3, 9, 9)),
         ((2, 7, 40), 32, (1, 5, 15)), ((3, 5, 12), 4, (5, 9, 9))]


def _problem(dims, C, window, dtype, seed):
    g = torch.Generator().manual_seed(seed)
    N, K = math.prod(dims), math.prod(window)
    x = torch.randn(N, C, generator=g).to(dtype)
    w = torch.randn(C, *window, generator=g) / math.sqrt(K)
    b = torch.randn(C, generator=g)
    add = torch.randn(N, C, generator=g).to(dtype)
    dy = torch.randn(N, C, generator=g).to(dtype)
    return x, w, b, add, dy


@pytest.mark.parametrize("dims,C,window", CASES)
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_forward_with_and_without_add(dims, C, window, dtype):
    td = torch.float32 if dtype == "f32" else torch.bfloat16
    x, w, b, add, _ = _problem(dims, C, window, td, sum(dims) + C)
    dx, dw_, db_, dadd = (t.cuda() for t in (x, w, b, add))
    y = abi.dwconv3d(dx, dw_, db_, dims)
    y_add = abi.dwconv3d(dx, dw_, db_, dims, add=dadd)
    inplace = dadd.clone()
    abi.dwconv3d(dx, dw_, db_, dims, add=inplace, out=inplace)  # y = conv + add, in place
    torch.cuda.synchronize()
    ref = oracle.dwconv3d(x, w, b, dims)
    assert_close("y", f64(y), ref, TOL[dtype])
    assert_close("y+add", f64(y_add), ref + f64(add), TOL[dtype])
    assert torch.equal(inplace, y_add)


@pytest.mark.parametrize("dims,C,window", CASES)
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_backward(dims, C, window, dtype):
    td = torch.float32 if dtype == "f32" else torch.bfloat16
    x, w, _, _, dy = _problem(dims, C, window, td, 3 * sum(dims) + C)
    gx, gw, gb = abi.dwconv3d_backward(x.cuda(), w.cuda(), dy.cuda(), dims)
    torch.cuda.synchronize()
    rx, rw, rb = oracle.dwconv3d_backward(x, w, dy.double().numpy(), dims)
    assert_close("dx", f64(gx), rx, TOL[dtype])
    for name, got, ref in (("dweight", gw, rw), ("dbias", gb, rb)):
        err = np.abs(f64(got) - ref).max()
        assert err <= 1e-4 * max(1.0, np.abs(ref).max()), (name, err)


def test_rejects_unsupported_and_overlapping():
    x = torch.zeros(24, 4, device="cuda", dtype=torch.bfloat16)
    w = torch.zeros(4, 1, 1, 17, device="cuda")
    y = torch.empty_like(x)
    st = torch.cuda.current_stream().cuda_stream
    assert abi.dsa3d_dwconv3d(x.data_ptr(), w.data_ptr(), None, None, y.data_ptr(), 1, 1, 24, 4, 1, 1,
                              17, abi.DSA3D_BF16, st) == 2  # kw > 15
    w3 = torch.zeros(4, 1, 1, 3, device="cuda")
    assert abi.dsa3d_dwconv3d(x.data_ptr(), w3.data_ptr(), None, None, x.data_ptr(), 1, 1, 24, 4, 1, 1,
                              3, abi.DSA3D_BF16, st) == 1  # y on top of x
    x3 = torch.zeros(24, 3, device="cuda", dtype=torch.bfloat16)
    assert abi.dsa3d_dwconv3d(x3.data_ptr(), w3.data_ptr(), None, None, y.data_ptr(), 1, 1, 24, 3, 1, 1,
                              3, abi.DSA3D_BF16, st) == 2  # odd channel count


@pytest.mark.parametrize("per_tap", [False, True])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_offset_network_forward(per_tap, dtype):
    """dsa3d_offset_head against oracle.offset_head (relative 1e-4: fp32 throughout), and the
    offsets it writes drive the attention exactly as the same offsets given by hand."""
    td = torch.float32 if dtype == "f32" else torch.bfloat16
    dims, heads, dh, window = (3, 5, 9), 2, 32, (3, 3, 3)  # dh 32: the smallest the attention takes
    C, N, K = heads * dh, math.prod(dims), math.prod(window)
    g = torch.Generator().manual_seed(77 + int(per_tap))
    x = torch.randn(N, C, generator=g).to(td)
    dw_w, dw_b = torch.randn(C, *window, generator=g) / math.sqrt(K), torch.randn(C, generator=g)
    width = heads * 3 * (K if per_tap else 1)
    pw_w, pw_b = torch.randn(C, width, generator=g) * 0.3, torch.randn(width, generator=g)
    off = abi.offset_head(x.cuda(), dw_w.cuda(), dw_b.cuda(), pw_w.cuda(), pw_b.cuda(), dims, heads,
                          per_tap=per_tap)
    torch.cuda.synchronize()
    ref = oracle.offset_head(x, dw_w, dw_b, pw_w, pw_b, dims, heads, K if per_tap else None)
    err = np.abs(f64(off) - ref).max()
    assert err <= 1e-4 * max(1.0, np.abs(ref).max()), err
    q, k, v = (torch.randn(N, heads, dh, generator=g).to(td).cuda() for _ in range(3))
    fwd = abi.forward_taps if per_tap else abi.forward
    out1, lse1 = fwd(q, k, v, off, dims, window)
    out2, lse2 = fwd(q, k, v, off.clone(), dims, window)
    torch.cuda.synchronize()
    assert torch.equal(out1, out2) and torch.equal(lse1, lse2)


@pytest.mark.parametrize("per_tap", [False, True])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_offset_network_backward(per_tap, dtype):
    """dsa3d_offset_head_backward against oracle.offset_head_backward: dx (the I/O tolerance) and
    the fp32 weight gradients (relative 1e-4)."""
    td = torch.float32 if dtype == "f32" else torch.bfloat16
    dims, heads, dh, window = (3, 5, 9), 2, 32, (3, 3, 3)  # dh 32: the smallest the attention takes
    C, N, K = heads * dh, math.prod(dims), math.prod(window)
    g = torch.Generator().manual_seed(91 + int(per_tap))
    x = torch.randn(N, C, generator=g).to(td)
    dw_w, dw_b = torch.randn(C, *window, generator=g) / math.sqrt(K), torch.randn(C, generator=g)
    width = heads * 3 * (K if per_tap else 1)
    pw_w = torch.randn(C, width, generator=g) / math.sqrt(C)
    doff = torch.randn((heads, N, K, 3) if per_tap else (heads, N, 3), generator=g) / math.sqrt(width)
    got = abi.offset_head_backward(x.cuda(), dw_w.cuda(), dw_b.cuda(), pw_w.cuda(), doff.cuda(), dims,
                                   heads, per_tap=per_tap)
    torch.cuda.synchronize()
    ref = oracle.offset_head_backward(x, dw_w, dw_b, pw_w, doff.double().numpy(), dims)
    assert_close("dx", f64(got[0]), ref[0], TOL[dtype])
    for name, a, b in zip(("d dw_weight", "d dw_bias", "d pw_weight", "d pw_bias"), got[1:], ref[1:]):
        err = np.abs(f64(a) - b).max()
        assert err <= 1e-4 * max(1.0, np.abs(b).max()), (name, err)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_layer_against_the_oracle_chain(dtype):
    """layer.forward / backward (offset network, attention, fused convolution) against the oracle's
    parts composed the same way, with the GPU's offsets fed to the oracle's attention (so that a
    floor decision near an integer cannot differ between the two)."""
    from deformable_slide_attention_b200 import layer
    td = torch.float32 if dtype == "f32" else torch.bfloat16
    dims, heads, dh, window = (3, 5, 9), 2, 32, (3, 3, 3)  # dh 32: the smallest the attention takes
    C, N, K = heads * dh, math.prod(dims), math.prod(window)
    g = torch.Generator().manual_seed(123)
    x = torch.randn(N, C, generator=g).to(td)
    q, k, v, dout = (torch.randn(N, heads, dh, generator=g).to(td) for _ in range(4))
    w = [torch.randn(C, *window, generator=g) / math.sqrt(K), torch.randn(C, generator=g),
         torch.randn(C, *window, generator=g) / math.sqrt(K), torch.randn(C, generator=g),
         torch.randn(C, heads * 3, generator=g) / math.sqrt(C), torch.randn(heads * 3, generator=g)]
    wts = layer.LayerWeights(*(t.cuda() for t in w))
    out, ctx = layer.forward(x.cuda(), q.cuda(), k.cuda(), v.cuda(), wts, dims, window)
    grads = layer.backward(ctx, dout.cuda())
    torch.cuda.synchronize()
    off = ctx[4].float().cpu()
    r_att, _ = oracle.full_forward(q, k, v, off, dims, window)
    r_out = r_att + oracle.dwconv3d(x, w[0], w[1], dims).reshape(N, heads, dh)
    assert_close("out", f64(out), r_out, 2 * TOL[dtype])  # attention and sum each rounded once
    r_dq, r_doff, r_dk, r_dv = oracle.full_backward(q, k, v, off, dout, dims, window)
    r_dx = (oracle.offset_head_backward(x, w[2], w[3], w[4], r_doff, dims)[0] +
            oracle.dwconv3d_backward(x, w[0], dout.double().numpy().reshape(N, C), dims)[0])
    assert_close("dx", f64(grads["x"]), r_dx, 2 * TOL[dtype])
    assert_close("dq", f64(grads["q"]), r_dq, TOL[dtype])


@pytest.mark.parametrize("name", ["720p-train-bf16", "1080p-long-bf16"])
def test_full_size_sampled_channels(name):
    """At a workload's full size, in the launch configuration bench.py times (C = heads x dh
    channels, the window's kernel, y += conv(x) in place, then the backward): every output of
    four channel pairs -- the first, the two on either side of the staged kernel's 64-channel
    group boundary, and the last -- against the oracle run on those channels alone (depthwise: a
    channel's outputs depend on that channel only).  bf16 outputs: |got - ref| <= 2^-8 |ref| +
    1e-4 (half an ulp of the rounding, plus the fp32 sum); dweight, dbias: 1e-4 of the largest."""
    from deformable_slide_attention_b200 import inputs
    w = inputs.BY_NAME[name]
    dev = torch.device("cuda", 0)
    C, N, K = w.heads * w.dh, w.N, w.K
    gen = torch.Generator(device=dev)
    gen.manual_seed(w.seed)
    x, y, dy = (torch.empty((N, C), dtype=w.torch_dtype, device=dev) for _ in range(3))
    for t in (x, y, dy):
        inputs._fill_normal_chunked(t, gen)
    weight = torch.empty((C, *w.window), dtype=torch.float32, device=dev)
    weight.normal_(0.0, 1.0 / math.sqrt(K), generator=gen)
    bias = torch.empty(C, dtype=torch.float32, device=dev).normal_(0.0, 1.0, generator=gen)
    pairs = [0, 31, 32, C // 2 - 1]
    add = {p: f64(y[:, 2 * p:2 * p + 2]) for p in pairs}
    abi.dwconv3d(x, weight, bias, w.dims, add=y, out=y)
    gx, gw, gb = abi.dwconv3d_backward(x, weight, dy, w.dims)
    torch.cuda.synchronize()
    try:
        for p in pairs:
            sl = slice(2 * p, 2 * p + 2)
            xs, ws, bs = x[:, sl].cpu(), weight[sl].cpu(), bias[sl].cpu()
            ref_y = oracle.dwconv3d(xs, ws, bs, w.dims) + add[p]
            rx, rw, rb = oracle.dwconv3d_backward(xs, ws, f64(dy[:, sl]), w.dims)
            for nm, got, ref in (("y", f64(y[:, sl]), ref_y), ("dx", f64(gx[:, sl]), rx)):
                err = np.abs(got - ref) - 2.0 ** -8 * np.abs(ref)
                assert err.max() <= 1e-4, (name, p, nm, float(err.max()))
            for nm, got, ref in (("dweight", f64(gw[sl]), rw), ("dbias", f64(gb[sl]), rb)):
                err = np.abs(got - ref).max()
                assert err <= 1e-4 * max(1.0, np.abs(ref).max()), (name, p, nm, err)
    finally:
        del x, y, dy, gx, gw, gb
        torch.cuda.empty_cache()


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_forward_kernels_agree_bit_for_bit(dtype):
    """The strip-pair kernel (C a multiple of 32) and the staged kernel (other channel counts) add
    the same products in the same order (kernel planes, then kernel rows, then taps, each output's
    sum starting from its bias), so a channel's outputs do not depend on which one ran: channels
    0..63 of a 66-channel problem (staged kernel) equal the 64-channel problem made of them
    (strip-pair kernel) exactly, for the forward with the add and for dX."""
    td = torch.float32 if dtype == "f32" else torch.bfloat16
    dims, window = (4, 9, 21), (3, 9, 9)
    x, w, b, add, dy = _problem(dims, 66, window, td, 66)
    sub = lambda t: t[:, :64].contiguous()
    y66 = abi.dwconv3d(x.cuda(), w.cuda(), b.cuda(), dims, add=add.cuda())
    y64 = abi.dwconv3d(sub(x).cuda(), w[:64].contiguous().cuda(), b[:64].contiguous().cuda(), dims,
                       add=sub(add).cuda())
    gx66, _, _ = abi.dwconv3d_backward(x.cuda(), w.cuda(), dy.cuda(), dims)
    gx64, _, _ = abi.dwconv3d_backward(sub(x).cuda(), w[:64].contiguous().cuda(), sub(dy).cuda(), dims)
    torch.cuda.synchronize()
    assert torch.equal(y66[:, :64], y64)
    assert torch.equal(gx66[:, :64], gx64)
