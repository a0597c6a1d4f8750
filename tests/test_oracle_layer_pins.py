"""Pins of the oracle's other two parts of the 3D-DSA layer (MegaSlide-DiT, the 3D-DSA
definition, Eq. 1): the DWConv3D term (reading R9) and the offset network (R10).

They are checked against what fixes them independently of the oracle:
- P15: PyTorch's conv3d with groups = C and padding k // 2 (the paper's implementation names
  nn.Conv3d with groups = hidden size), in fp64, for fp32 and bf16 inputs;
- P16: closed forms: a centred delta kernel is the identity plus the bias, an off-centre delta is
  a shift with zero fill, an all-ones kernel on an all-ones input counts the in-volume window;
- P17: the backward equals torch autograd, and is the adjoint of the (linear) forward in x and
  in the kernel;
- P18: the offset network equals torch's conv3d followed by a linear layer, in the attention's
  offset layout (per token and per tap), and its backward equals torch autograd;
- P19: the chain rule through the whole layer: for
  L(X) = sum dO . (DWConv3D(X) + attention(q, k, v, offsets(X))), the sum of the conv backward
  and the offset network's backward of the attention's offset gradient equals central finite
  differences of L along a random direction.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from deformable_slide_attention_b200 import inputs

pytestmark = pytest.mark.usefixtures("oracle_lib")


def _problem(dims, C, window, seed, dtype=torch.float32):
    g = torch.Generator().manual_seed(seed)
    N = math.prod(dims)
    x = torch.randn(N, C, generator=g).to(dtype)
    w = torch.randn(C, *window, generator=g)
    b = torch.randn(C, generator=g)
    return x, w, b


def _torch_conv(x, w, b, dims):
    """Reference: torch conv3d on [1][C][F][Hp][Wp] in fp64; returns [N][C]."""
    N, C = x.shape
    xt = x.double().T.reshape(1, C, *dims)
    pad = tuple(k // 2 for k in w.shape[1:])
    y = torch.nn.functional.conv3d(xt, w.double().unsqueeze(1), None if b is None else b.double(),
                                   padding=pad, groups=C)
    return y.reshape(C, N).T


@pytest.mark.parametrize("dims,window", [((3, 5, 6), (3, 3, 3)), ((4, 6, 7), (1, 3, 5)),
                                         ((2, 7, 9), (3, 5, 7)), ((1, 4, 5), (1, 1, 1)),
                                         ((5, 3, 4), (5, 3, 1))])
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_p15_dwconv3d_equals_torch_conv3d(dims, window, dtype):
    x, w, b = _problem(dims, 5, window, 1 + sum(window), dtype)
    for bias in (b, None):
        y = oracle.dwconv3d(x, w, bias, dims)
        ref = _torch_conv(x.float(), w, bias, dims).numpy()
        assert np.abs(y - ref).max() <= 1e-12 * max(1.0, np.abs(ref).max())


def test_p16_closed_forms():
    dims, C, window = (3, 4, 5), 3, (3, 3, 5)
    F, Hp, Wp = dims
    x, _, b = _problem(dims, C, window, 7)
    xv = x.double().numpy().reshape(F, Hp, Wp, C)
    # centred delta: identity plus bias
    w = torch.zeros(C, *window)
    w[:, 1, 1, 2] = 1.0
    y = oracle.dwconv3d(x, w, b, dims).reshape(F, Hp, Wp, C)
    assert np.array_equal(y, xv + b.double().numpy())
    # delta at (u, v, w) = (2, 0, 4): y(t, y, x) = X(t + 1, y - 1, x + 2), zero outside
    w = torch.zeros(C, *window)
    w[:, 2, 0, 4] = 1.0
    y = oracle.dwconv3d(x, w, None, dims).reshape(F, Hp, Wp, C)
    ref = np.zeros_like(xv)
    ref[:F - 1, 1:, :Wp - 2] = xv[1:, :Hp - 1, 2:]
    assert np.array_equal(y, ref)
    # all-ones kernel on an all-ones input: the number of in-volume window positions
    ones = torch.ones(math.prod(dims), C)
    y = oracle.dwconv3d(ones, torch.ones(C, *window), None, dims).reshape(F, Hp, Wp, C)
    cnt = lambda D, k, p: min(p + k // 2, D - 1) - max(p - k // 2, 0) + 1
    for t in range(F):
        for yy in range(Hp):
            for xx in range(Wp):
                want = cnt(F, 3, t) * cnt(Hp, 3, yy) * cnt(Wp, 5, xx)
                assert (y[t, yy, xx] == want).all()


@pytest.mark.parametrize("dims,window", [((3, 5, 6), (3, 3, 3)), ((2, 6, 7), (1, 5, 3))])
def test_p17_dwconv3d_backward(dims, window):
    C = 4
    x, w, b = _problem(dims, C, window, 11)
    g = torch.Generator().manual_seed(12)
    dy = torch.randn(math.prod(dims), C, generator=g, dtype=torch.float64)
    dx, dw, db = oracle.dwconv3d_backward(x, w, dy.numpy(), dims)
    xt, wt, bt = (t.double().clone().requires_grad_(True) for t in (x, w, b))
    (_torch_conv(xt, wt, bt, dims) * dy).sum().backward()
    assert np.abs(dx - xt.grad.numpy()).max() < 1e-12
    assert np.abs(dw - wt.grad.numpy()).max() < 1e-11
    assert np.abs(db - bt.grad.numpy()).max() < 1e-11
    # the forward is linear in x and in w: the backward is its adjoint,
    # <dy, conv_w(d)> = <dx, d> and <dy, conv_e(x)> = <dw, e>, the forward applied to d (or with
    # kernel e) without bias
    d = torch.randn(x.shape, generator=g)
    lhs = (oracle.dwconv3d(d, w, None, dims) * dy.numpy()).sum()
    assert abs(lhs - (dx * d.double().numpy()).sum()) < 1e-12 * max(1.0, abs(lhs))
    ew = torch.randn(w.shape, generator=g)
    lhs = (oracle.dwconv3d(x, ew, None, dims) * dy.numpy()).sum()
    assert abs(lhs - (dw * ew.double().numpy()).sum()) < 1e-12 * max(1.0, abs(lhs))


def _head_params(C, heads, window, taps, seed):
    g = torch.Generator().manual_seed(seed)
    width = heads * 3 * (taps or 1)
    return (torch.randn(C, *window, generator=g), torch.randn(C, generator=g),
            torch.randn(C, width, generator=g) * 0.3, torch.randn(width, generator=g))


@pytest.mark.parametrize("taps", [None, 27])
def test_p18_offset_network_equals_torch(taps):
    dims, heads, dh, window = (3, 4, 5), 2, 4, (3, 3, 3)
    C = heads * dh
    x, _, _ = _problem(dims, C, window, 21)
    dw_w, dw_b, pw_w, pw_b = _head_params(C, heads, window, taps, 22)
    off = oracle.offset_head(x, dw_w, dw_b, pw_w, pw_b, dims, heads, taps)
    N = math.prod(dims)
    # torch: conv3d (groups = C) then a linear layer, then the attention's layout
    xt, a, bb, pw, pb = (t.double().clone().requires_grad_(True) for t in (x, dw_w, dw_b, pw_w, pw_b))
    flat = _torch_conv(xt, a, bb, dims) @ pw + pb
    ref = flat.reshape(N, heads, 3) if taps is None else flat.reshape(N, heads, taps, 3)
    ref = ref.transpose(0, 1)
    assert off.shape == tuple(ref.shape)
    assert np.abs(off - ref.detach().numpy()).max() < 1e-11
    # element (h, n, a) is output channel h*3 + a (per token) or (h*K + tau)*3 + a (per tap)
    n, h = 17, 1
    z = _torch_conv(x, dw_w, dw_b, dims)[n]
    ch = h * 3 + 2 if taps is None else (h * taps + 5) * 3 + 2
    want = float(z @ pw_w[:, ch].double() + pw_b[ch])
    got = off[h, n, 2] if taps is None else off[h, n, 5, 2]
    assert abs(got - want) < 1e-11
    g = torch.Generator().manual_seed(23)
    doff = torch.randn(ref.shape, generator=g, dtype=torch.float64)
    (ref * doff).sum().backward()
    grads = oracle.offset_head_backward(x, dw_w, dw_b, pw_w, doff.numpy(), dims)
    for got, t in zip(grads, (xt, a, bb, pw, pb)):
        assert np.abs(got - t.grad.numpy()).max() < 1e-10


def _dyadic(shape, gen, step, lim):
    """Random multiples of step in [-lim, lim] (exact in fp32)."""
    return torch.round((torch.rand(shape, generator=gen) * 2 - 1) * lim / step) * step


@pytest.mark.parametrize("taps", [False, True])
def test_p19_chain_rule_through_the_layer(taps):
    """L(X) = sum dO . (DWConv3D(X) + attention(q, k, v, offset_head(X))); dL/dX assembled from
    the three oracle backwards equals central differences of L in single entries of X.

    X and the weights lie on dyadic grids (X in steps of 2^-4, kernels 2^-4, pointwise weights
    2^-6), so every offset is an exact fp32 number (the attention decodes it without rounding),
    and the step 2^-8 keeps them exact; the test checks that no offset the step moves crosses an
    integer, where the derivative (mask and integer part held fixed) does not apply."""
    dims, heads, dh, window = (3, 5, 6), 2, 8, (3, 3, 3)
    C, N, K = heads * dh, math.prod(dims), math.prod(window)
    T = K if taps else None
    _, inp = inputs.custom(*dims, heads, dh, window, "f32", seed=31)
    q, k, v, dout = inp["q"], inp["k"], inp["v"], inp["dout"]
    gen = torch.Generator().manual_seed(32)
    x = _dyadic((N, C), gen, 2.0 ** -4, 2.0)
    cw, cb = _dyadic((C, *window), gen, 2.0 ** -4, 1.0), _dyadic((C,), gen, 2.0 ** -4, 1.0)
    dw_w, dw_b = _dyadic((C, *window), gen, 2.0 ** -4, 1.0), _dyadic((C,), gen, 2.0 ** -4, 1.0)
    width = heads * 3 * (K if taps else 1)
    pw_w, pw_b = _dyadic((C, width), gen, 2.0 ** -6, 0.125), _dyadic((width,), gen, 2.0 ** -4, 2.0)

    def offsets(xx):
        off = oracle.offset_head(xx, dw_w, dw_b, pw_w, pw_b, dims, heads, T)
        assert np.array_equal(off, off.astype(np.float32))  # exact in fp32
        return off

    def layer(xx, with_conv=True):
        off = torch.from_numpy(offsets(xx)).float()
        out, _ = oracle.full_forward(q, k, v, off, dims, window, per_tap=taps)
        conv = oracle.dwconv3d(xx, cw, cb, dims) if with_conv else 0.0
        return float((dout.double().numpy().reshape(N, C) * (conv + out.reshape(N, C))).sum())

    off32 = torch.from_numpy(offsets(x)).float()
    _, doff, _, _ = oracle.full_backward(q, k, v, off32, dout, dims, window, per_tap=taps)
    dx_conv, _, _ = oracle.dwconv3d_backward(x, cw, dout.double().numpy().reshape(N, C), dims)
    dx_off = oracle.offset_head_backward(x, dw_w, dw_b, pw_w, doff, dims)[0]
    grad = dx_conv + dx_off
    e = 2.0 ** -8
    checked = 0
    for n0, c0 in ((40, 3), (47, 12), (61, 7), (29, 0), (55, 15)):
        lo, hi = x.clone(), x.clone()
        lo[n0, c0] -= e
        hi[n0, c0] += e
        if not np.array_equal(np.floor(offsets(lo)), np.floor(offsets(hi))):
            continue  # the step crosses an integer part
        fd = (layer(hi) - layer(lo)) / (2 * e)
        assert abs(fd - grad[n0, c0]) <= 1e-4 + 1e-3 * abs(grad[n0, c0]), (n0, c0, fd, grad[n0, c0])
        # the attention term alone, through the offsets
        fd = (layer(hi, False) - layer(lo, False)) / (2 * e)
        assert abs(fd - dx_off[n0, c0]) <= 1e-4 + 1e-3 * abs(dx_off[n0, c0]), (n0, c0, fd)
        checked += 1
    assert checked >= 3
