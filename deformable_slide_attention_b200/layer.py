"""The 3D-DSA layer of MegaSlide-DiT (arXiv 2607.22696, the 3D-DSA definition, Eq. 1) composed
from the library's calls:

    offsets = OffsetNet(X)                           (depthwise conv + pointwise layer)
    out     = DWConv3D(X) + Attention(q, k, v, offsets)

forward() returns out [N][heads][dh] and a context; backward() takes dO and returns the
gradients with respect to X (the offset network's and the convolution's parts, summed), q, k, v
and every weight.  q, k and v come from the caller (the paper's W_q, W_k, W_v projections of X,
like the layer norm and residual around the operator, are outside the operator), so their
gradients are returned for the caller to carry back through those projections.  Every step runs
in the library's CUDA kernels; this module only orders the calls and adds the two dX parts.
"""
from __future__ import annotations

import dataclasses

from . import abi


@dataclasses.dataclass
class LayerWeights:
    """fp32 weights: conv_weight [C][kt][kh][kw] and conv_bias [C] (the DWConv3D term);
    off_dw_weight [C][kt][kh][kw], off_dw_bias [C], off_pw_weight [C][heads*(K)*3] and
    off_pw_bias [heads*(K)*3] (the offset network; K = kt*kh*kw with per-tap offsets)."""
    conv_weight: object
    conv_bias: object
    off_dw_weight: object
    off_dw_bias: object
    off_pw_weight: object
    off_pw_bias: object


def forward(x, q, k, v, wts: LayerWeights, dims, window, per_tap=False, ops=abi):
    """x [N][C] with C = heads*dh; q, k, v [N][heads][dh].  Returns (out [N][heads][dh], ctx)."""
    heads = q.shape[1]
    offsets = ops.offset_head(x, wts.off_dw_weight, wts.off_dw_bias, wts.off_pw_weight,
                              wts.off_pw_bias, dims, heads, per_tap=per_tap)
    fwd = ops.forward_taps if per_tap else ops.forward
    out, lse = fwd(q, k, v, offsets, dims, window)
    flat = out.view(out.shape[0], -1)
    ops.dwconv3d(x, wts.conv_weight, wts.conv_bias, dims, add=flat, out=flat)  # out += DWConv3D(x)
    return out, (x, q, k, v, offsets, lse, wts, tuple(dims), tuple(window), per_tap)


def backward(ctx, dout, ops=abi):
    """dout [N][heads][dh] -> dict of gradients: x, q, k, v, conv_weight, conv_bias,
    off_dw_weight, off_dw_bias, off_pw_weight, off_pw_bias (and offsets, the attention's)."""
    x, q, k, v, offsets, lse, wts, dims, window, per_tap = ctx
    heads = q.shape[1]
    bwd = ops.backward_taps if per_tap else ops.backward
    dq, dk, dv, doff = bwd(q, k, v, offsets, lse, dout, dims, window)
    dx_off, d_odw, d_odb, d_opw, d_opb = ops.offset_head_backward(
        x, wts.off_dw_weight, wts.off_dw_bias, wts.off_pw_weight, doff, dims, heads, per_tap=per_tap)
    dx_conv, d_cw, d_cb = ops.dwconv3d_backward(x, wts.conv_weight, dout.view(dout.shape[0], -1), dims)
    dx = (dx_off.float() + dx_conv.float()).to(x.dtype)
    return {"x": dx, "q": dq, "k": dk, "v": dv, "offsets": doff, "conv_weight": d_cw,
            "conv_bias": d_cb, "off_dw_weight": d_odw, "off_dw_bias": d_odb,
            "off_pw_weight": d_opw, "off_pw_bias": d_opb}
