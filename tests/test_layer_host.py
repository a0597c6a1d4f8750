"""deformable_slide_attention_b200.layer orders the library's calls for Eq. 1's layer: on the CPU,
with stand-in operations that record the calls, the forward runs the offset network, the
attention and the fused convolution add, and the backward sums the offset network's and the
convolution's parts of dX."""
import types

import torch

from deformable_slide_attention_b200 import layer

N, H, DH = 12, 2, 4
C = H * DH


def _ops(log):
    def offset_head(x, dw, db, pw, pb, dims, heads, per_tap=False):
        log.append("offset_head")
        return torch.full((heads, x.shape[0], 3), 0.5)

    def forward(q, k, v, off, dims, window):
        log.append("forward")
        return q * 2.0, torch.zeros(q.shape[1], q.shape[0])

    def dwconv3d(x, w, b, dims, add=None, out=None):
        log.append("dwconv3d")
        out += x * 10.0  # stand-in for conv(x), added in place
        return out

    def backward(q, k, v, off, lse, dout, dims, window):
        log.append("backward")
        return dout * 2.0, dout * 3.0, dout * 4.0, torch.ones_like(off)

    def offset_head_backward(x, dw, db, pw, doff, dims, heads, per_tap=False):
        log.append("offset_head_backward")
        return torch.full_like(x, 1.0), dw * 0, db * 0, pw * 0, torch.zeros(pw.shape[1])

    def dwconv3d_backward(x, w, dy, dims):
        log.append("dwconv3d_backward")
        return dy * 10.0, w * 0, torch.zeros(x.shape[1])

    return types.SimpleNamespace(**{f.__name__: f for f in (
        offset_head, forward, dwconv3d, backward, offset_head_backward, dwconv3d_backward)},
        forward_taps=forward, backward_taps=backward)


def test_layer_orders_the_calls_and_sums_dx():
    log = []
    ops = _ops(log)
    g = torch.Generator().manual_seed(0)
    x = torch.randn(N, C, generator=g)
    q, k, v, dout = (torch.randn(N, H, DH, generator=g) for _ in range(4))
    wts = layer.LayerWeights(torch.zeros(C, 1, 3, 3), torch.zeros(C), torch.zeros(C, 1, 3, 3),
                             torch.zeros(C), torch.zeros(C, H * 3), torch.zeros(H * 3))
    out, ctx = layer.forward(x, q, k, v, wts, (1, 3, 4), (1, 3, 3), ops=ops)
    assert log == ["offset_head", "forward", "dwconv3d"]
    assert torch.equal(out, q * 2.0 + (x * 10.0).view(N, H, DH))  # attention + conv, in place
    grads = layer.backward(ctx, dout, ops=ops)
    assert log[3:] == ["backward", "offset_head_backward", "dwconv3d_backward"]
    assert torch.equal(grads["x"], 1.0 + dout.view(N, C) * 10.0)  # offset network + convolution
    assert torch.equal(grads["q"], dout * 2.0) and torch.equal(grads["v"], dout * 4.0)
    assert set(grads) == {"x", "q", "k", "v", "offsets", "conv_weight", "conv_bias", "off_dw_weight",
                          "off_dw_bias", "off_pw_weight", "off_pw_bias"}
