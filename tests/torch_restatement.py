"""An independent restatement of 3D-DSA in plain torch (CPU, float64), used only to pin the oracle.

It follows the paper's own description of the implementation (MegaSlide-DiT, arXiv 2607.22696,
the paragraph after the 3D-DSA definition): trilinear sampling by ``F.grid_sample`` in bilinear
mode on 5-D tensors, here with ``align_corners=True`` and zero padding, then a softmax over the
window taps (Eq. 1 and the softmax that follows it), with out-of-volume taps masked.  Gradients
come from torch autograd, so this route shares nothing with the oracle's hand-written backward.
"""
from __future__ import annotations

import math

import torch
import torch.nn.functional as Fn


def tap_offsets(window):
    kt, kh, kw = window
    r = [(k - 1) // 2 for k in window]
    u = torch.arange(kt) - r[0]
    v = torch.arange(kh) - r[1]
    w = torch.arange(kw) - r[2]
    U, V, W = torch.meshgrid(u, v, w, indexing="ij")
    return torch.stack([U, V, W], dim=-1).reshape(-1, 3).double()  # [K][3], u outermost


def token_coords(dims):
    F, Hp, Wp = dims
    n = torch.arange(F * Hp * Wp)
    return torch.stack([n // (Hp * Wp), (n // Wp) % Hp, n % Wp], dim=-1).double()  # [N][3]


def dsa3d(q, k, v, off, dims, window):
    """q, k, v: [N][H][dh] float64; off: [H][N][3] float64 (one offset per query), or [H][N][K][3]
    (one per window tap).  Returns out [N][H][dh], lse [H][N]."""
    F, Hp, Wp = dims
    N, H, dh = q.shape
    assert min(dims) >= 2, "grid_sample normalisation needs every extent >= 2"
    per_tap = off if off.dim() == 4 else off[:, :, None, :]
    pos = token_coords(dims)[None, :, None, :] + tap_offsets(window)[None, None] + per_tap
    ext = torch.tensor([F - 1, Hp - 1, Wp - 1], dtype=torch.float64)
    valid = ((pos >= 0) & (pos <= ext)).all(-1)  # [H][N][K]
    g = 2.0 * pos / ext - 1.0
    grid = torch.stack([g[..., 2], g[..., 1], g[..., 0]], dim=-1).unsqueeze(-2)  # [H][N][K][1][3]

    def sample(src):
        vol = src.permute(1, 2, 0).reshape(H, dh, F, Hp, Wp)
        s = Fn.grid_sample(vol, grid, mode="bilinear", padding_mode="zeros", align_corners=True)
        return s[..., 0].permute(0, 2, 3, 1)  # [H][N][K][dh]

    ks, vs = sample(k), sample(v)
    qh = q.permute(1, 0, 2)  # [H][N][dh]
    s = (qh[:, :, None, :] * ks).sum(-1) / math.sqrt(dh)
    s = s.masked_fill(~valid, float("-inf"))
    lse = torch.logsumexp(s, dim=-1)
    any_valid = valid.any(-1)
    safe_lse = torch.where(any_valid, lse, torch.zeros_like(lse))
    p = torch.where(valid, torch.exp(s - safe_lse[..., None]), torch.zeros_like(s))
    out = (p[..., None] * vs).sum(-2)
    return out.permute(1, 0, 2), lse


def dense_masked_attention(q, k, v, mask):
    """Brute-force attention over all N tokens with a boolean mask [H][N][N] (query, key)."""
    N, H, dh = q.shape
    qh, kh, vh = (x.permute(1, 0, 2) for x in (q, k, v))
    s = qh @ kh.transpose(1, 2) / math.sqrt(dh)
    s = s.masked_fill(~mask, float("-inf"))
    lse = torch.logsumexp(s, dim=-1)
    any_valid = mask.any(-1)
    safe = torch.where(any_valid, lse, torch.zeros_like(lse))
    p = torch.where(mask, torch.exp(s - safe[..., None]), torch.zeros_like(s))
    return (p @ vh).permute(1, 0, 2), lse
