"""Seeded synthetic inputs for 3D-DSA.

This module holds no arithmetic of the operator: it only draws random tensors.  Both the CUDA
path's tests and benchmark and the CPU oracle's tests take their inputs from here.

Workloads (draw order q, k, v, offsets, dO from one torch.Generator seeded per workload):

  tiny-f32         F=4,   8x8 grid   (N=256),       2 heads x dh 32,  window 3x3x3, fp32,
                   offsets U(-1.5, 1.5) per (head, token, axis), seed 0, forward only.
  small-bf16       F=16,  32x32 grid (N=16,384),    8 heads x dh 64,  window 3x7x7, bf16,
                   offsets N(0, 2^2) clamped so the window centre stays in the volume, then a
                   quarter of the (head, frame, 8x8 block) cells set to exactly zero offset
                   (chosen by seeded permutation), seed 1, forward.
  720p-bf16        F=32,  45x80 grid (N=115,200),   16 heads x dh 128, window 3x9x9, bf16,
                   offsets N(0, 3^2) unclamped, seed 2, forward.
  720p-train-bf16  as 720p-bf16 plus dO ~ N(0,1), seed 3, forward (saving lse) + backward.
  1080p-long-bf16  F=256, 68x120 grid (N=2,088,960), 32 heads x dh 128, window 3x9x9, bf16,
                   offsets per (head, axis) = A sin(2 pi (kt t/F + ky y/Hp + kx x/Wp) + phi)
                   + N(0, 0.5^2) with kt, ky, kx in {1, 2} and phi ~ U(0, 2 pi) drawn per
                   (head, axis), A = sqrt(2 * 15.75) so the total std is 4; seed 4; forward +
                   backward.  Generated on the device (its tensors are 17 GB each).
  720p-train-taps-bf16  the 720p-train-bf16 shapes with per-tap offsets: one offset 3-vector per
                   (head, token, window tap), [heads][N][243][3] (5.4 GB), each component
                   N(0, 3^2) unclamped like the per-token 720p offsets; dO ~ N(0,1); seed 5;
                   forward + backward.  Generated on the device.

q, k, v and dO are N(0,1), rounded to bf16 (round to nearest even) for the bf16 workloads.
Layouts: q/k/v/dO [N][heads][dh]; offsets [heads][N][3] fp32 in (dt, dy, dx) order, or
[heads][N][K][3] (K = kt*kh*kw, tap order u, v, w with w fastest) for per-tap workloads.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    F: int
    Hp: int
    Wp: int
    heads: int
    dh: int
    window: tuple
    dtype: str  # "f32" or "bf16"
    seed: int
    offsets: str  # "uniform", "normal_clamped_zero_blocks", "normal", "smooth"
    scale: float = 0.0  # offset range / std
    backward: bool = False
    device_generated: bool = False
    per_tap: bool = False  # offsets per (head, token, tap) instead of per (head, token)
    extra: dict = field(default_factory=dict)

    @property
    def dims(self):
        return (self.F, self.Hp, self.Wp)

    @property
    def N(self):
        return self.F * self.Hp * self.Wp

    @property
    def K(self):
        return self.window[0] * self.window[1] * self.window[2]

    @property
    def torch_dtype(self):
        return torch.float32 if self.dtype == "f32" else torch.bfloat16


WORKLOADS = [
    Workload("tiny-f32", 4, 8, 8, 2, 32, (3, 3, 3), "f32", 0, "uniform", 1.5),
    Workload("small-bf16", 16, 32, 32, 8, 64, (3, 7, 7), "bf16", 1, "normal_clamped_zero_blocks", 2.0),
    Workload("720p-bf16", 32, 45, 80, 16, 128, (3, 9, 9), "bf16", 2, "normal", 3.0),
    Workload("720p-train-bf16", 32, 45, 80, 16, 128, (3, 9, 9), "bf16", 3, "normal", 3.0, backward=True),
    Workload("1080p-long-bf16", 256, 68, 120, 32, 128, (3, 9, 9), "bf16", 4, "smooth", 4.0,
             backward=True, device_generated=True),
    Workload("720p-train-taps-bf16", 32, 45, 80, 16, 128, (3, 9, 9), "bf16", 5, "normal", 3.0,
             backward=True, device_generated=True, per_tap=True),
]
BY_NAME = {w.name: w for w in WORKLOADS}


def _normal(shape, gen, device, dtype):
    x = torch.empty(shape, dtype=torch.float32, device=device)
    x.normal_(0.0, 1.0, generator=gen)
    return x.to(dtype)


def _fill_normal_chunked(t: torch.Tensor, gen, chunk: int = 1 << 28):
    """Fill a (possibly huge) tensor with N(0,1) in fixed-size chunks (deterministic per seed)."""
    flat = t.view(-1)
    for s in range(0, flat.numel(), chunk):
        part = flat[s:s + chunk]
        tmp = torch.empty(part.numel(), dtype=torch.float32, device=t.device)
        tmp.normal_(0.0, 1.0, generator=gen)
        part.copy_(tmp)
        del tmp


def _coords(F, Hp, Wp, device):
    n = torch.arange(F * Hp * Wp, device=device)
    x = n % Wp
    y = (n // Wp) % Hp
    t = n // (Wp * Hp)
    return t, y, x


def _offset_shape(heads, N, taps):
    return (heads, N, 3) if taps is None else (heads, N, taps, 3)


def offsets_uniform(gen, heads, N, half_range, device="cpu", taps=None):
    u = torch.empty(_offset_shape(heads, N, taps), dtype=torch.float32, device=device)
    u.uniform_(-half_range, half_range, generator=gen)
    return u


def offsets_normal(gen, heads, N, std, device="cpu", taps=None):
    o = torch.empty(_offset_shape(heads, N, taps), dtype=torch.float32, device=device)
    o.normal_(0.0, std, generator=gen)
    return o


def offsets_normal_clamped_zero_blocks(gen, F, Hp, Wp, heads, std, block=8, zero_frac=0.25):
    N = F * Hp * Wp
    o = offsets_normal(gen, heads, N, std)
    t, y, x = _coords(F, Hp, Wp, "cpu")
    lo = torch.stack([-t, -y, -x], dim=-1).float()
    hi = torch.stack([F - 1 - t, Hp - 1 - y, Wp - 1 - x], dim=-1).float()
    o = torch.maximum(torch.minimum(o, hi[None]), lo[None])
    by, bx = (Hp + block - 1) // block, (Wp + block - 1) // block
    cells = heads * F * by * bx
    n_zero = int(math.floor(zero_frac * cells))
    chosen = torch.randperm(cells, generator=gen)[:n_zero]
    cell_of_token = ((t * by + y // block) * bx + x // block)  # [N], per head offset below
    mask = torch.zeros(cells, dtype=torch.bool)
    mask[chosen] = True
    mask = mask.view(heads, F * by * bx)[:, cell_of_token]
    o[mask] = 0.0
    return o.contiguous()


def offsets_smooth(gen, F, Hp, Wp, heads, total_std=4.0, noise_std=0.5, device="cpu"):
    """Per-(head, axis) low-frequency 3-D sinusoid plus white noise; total std = total_std."""
    N = F * Hp * Wp
    amp = math.sqrt(2.0 * (total_std ** 2 - noise_std ** 2))
    freq = torch.randint(1, 3, (heads, 3, 3), generator=gen, device=device).float()  # [h][axis][kt,ky,kx]
    phase = torch.empty((heads, 3), dtype=torch.float32, device=device)
    phase.uniform_(0.0, 2.0 * math.pi, generator=gen)
    t, y, x = _coords(F, Hp, Wp, device)
    tf, yf, xf = t.float() / F, y.float() / Hp, x.float() / Wp
    o = torch.empty((heads, N, 3), dtype=torch.float32, device=device)
    for h in range(heads):
        for a in range(3):
            arg = 2.0 * math.pi * (freq[h, a, 0] * tf + freq[h, a, 1] * yf + freq[h, a, 2] * xf) + phase[h, a]
            o[h, :, a] = amp * torch.sin(arg)
    noise = torch.empty_like(o)
    noise.normal_(0.0, noise_std, generator=gen)
    o += noise
    return o


def make(w: Workload, device="cpu", with_dout=None):
    """Draw one workload's inputs: dict(q, k, v, offsets[, dout]) on ``device``.

    CPU-generated workloads are drawn on the CPU and then moved; device-generated ones (the
    1080p workload) are drawn directly on ``device`` (which must then be a CUDA device).
    """
    with_dout = w.backward if with_dout is None else with_dout
    gen_device = device if w.device_generated else "cpu"
    gen = torch.Generator(device=gen_device)
    gen.manual_seed(w.seed)
    N, shape = w.N, (w.N, w.heads, w.dh)
    out = {}
    if w.device_generated:
        for name in ("q", "k", "v"):
            t = torch.empty(shape, dtype=w.torch_dtype, device=device)
            _fill_normal_chunked(t, gen)
            out[name] = t
    else:
        for name in ("q", "k", "v"):
            out[name] = _normal(shape, gen, "cpu", w.torch_dtype)
    taps = w.K if w.per_tap else None
    if w.offsets == "uniform":
        off = offsets_uniform(gen, w.heads, N, w.scale, gen_device, taps)
    elif w.offsets == "normal":
        off = offsets_normal(gen, w.heads, N, w.scale, gen_device, taps)
    elif w.per_tap:
        raise ValueError(f"per-tap offsets are drawn uniform or normal, not {w.offsets}")
    elif w.offsets == "normal_clamped_zero_blocks":
        off = offsets_normal_clamped_zero_blocks(gen, w.F, w.Hp, w.Wp, w.heads, w.scale)
    elif w.offsets == "smooth":
        off = offsets_smooth(gen, w.F, w.Hp, w.Wp, w.heads, w.scale, device=gen_device)
    else:
        raise ValueError(w.offsets)
    out["offsets"] = off.contiguous()
    if with_dout:
        if w.device_generated:
            t = torch.empty(shape, dtype=w.torch_dtype, device=device)
            _fill_normal_chunked(t, gen)
            out["dout"] = t
        else:
            out["dout"] = _normal(shape, gen, "cpu", w.torch_dtype)
    if not w.device_generated and str(device) != "cpu":
        out = {k: v.to(device) for k, v in out.items()}
    return out


def custom(F, Hp, Wp, heads, dh, window, dtype="f32", seed=0, offsets="uniform", scale=1.5,
           with_dout=True, per_tap=False):
    """A small ad-hoc workload (CPU tensors) for tests; same draw order as the named ones."""
    w = Workload(f"custom-{F}x{Hp}x{Wp}", F, Hp, Wp, heads, dh, tuple(window), dtype, seed, offsets,
                 scale, backward=with_dout, per_tap=per_tap)
    return w, make(w, "cpu", with_dout)
