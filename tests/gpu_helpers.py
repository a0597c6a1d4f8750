"""Shared helpers of the GPU parity tests: run the CUDA path through the C ABI binding and
compare with the CPU oracle on the same seeded inputs."""
from __future__ import annotations

import numpy as np
import torch

import oracle
from deformable_slide_attention_b200 import abi

TOL = {"f32": 1e-5, "bf16": 2e-2}


def to_cuda(inp):
    return {k: v.cuda().contiguous() for k, v in inp.items()}


def gpu_forward(d, dims, window):
    out, lse = abi.forward(d["q"], d["k"], d["v"], d["offsets"], dims, window)
    torch.cuda.synchronize()
    return out, lse


def gpu_backward(d, lse, dims, window):
    grads = abi.backward(d["q"], d["k"], d["v"], d["offsets"], lse, d["dout"], dims, window)
    torch.cuda.synchronize()
    return grads


def f64(t):
    return t.detach().float().cpu().double().numpy()


def items_of(heads, N, n_sample, seed, include_edges=True):
    """A seeded sample of h*N + n items, with each head's first and last tokens included."""
    g = np.random.default_rng(seed)
    items = set(g.integers(0, heads * N, size=n_sample).tolist())
    if include_edges:
        for h in range(heads):
            items.update([h * N, h * N + N - 1])
    return np.array(sorted(items), dtype=np.int64)


def edge_keys(dims, heads, seed, n_random=0):
    """Key items h*N + n on the edges the key-side kernels tile by, for each head in ``heads``:
    the first, second, middle and last two frames, the first and last rows, rows 3 and 4 (a
    4-row tile boundary) and the middle row, and the columns 0, 31, 32 (a 32-key tile boundary),
    the middle and the last -- every combination -- plus n_random seeded keys per head."""
    F, Hp, Wp = dims
    N = F * Hp * Wp
    pick = lambda vals, hi: sorted({min(max(v, 0), hi - 1) for v in vals})
    ts = pick([0, 1, F // 2, F - 2, F - 1], F)
    ys = pick([0, 3, 4, Hp // 2, Hp - 1], Hp)
    xs = pick([0, 31, 32, Wp // 2, Wp - 1], Wp)
    g = np.random.default_rng(seed)
    items = set()
    for h in heads:
        for t in ts:
            for y in ys:
                for x in xs:
                    items.add(h * N + (t * Hp + y) * Wp + x)
        items.update((h * N + g.integers(0, N, size=n_random)).tolist())
    return np.array(sorted(items), dtype=np.int64)


def gather_rows(t, items, N):
    """t [N][heads][dh] -> rows [len(items)][dh] for items h*N + n."""
    h, n = items // N, items % N
    return f64(t)[n, h]


def assert_close(name, got, ref, tol):
    got, ref = np.asarray(got, np.float64), np.asarray(ref, np.float64)
    assert got.shape == ref.shape, (name, got.shape, ref.shape)
    fin = np.isfinite(ref)
    assert np.array_equal(np.isfinite(got), fin), f"{name}: finiteness differs"
    err = np.abs(got[fin] - ref[fin]).max(initial=0.0)
    scale = np.abs(ref[fin]).max(initial=0.0)
    assert err <= tol, f"{name}: max-abs error {err:.3e} > {tol:.1e} (max |ref| {scale:.3g})"
    eq_inf = got[~fin] == ref[~fin]
    assert eq_inf.all(), f"{name}: non-finite entries differ"
    return err


def has_mma_path(d, dims, window):
    heads, dh = d["q"].shape[1], d["q"].shape[2]
    code = abi.DSA3D_BF16 if d["q"].dtype == torch.bfloat16 else abi.DSA3D_F32
    return abi.dsa3d_forward_workspace_bytes(*dims, heads, dh, *window, code) > 0


def full_parity(inp, dims, window, dtype, backward=True):
    """Element-by-element comparison of every output with the oracle.  Where the shape has a
    tensor-core forward, the general CUDA-core forward (no workspace) is checked as well."""
    tol = TOL[dtype]
    d = to_cuda(inp)
    out, lse = gpu_forward(d, dims, window)
    r_out, r_lse = oracle.full_forward(inp["q"], inp["k"], inp["v"], inp["offsets"], dims, window)
    errs = {"out": assert_close("out", f64(out), r_out, tol),
            "lse": assert_close("lse", f64(lse), r_lse, max(tol, 1e-5))}
    if has_mma_path(d, dims, window):
        out_cc, lse_cc = abi.forward(d["q"], d["k"], d["v"], d["offsets"], dims, window, workspace=None)
        torch.cuda.synchronize()
        errs["out_cc"] = assert_close("out (CUDA-core)", f64(out_cc), r_out, tol)
        errs["lse_cc"] = assert_close("lse (CUDA-core)", f64(lse_cc), r_lse, max(tol, 1e-5))
    if backward:
        dq, dk, dv, doff = gpu_backward(d, lse, dims, window)
        r = oracle.full_backward(inp["q"], inp["k"], inp["v"], inp["offsets"], inp["dout"], dims,
                                 window)
        for name, got, ref in (("dq", dq, r[0]), ("doff", doff, r[1]), ("dk", dk, r[2]),
                               ("dv", dv, r[3])):
            errs[name] = assert_close(name, f64(got), ref, tol)
    return errs
