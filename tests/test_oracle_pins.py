"""Pins of the CPU oracle against what the paper and the mathematics fix (no GPU needed).

Paper: MegaSlide-DiT (arXiv 2607.22696), 3D-DSA definition (Eq. 1 and its softmax), the
fixed-window ablation (zero offsets reduce 3D-DSA to fixed local attention with kernel
(k_t,k_h,k_w)), the implementation paragraph (trilinear sampling = grid_sample, bilinear, 5-D) and
the complexity statement (O(N k_t k_h k_w), linear in N).

Each pin is chosen so that a plausible mistake in the oracle fails at least one of them:
  P1 full-volume window, zero offsets == brute-force softmax attention  (mask, softmax, scale use)
  P2 zero offsets, any window == dense attention with a centred box mask   (window geometry)
  P3 integer offsets == dense attention with a shifted box mask; samples bit-equal to K rows
  P4 constant V gives out == V (valid queries) and 0 / -inf (queries with no valid tap)
  P5 per-tap trilinear samples and their derivative == torch grid_sample (+ autograd)
  P6 central finite differences of the whole forward == the oracle backward
  P7 torch float64 autograd of a grid_sample restatement == the oracle backward
  P8 invariants: sum dV = sum dO over valid queries, sum dK = 0, out inside the box hull of V,
     lse >= max tap score
  P9 work counter scales linearly in N
  P10 heads are independent; permuting heads permutes the result
Per-tap offsets (the paper's offset tensor with one 3-vector per window tap, reading R8):
  P11 every tap carrying the query's offset == the per-token oracle (exactly); the per-tap offset
      gradients sum to the per-token one
  P12 torch float64 autograd of the grid_sample restatement with per-tap offsets == the oracle
  P13 central finite differences along single taps' offsets == the per-tap offset gradient
  P14 a tap with a non-finite offset is masked alone (== the same tap moved out of the volume)
"""
import math

import numpy as np
import pytest
import torch

import oracle
from deformable_slide_attention_b200 import inputs
from tests import torch_restatement as tr

pytestmark = pytest.mark.usefixtures("oracle_lib")


def box_mask(dims, window, int_off=None):
    """mask[h][n][j]: key j lies in query n's (shifted) window; int_off [H][N][3] integer offsets."""
    c = tr.token_coords(dims)
    r = torch.tensor([(k - 1) // 2 for k in window], dtype=torch.float64)
    centre = c[None] if int_off is None else c[None] + int_off
    d = (c[None, None, :, :] - centre[:, :, None, :]).abs()
    return (d <= r).all(-1)


def run_oracle(inp, dims, window):
    out, lse = oracle.full_forward(inp["q"], inp["k"], inp["v"], inp["offsets"], dims, window)
    return torch.from_numpy(out), torch.from_numpy(lse)


def as64(x):
    return x.double() if isinstance(x, torch.Tensor) else torch.from_numpy(x).double()


# ---------------------------------------------------------------------------------------------
@pytest.mark.parametrize("dims,dtype", [((2, 3, 4), "f32"), ((3, 2, 5), "bf16"), ((1, 4, 3), "f32")])
def test_p1_full_window_equals_dense_attention(dims, dtype):
    window = tuple(2 * d - 1 for d in dims)
    _, inp = inputs.custom(*dims, 3, 8, window, dtype, seed=11, with_dout=False)
    inp["offsets"].zero_()
    out, lse = run_oracle(inp, dims, window)
    H, N = 3, math.prod(dims)
    mask = torch.ones(H, N, N, dtype=torch.bool)
    ref_out, ref_lse = tr.dense_masked_attention(as64(inp["q"]), as64(inp["k"]), as64(inp["v"]), mask)
    assert torch.allclose(out, ref_out, atol=1e-12, rtol=0)
    assert torch.allclose(lse, ref_lse, atol=1e-12, rtol=0)


@pytest.mark.parametrize("window", [(1, 3, 3), (3, 3, 5), (3, 5, 1), (5, 1, 3)])
def test_p2_zero_offsets_equal_local_box_attention(window):
    dims = (4, 5, 6)
    _, inp = inputs.custom(*dims, 2, 16, window, "f32", seed=12, with_dout=False)
    inp["offsets"].zero_()
    out, lse = run_oracle(inp, dims, window)
    mask = box_mask(dims, window).expand(2, -1, -1)
    ref_out, ref_lse = tr.dense_masked_attention(as64(inp["q"]), as64(inp["k"]), as64(inp["v"]), mask)
    assert torch.allclose(out, ref_out, atol=1e-12, rtol=0)
    assert torch.allclose(lse, ref_lse, atol=1e-12, rtol=0)


def test_p3_integer_offsets_equal_shifted_gather():
    dims, window = (5, 6, 7), (3, 3, 3)
    _, inp = inputs.custom(*dims, 2, 8, window, "bf16", seed=13, with_dout=False)
    g = torch.Generator().manual_seed(5)
    int_off = torch.randint(-3, 4, (2, math.prod(dims), 3), generator=g).float()
    inp["offsets"] = int_off
    out, lse = run_oracle(inp, dims, window)
    mask = box_mask(dims, window, int_off.double())
    ref_out, ref_lse = tr.dense_masked_attention(as64(inp["q"]), as64(inp["k"]), as64(inp["v"]), mask)
    fin = torch.isfinite(ref_lse)
    assert (torch.isfinite(lse) == fin).all()
    assert torch.allclose(out, ref_out, atol=1e-12, rtol=0)
    assert torch.allclose(lse[fin], ref_lse[fin], atol=1e-12, rtol=0)
    # each valid tap's sample is exactly the key row at the shifted position
    kf = inp["k"].float().double()
    Hp, Wp = dims[1], dims[2]
    for (h, n, tau) in [(0, 0, 13), (1, 100, 0), (0, 150, 26), (1, 77, 5), (0, 209, 20)]:
        valid, base, frac, samp, _ = oracle.tap(inp["k"], int_off, dims, window, h, n, tau)
        assert np.all(frac == 0.0)
        if valid:
            j = (base[0] * Hp + base[1]) * Wp + base[2]
            assert np.array_equal(samp, kf[j, h].numpy())


def test_p4_constant_values_give_constant_output():
    dims, window = (4, 6, 6), (3, 3, 3)
    _, inp = inputs.custom(*dims, 2, 8, window, "f32", seed=14, offsets="normal", scale=3.0,
                           with_dout=False)
    c = torch.linspace(-2.0, 3.0, 8)
    inp["v"] = c.expand(math.prod(dims), 2, 8).contiguous()
    out, lse = run_oracle(inp, dims, window)
    fin = torch.isfinite(lse)  # [H][N]
    assert fin.any() and (~fin).any(), "the draw should include queries with no valid tap"
    finq = fin.t()  # [N][H]
    assert torch.allclose(out[finq], c.double().expand(int(finq.sum()), 8), atol=1e-12, rtol=0)
    assert (out[~finq] == 0).all()
    assert (lse[~fin] == float("-inf")).all()


def test_p5_samples_match_grid_sample():
    dims, window = (4, 5, 6), (3, 3, 3)
    F, Hp, Wp = dims
    _, inp = inputs.custom(*dims, 2, 8, window, "bf16", seed=15, scale=1.5, with_dout=False)
    k64 = as64(inp["k"].float())
    g = torch.Generator().manual_seed(3)
    checked = 0
    for _ in range(200):
        h = int(torch.randint(0, 2, (1,), generator=g))
        n = int(torch.randint(0, math.prod(dims), (1,), generator=g))
        tau = int(torch.randint(0, 27, (1,), generator=g))
        valid, base, frac, samp, dsamp = oracle.tap(inp["k"], inp["offsets"], dims, window, h, n, tau)
        p = tr.token_coords(dims)[n]
        uvw = tr.tap_offsets(window)[tau]
        exact = p + uvw + inp["offsets"][h, n].double()
        decoded = torch.from_numpy(base).double() + torch.from_numpy(frac).double()
        assert torch.all((decoded - exact).abs() <= 2.0 ** -23)  # single-precision decode
        assert np.all((frac >= 0) & (frac < 1))
        ext = torch.tensor([F - 1, Hp - 1, Wp - 1], dtype=torch.float64)
        assert valid == bool(((decoded >= 0) & (decoded <= ext)).all())
        if not valid:
            continue
        pos = decoded.clone().requires_grad_(True)
        gn = 2.0 * pos / ext - 1.0
        grid = torch.stack([gn[2], gn[1], gn[0]]).view(1, 1, 1, 1, 3)
        vol = k64[:, h, :].t().reshape(1, 8, F, Hp, Wp)
        ref = torch.nn.functional.grid_sample(vol, grid, mode="bilinear", padding_mode="zeros",
                                              align_corners=True).view(8)
        assert np.allclose(samp, ref.detach().numpy(), atol=1e-12, rtol=0)
        # derivative along each axis (at a fractional point): d sample_e / d pos_a
        if np.all((frac > 1e-3) & (frac < 1 - 1e-3)):
            for e in range(8):
                (gr,) = torch.autograd.grad(ref[e], pos, retain_graph=True)
                assert np.allclose(dsamp[:, e], gr.numpy(), atol=1e-12, rtol=0)
        checked += 1
    assert checked > 50


def _fd_problem(seed, dtype_scale=2 ** -12):
    """Small fp32 problem whose inputs and offsets are coarse binary fractions, so that every
    +-eps perturbation below is exact in fp32 and the offset decode stays exact."""
    dims, window = (3, 4, 5), (3, 3, 3)
    H, dh = 2, 4
    N = math.prod(dims)
    g = torch.Generator().manual_seed(seed)
    q, k, v, do = (torch.round(torch.randn(N, H, dh, generator=g) / dtype_scale) * dtype_scale
                   for _ in range(4))
    off = torch.empty(H, N, 3).uniform_(-1.4, 1.4, generator=g)
    frac = off - off.floor()
    off = torch.where(frac < 0.01, off + 0.02, off)
    off = torch.where(frac > 0.99, off - 0.02, off)
    off = torch.round(off * 1024) / 1024
    return dims, window, q.float(), k.float(), v.float(), do.float(), off.float()


def _loss(q, k, v, off, do, dims, window):
    out, _ = oracle.full_forward(q, k, v, off, dims, window)
    return float((out * do.double().numpy()).sum())


def test_p6_finite_differences():
    dims, window, q, k, v, do, off = _fd_problem(21)
    N, H, dh = q.shape
    dq, doff, dk, dv = oracle.full_backward(q, k, v, off, do, dims, window)
    g = torch.Generator().manual_seed(4)
    eps = 2.0 ** -12
    for name, tensor, grad in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        for _ in range(6):
            n = int(torch.randint(0, N, (1,), generator=g))
            h = int(torch.randint(0, H, (1,), generator=g))
            e = int(torch.randint(0, dh, (1,), generator=g))
            args = {"q": q, "k": k, "v": v}
            plus = {kk: vv.clone() for kk, vv in args.items()}
            minus = {kk: vv.clone() for kk, vv in args.items()}
            plus[name][n, h, e] += eps
            minus[name][n, h, e] -= eps
            fd = (_loss(plus["q"], plus["k"], plus["v"], off, do, dims, window)
                  - _loss(minus["q"], minus["k"], minus["v"], off, do, dims, window)) / (2 * eps)
            an = grad[n, h, e]
            assert abs(fd - an) <= 1e-6 * max(1.0, abs(an)), (name, n, h, e, fd, an)
    eps = 2.0 ** -14
    for _ in range(8):
        n = int(torch.randint(0, N, (1,), generator=g))
        h = int(torch.randint(0, H, (1,), generator=g))
        a = int(torch.randint(0, 3, (1,), generator=g))
        op, om = off.clone(), off.clone()
        op[h, n, a] += eps
        om[h, n, a] -= eps
        fd = (_loss(q, k, v, op, do, dims, window) - _loss(q, k, v, om, do, dims, window)) / (2 * eps)
        an = doff[h, n, a]
        assert abs(fd - an) <= 1e-6 * max(1.0, abs(an)), ("offsets", n, h, a, fd, an)


def test_p7_matches_torch_autograd_restatement():
    dims, window, q, k, v, do, off = _fd_problem(22)
    q64, k64, v64, off64 = (x.double().clone().requires_grad_(True) for x in (q, k, v, off))
    out, lse = tr.dsa3d(q64, k64, v64, off64, dims, window)
    (out * do.double()).sum().backward()
    o_out, o_lse = run_oracle({"q": q, "k": k, "v": v, "offsets": off}, dims, window)
    assert torch.allclose(o_out, out.detach(), atol=1e-12, rtol=0)
    fin = torch.isfinite(lse)
    assert torch.equal(torch.isfinite(o_lse), fin)
    assert torch.allclose(o_lse[fin], lse.detach()[fin], atol=1e-12, rtol=0)
    dq, doff, dk, dv = oracle.full_backward(q, k, v, off, do, dims, window)
    for name, a, b in (("dq", dq, q64.grad), ("dk", dk, k64.grad), ("dv", dv, v64.grad),
                       ("doff", doff, off64.grad)):
        assert np.allclose(a, b.numpy(), atol=1e-10, rtol=0), name


def test_p8_invariants():
    dims, window = (4, 5, 6), (3, 3, 3)
    _, inp = inputs.custom(*dims, 2, 8, window, "f32", seed=16, scale=1.5, with_dout=True)
    q, k, v, off, do = (inp[n] for n in ("q", "k", "v", "offsets", "dout"))
    out, lse = oracle.full_forward(q, k, v, off, dims, window)
    dq, doff, dk, dv = oracle.full_backward(q, k, v, off, do, dims, window)
    fin = np.isfinite(lse).T  # [N][H]
    do64 = do.double().numpy()
    for h in range(2):
        assert np.allclose(dv[:, h].sum(0), do64[fin[:, h], h].sum(0), atol=1e-10)
        assert np.allclose(dk[:, h].sum(0), 0.0, atol=1e-10)
    # out inside the per-dimension hull of V over the query's corner tokens; lse >= max score
    v64 = v.double().numpy()
    N = math.prod(dims)
    for h in range(2):
        for n in range(0, N, 7):
            if not fin[n, h]:
                continue
            toks, smax = [], -np.inf
            for tau in range(27):
                valid, base, frac, samp, _ = oracle.tap(k, off, dims, window, h, n, tau)
                if not valid:
                    continue
                smax = max(smax, float(samp @ q[n, h].double().numpy()) / math.sqrt(8))
                for c in range(8):
                    b = base + np.array([(c >> 2) & 1, (c >> 1) & 1, c & 1])
                    if np.all(b < np.array(dims)):
                        toks.append((b[0] * dims[1] + b[1]) * dims[2] + b[2])
            vals = v64[toks, h]
            assert np.all(out[n, h] >= vals.min(0) - 1e-12) and np.all(out[n, h] <= vals.max(0) + 1e-12)
            assert lse[h, n] >= smax - 1e-12


def test_p9_linear_cost():
    reads = []
    for F in (8, 16, 32):
        dims = (F, 6, 6)
        _, inp = inputs.custom(*dims, 1, 4, (3, 3, 3), "f32", seed=17, with_dout=False)
        _, _, r = oracle.forward(inp["q"], inp["k"], inp["v"], inp["offsets"], dims, (3, 3, 3),
                                 return_reads=True)
        assert r <= math.prod(dims) * 27 * 8 * 2
        reads.append(r)
    assert abs(reads[1] / reads[0] - 2) < 0.2 and abs(reads[2] / reads[1] - 2) < 0.2


def test_p10_heads_independent_and_permutable():
    dims, window = (3, 4, 5), (3, 3, 3)
    _, inp = inputs.custom(*dims, 3, 8, window, "bf16", seed=18, with_dout=True)
    q, k, v, off, do = (inp[n] for n in ("q", "k", "v", "offsets", "dout"))
    out, lse = oracle.full_forward(q, k, v, off, dims, window)
    dq, doff, dk, dv = oracle.full_backward(q, k, v, off, do, dims, window)
    perm = [2, 0, 1]
    out_p, lse_p = oracle.full_forward(q[:, perm], k[:, perm], v[:, perm], off[perm], dims, window)
    assert np.array_equal(out_p, out[:, perm]) and np.array_equal(lse_p, lse[perm])
    gp = oracle.full_backward(q[:, perm], k[:, perm], v[:, perm], off[perm], do[:, perm], dims, window)
    assert np.array_equal(gp[0], dq[:, perm]) and np.array_equal(gp[1], doff[perm])
    assert np.array_equal(gp[2], dk[:, perm]) and np.array_equal(gp[3], dv[:, perm])
    h = 1
    one = oracle.full_forward(q[:, h:h + 1].contiguous(), k[:, h:h + 1].contiguous(),
                              v[:, h:h + 1].contiguous(), off[h:h + 1].contiguous(), dims, window)
    assert np.array_equal(one[0][:, 0], out[:, h]) and np.array_equal(one[1][0], lse[h])


def test_closed_form_two_valid_taps():
    """Hand-derived case: 1x1x3 volume, dh = 2, window 1x1x3, query x=1 with dx = 0.5.
    Taps sample x = 0.5, 1.5 (x = 2.5 leaves the volume and is masked)."""
    dims, window = (1, 1, 3), (1, 1, 3)
    q = torch.tensor([[[0.0, 0.0]], [[1.0, 0.0]], [[0.0, 0.0]]])  # only token 1 queries
    k = torch.tensor([[[0.0, 5.0]], [[2.0, -1.0]], [[4.0, 3.0]]])
    v = torch.tensor([[[1.0, 0.0]], [[0.0, 1.0]], [[1.0, 1.0]]])
    off = torch.zeros(1, 3, 3)
    off[0, 1, 2] = 0.5
    out, lse = oracle.forward(q, k, v, off, dims, window, items=[1])
    s1, s2 = 1.0 / math.sqrt(2), 3.0 / math.sqrt(2)  # q.k~ = 0.5*0+0.5*2, 0.5*2+0.5*4
    a1, a2 = math.exp(s1) / (math.exp(s1) + math.exp(s2)), math.exp(s2) / (math.exp(s1) + math.exp(s2))
    expect = np.array([0.5 * a1 + 0.5 * a2, 0.5 * a1 + 1.0 * a2])  # v~ = (0.5,0.5), (0.5,1)
    assert np.allclose(out[0], expect, atol=1e-14, rtol=0)
    assert abs(lse[0] - math.log(math.exp(s1) + math.exp(s2))) < 1e-14


def test_invalid_offsets_make_query_invalid():
    dims, window = (2, 3, 3), (1, 3, 3)
    _, inp = inputs.custom(*dims, 1, 4, window, "f32", seed=19, with_dout=True)
    off = inp["offsets"].clone()
    off[0, 0, 1] = float("nan")
    off[0, 1, 0] = float("inf")
    off[0, 2, 2] = 2.0 ** 25
    out, lse = oracle.forward(inp["q"], inp["k"], inp["v"], off, dims, window, items=[0, 1, 2, 3])
    assert np.all(out[:3] == 0) and np.all(lse[:3] == -np.inf)
    dq, doff, _, _ = oracle.backward(inp["q"], inp["k"], inp["v"], off, inp["dout"], dims, window,
                                     q_items=[0, 1, 2], k_items=[])
    assert np.all(dq == 0) and np.all(doff == 0)


def test_fraction_carry_rule():
    """A tiny negative offset whose fractional part rounds to 1.0f carries into the integer part."""
    dims, window = (1, 1, 4), (1, 1, 1)
    k = torch.arange(4, dtype=torch.float32).view(4, 1, 1)
    off = torch.zeros(1, 4, 3)
    off[0, 2, 2] = -2.0 ** -30  # floor = -1, 1 - 2^-30 rounds to 1.0f -> i = 0, f = 0
    valid, base, frac, samp, _ = oracle.tap(k, off, dims, window, 0, 2, 0)
    assert valid and base[2] == 2 and frac[2] == 0.0 and samp[0] == 2.0


def test_golden_regression_snapshot():
    """The oracle still reproduces its committed snapshot (tests/golden/make_golden.py)."""
    import json
    import os
    from tests.golden.make_golden import ITEMS
    rec = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "tiny_f32.json")))
    w = inputs.BY_NAME["tiny-f32"]
    inp = inputs.make(w, "cpu", with_dout=True)
    out, lse = oracle.forward(inp["q"], inp["k"], inp["v"], inp["offsets"], w.dims, w.window, ITEMS)
    dq, doff, dk, dv = oracle.backward(inp["q"], inp["k"], inp["v"], inp["offsets"], inp["dout"],
                                       w.dims, w.window, ITEMS, ITEMS)
    for name, got in (("out", out), ("lse", lse), ("dq", dq), ("doff", doff), ("dk", dk), ("dv", dv)):
        assert np.allclose(got, np.array(rec[name]), atol=1e-12, rtol=0), name


# ---------------------------------------------------------------------------------------------
# per-tap offsets (R8)
def _taps_problem(seed):
    """The P6/P7 problem with one offset per window tap: coarse binary fractions away from integers,
    so the finite differences below stay exact and never cross a cell or a box face."""
    dims, window, q, k, v, do, _ = _fd_problem(seed)
    H, N, K = q.shape[1], q.shape[0], math.prod(window)
    g = torch.Generator().manual_seed(seed + 1000)
    off = torch.empty(H, N, K, 3).uniform_(-1.4, 1.4, generator=g)
    frac = off - off.floor()
    off = torch.where(frac < 0.01, off + 0.02, off)
    off = torch.where(frac > 0.99, off - 0.02, off)
    off = (torch.round(off * 1024) / 1024).float()
    return dims, window, q, k, v, do, off


def _loss_taps(q, k, v, off, do, dims, window):
    out, _ = oracle.full_forward(q, k, v, off, dims, window, per_tap=True)
    return float((out * do.double().numpy()).sum())


def test_p11_shared_tap_offsets_equal_per_token():
    dims, window, q, k, v, do, off = _fd_problem(31)
    K = math.prod(window)
    taps = off[:, :, None, :].expand(-1, -1, K, -1).contiguous()
    o1, l1 = oracle.full_forward(q, k, v, off, dims, window)
    o2, l2 = oracle.full_forward(q, k, v, taps, dims, window, per_tap=True)
    assert np.array_equal(o1, o2) and np.array_equal(l1, l2)
    g1 = oracle.full_backward(q, k, v, off, do, dims, window)
    g2 = oracle.full_backward(q, k, v, taps, do, dims, window, per_tap=True)
    for name, a, b in (("dq", g1[0], g2[0]), ("dk", g1[2], g2[2]), ("dv", g1[3], g2[3])):
        assert np.array_equal(a, b), name
    assert g2[1].shape == off.shape[:2] + (K, 3)
    assert np.allclose(g2[1].sum(axis=2), g1[1], atol=1e-12, rtol=0)


def test_p12_per_tap_matches_torch_autograd_restatement():
    dims, window, q, k, v, do, off = _taps_problem(32)
    q64, k64, v64, off64 = (x.double().clone().requires_grad_(True) for x in (q, k, v, off))
    out, lse = tr.dsa3d(q64, k64, v64, off64, dims, window)
    (out * do.double()).sum().backward()
    o_out, o_lse = oracle.full_forward(q, k, v, off, dims, window, per_tap=True)
    assert np.allclose(o_out, out.detach().numpy(), atol=1e-12, rtol=0)
    fin = torch.isfinite(lse).numpy()
    assert np.array_equal(np.isfinite(o_lse), fin)
    assert np.allclose(o_lse[fin], lse.detach().numpy()[fin], atol=1e-12, rtol=0)
    dq, doff, dk, dv = oracle.full_backward(q, k, v, off, do, dims, window, per_tap=True)
    for name, a, b in (("dq", dq, q64.grad), ("dk", dk, k64.grad), ("dv", dv, v64.grad),
                       ("doff", doff, off64.grad)):
        assert np.allclose(a, b.numpy(), atol=1e-10, rtol=0), name


def test_p13_per_tap_finite_differences():
    dims, window, q, k, v, do, off = _taps_problem(33)
    H, N, K = off.shape[0], off.shape[1], off.shape[2]
    _, doff, _, _ = oracle.full_backward(q, k, v, off, do, dims, window, per_tap=True)
    g = torch.Generator().manual_seed(5)
    eps = 2.0 ** -14
    checked = 0
    for _ in range(48):
        h, n = int(torch.randint(0, H, (1,), generator=g)), int(torch.randint(0, N, (1,), generator=g))
        tau, a = int(torch.randint(0, K, (1,), generator=g)), int(torch.randint(0, 3, (1,), generator=g))
        op, om = off.clone(), off.clone()
        op[h, n, tau, a] += eps
        om[h, n, tau, a] -= eps
        fd = (_loss_taps(q, k, v, op, do, dims, window) - _loss_taps(q, k, v, om, do, dims, window)) / (2 * eps)
        an = doff[h, n, tau, a]
        assert abs(fd - an) <= 1e-6 * max(1.0, abs(an)), (h, n, tau, a, fd, an)
        checked += an != 0.0
    assert checked >= 8  # enough of the sampled taps lie inside the small volume


def test_p14_non_finite_tap_offset_masks_that_tap_only():
    dims, window, q, k, v, _, off = _taps_problem(34)
    K = off.shape[2]
    o_ref, l_ref = oracle.forward(q, k, v, off, dims, window, items=np.array([7]), per_tap=True)
    bad, far = off.clone(), off.clone()
    # a tap of query 7 (head 0) whose sample position lies inside the volume
    pos = tr.token_coords(dims)[7][None] + tr.tap_offsets(window) + off[0, 7].double()
    ext = torch.tensor([d - 1 for d in dims], dtype=torch.float64)
    inside = ((pos >= 0) & (pos <= ext)).all(-1)
    assert inside.sum() >= 2
    tau0 = int(torch.nonzero(inside)[0])
    bad[0, 7, tau0] = float("nan")
    far[0, 7, tau0, 0] = 1.0e6
    o_bad, l_bad = oracle.forward(q, k, v, bad, dims, window, items=np.array([7]), per_tap=True)
    o_far, l_far = oracle.forward(q, k, v, far, dims, window, items=np.array([7]), per_tap=True)
    assert np.isfinite(l_bad).all()
    assert np.array_equal(o_bad, o_far) and np.array_equal(l_bad, l_far)
    assert not np.array_equal(o_bad, o_ref)
