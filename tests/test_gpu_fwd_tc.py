"""The tcgen05 forward (tensor-memory accumulators, TMA tiles) against the oracle, against the
mma.sync forward it replaces, and across its tile geometries.

DSA3D_FWD_KERNEL=mma selects the mma.sync forward (the library reads it at every call);
DSA3D_TC_RY sets the bucket rows per tile of the tcgen05 forward.  Each query's arithmetic does not
depend on the tile it falls in (its lane, its pass, the tile's union rows only add exact zeros),
so every tile geometry must give bit-equal results.
"""
import os

import pytest
import torch

import oracle
from deformable_slide_attention_b200 import abi, inputs
from tests.gpu_helpers import TOL, assert_close, f64, to_cuda

pytestmark = [pytest.mark.gpu, pytest.mark.usefixtures("gpu_lib", "oracle_lib")]

CASES = [((3, 7, 9), 3, 64, (3, 5, 5), 2.5),
         ((5, 10, 11), 2, 128, (3, 9, 9), 3.0),
         ((4, 12, 20), 2, 64, (3, 7, 7), 4.0),
         ((6, 9, 33), 2, 128, (1, 3, 15), 2.0),
         ((2, 5, 40), 1, 64, (3, 1, 1), 1.5)]


class _env:
    def __init__(self, **kv):
        self.kv = kv

    def __enter__(self):
        self.old = {k: os.environ.get(k) for k in self.kv}
        os.environ.update({k: str(v) for k, v in self.kv.items()})

    def __exit__(self, *exc):
        for k, v in self.old.items():
            if v is None:
                os.environ.pop(k, None)
            else:
                os.environ[k] = v


def _fwd(d, dims, window):
    out, lse = abi.forward(d["q"], d["k"], d["v"], d["offsets"], dims, window)
    torch.cuda.synchronize()
    return out, lse


@pytest.mark.parametrize("case", range(len(CASES)))
def test_tc_and_mma_forwards_match_the_oracle(case):
    dims, heads, dh, window, scale = CASES[case]
    _, inp = inputs.custom(*dims, heads, dh, window, "bf16", seed=500 + case, scale=scale)
    d = to_cuda(inp)
    r_out, r_lse = oracle.full_forward(inp["q"], inp["k"], inp["v"], inp["offsets"], dims, window)
    tol = TOL["bf16"]
    out, lse = _fwd(d, dims, window)
    assert_close("out (tcgen05)", f64(out), r_out, tol)
    assert_close("lse (tcgen05)", f64(lse), r_lse, tol)
    with _env(DSA3D_FWD_KERNEL="mma"):
        out_m, lse_m = _fwd(d, dims, window)
    assert_close("out (mma.sync)", f64(out_m), r_out, tol)
    assert_close("lse (mma.sync)", f64(lse_m), r_lse, tol)


def test_large_score_range_takes_the_rescale_path():
    # q scaled by 12: scores spread over tens of units (base 2), so later tap rows raise the max
    # by more than the lazy-rescale threshold and the accumulators are rescaled
    dims, heads, dh, window = (4, 10, 14), 2, 128, (3, 7, 7)
    _, inp = inputs.custom(*dims, heads, dh, window, "bf16", seed=611, scale=2.0)
    inp["q"] = (inp["q"].float() * 12).to(torch.bfloat16)
    d = to_cuda(inp)
    out, lse = _fwd(d, dims, window)
    r_out, r_lse = oracle.full_forward(inp["q"], inp["k"], inp["v"], inp["offsets"], dims, window)
    assert_close("out", f64(out), r_out, TOL["bf16"])
    # lse grows with the scores; its bf16-input error grows with it (relative 2^-8 of the scores)
    assert_close("lse", f64(lse), r_lse, max(TOL["bf16"], 2e-3 * float(abs(r_lse[abs(r_lse) < 1e30]).max())))


@pytest.mark.parametrize("case", [0, 2])
def test_every_tile_geometry_gives_the_same_bits(case):
    dims, heads, dh, window, scale = CASES[case]
    _, inp = inputs.custom(*dims, heads, dh, window, "bf16", seed=700 + case, scale=scale)
    d = to_cuda(inp)
    ref = _fwd(d, dims, window)
    for ry in (1, 3, 8, 12):
        with _env(DSA3D_TC_RY=ry):
            got = _fwd(d, dims, window)
        assert torch.equal(got[0], ref[0]) and torch.equal(got[1], ref[1]), f"Ry={ry}"
