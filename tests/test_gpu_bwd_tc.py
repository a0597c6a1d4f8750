"""The tcgen05 passes of the backward -- the key side (dK, dV in tensor memory) and dq (dq in
tensor memory) -- against the oracle and against the mma.sync passes they replace.

DSA3D_KV_KERNEL=mma and DSA3D_DQ_KERNEL=mma select the mma.sync passes (the library reads them at
every call).  Both forms sum the same bf16 products in fp32, in different orders; their results
agree to the oracle's tolerance, and each is bit-for-bit repeatable
(tests/test_gpu_determinism.py).  A window whose key tiles span more bucket-row ranges than the
tcgen05 key side takes ((kt + 1)(4 + kh) > 128) falls back to the mma.sync key side.
"""
import os

import pytest
import torch

import oracle
from deformable_slide_attention_b200 import abi, inputs
from tests.gpu_helpers import TOL, assert_close, f64, to_cuda

pytestmark = [pytest.mark.gpu, pytest.mark.usefixtures("gpu_lib", "oracle_lib")]

# (dims, heads, dh, window, offset scale): ragged key tiles in y (H' not a multiple of 4) and x
# (W' not a multiple of 32), dh 64 and 128, frames at both ends, wide and flat windows
CASES = [((3, 7, 9), 3, 64, (3, 5, 5), 2.5),
         ((4, 10, 37), 2, 128, (3, 7, 7), 3.0),
         ((5, 13, 70), 1, 64, (3, 9, 9), 4.0),
         ((2, 6, 33), 2, 128, (1, 3, 15), 2.0),
         ((6, 5, 40), 1, 64, (5, 1, 1), 1.5),
         ((5, 9, 12), 1, 64, (7, 13, 3), 2.0)]   # (7 + 1)(4 + 13) > 128: the mma.sync fallback


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


def _bwd(d, lse, dims, window):
    grads = abi.backward(d["q"], d["k"], d["v"], d["offsets"], lse, d["dout"], dims, window)
    torch.cuda.synchronize()
    return grads


@pytest.mark.parametrize("case", range(len(CASES)))
def test_key_side_matches_the_oracle_and_the_mma_key_side(case):
    dims, heads, dh, window, scale = CASES[case]
    _, inp = inputs.custom(*dims, heads, dh, window, "bf16", seed=900 + case, scale=scale)
    d = to_cuda(inp)
    _, lse = abi.forward(d["q"], d["k"], d["v"], d["offsets"], dims, window)
    r_dq, r_doff, r_dk, r_dv = oracle.full_backward(inp["q"], inp["k"], inp["v"], inp["offsets"],
                                                    inp["dout"], dims, window)
    tol = TOL["bf16"]
    dq, dk, dv, doff = _bwd(d, lse, dims, window)
    assert_close("dk", f64(dk), r_dk, tol)
    assert_close("dv", f64(dv), r_dv, tol)
    assert_close("dq", f64(dq), r_dq, tol)
    with _env(DSA3D_KV_KERNEL="mma"):
        dq_m, dk_m, dv_m, _ = _bwd(d, lse, dims, window)
    assert_close("dk (mma.sync)", f64(dk_m), r_dk, tol)
    assert_close("dv (mma.sync)", f64(dv_m), r_dv, tol)
    assert torch.equal(dq, dq_m), "the key side must not change dq"
    # the two key sides sum the same bf16 products of each key in fp32, in different orders
    assert abs(f64(dk) - f64(dk_m)).max() <= tol
    assert abs(f64(dv) - f64(dv_m)).max() <= tol
    with _env(DSA3D_DQ_KERNEL="mma"):
        dq_q, dk_q, dv_q, doff_q = _bwd(d, lse, dims, window)
    assert_close("dq (mma.sync)", f64(dq_q), r_dq, tol)
    assert abs(f64(dq) - f64(dq_q)).max() <= tol
    assert torch.equal(dk, dk_q) and torch.equal(dv, dv_q) and torch.equal(doff, doff_q), \
        "the dq pass must not change the other gradients"


def test_720p_train_tc_passes_agree_with_the_mma_passes():
    # the full 720p training workload (16 heads x 115,200 tokens): every key and query of every
    # head, against the mma.sync passes, to the bf16 output rounding of the two summation orders
    w = inputs.BY_NAME["720p-train-bf16"]
    inp = inputs.make(w, "cpu", with_dout=True)
    d = to_cuda(inp)
    _, lse = abi.forward(d["q"], d["k"], d["v"], d["offsets"], w.dims, w.window)
    dq, dk, dv, _ = _bwd(d, lse, w.dims, w.window)
    with _env(DSA3D_KV_KERNEL="mma", DSA3D_DQ_KERNEL="mma"):
        dq_m, dk_m, dv_m, _ = _bwd(d, lse, w.dims, w.window)
    for name, a, b in (("dq", dq, dq_m), ("dk", dk, dk_m), ("dv", dv, dv_m)):
        a, b = a.float(), b.float()
        err = (a - b).abs()
        bound = 2e-2 + 2.0 ** -7 * torch.maximum(a.abs(), b.abs())
        assert bool((err <= bound).all()), f"{name}: max error {err.max().item():.3e}"
