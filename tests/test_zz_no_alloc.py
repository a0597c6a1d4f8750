"""The allocation-free backward entry point (dsa3d_backward_noalloc).

It is for callers that cannot allocate device memory or pass a workspace -- plugin hosts that own
every allocation, fixed call signatures without a workspace argument, steps that must not pay
cudaMalloc's device-wide synchronisation.  Its scratch is a fixed device array inside the library,
so these tests check that two calls in a row (the second finds the first call's leftovers in the
shared array) both reproduce the regular workspace entry point, and that a problem too large for
the array is refused before anything runs.  This file is named to be collected last.
"""
import pytest
import torch

from deformable_slide_attention_b200 import abi, inputs
from tests.gpu_helpers import TOL, to_cuda

pytestmark = [pytest.mark.gpu, pytest.mark.usefixtures("gpu_lib")]


def _noalloc(d, lse, dims, window, dtype_code):
    N = dims[0] * dims[1] * dims[2]
    heads, dh = d["q"].shape[1], d["q"].shape[2]
    grads = (torch.empty_like(d["q"]), torch.empty_like(d["k"]), torch.empty_like(d["v"]),
             torch.empty_like(d["offsets"]))
    st = abi.dsa3d_backward_noalloc(
        d["q"].data_ptr(), d["k"].data_ptr(), d["v"].data_ptr(), d["offsets"].data_ptr(),
        lse.data_ptr(), d["dout"].data_ptr(), *(g.data_ptr() for g in grads),
        *dims, heads, dh, *window, dtype_code, torch.cuda.current_stream().cuda_stream)
    torch.cuda.synchronize()
    assert st == 0, abi.dsa3d_status_string(st)
    assert grads[0].shape[0] == N
    return grads


@pytest.mark.parametrize("dims,heads,dh,window", [
    ((16, 32, 32), 8, 64, (3, 7, 7)),    # tensor-core path, all heads in one pass of the scratch
    ((16, 64, 64), 2, 128, (3, 5, 5)),   # tensor-core path, both heads in one pass (~58 MiB)
    ((32, 45, 80), 2, 128, (3, 3, 3)),   # tensor-core path: one head's sort and splats (~26 MB)
                                         # fit, although its fp32 accumulators (118 MB) would not
    ((16, 96, 96), 2, 32, (3, 3, 3)),    # dh 32: the general path; one head's accumulators
                                         # (37.7 MB) fit, two do not: two passes of the scratch
])
def test_noalloc_matches_workspace_backward_twice(dims, heads, dh, window):
    _, inp = inputs.custom(*dims, heads, dh, window, "bf16", seed=41, scale=2.0)
    d = to_cuda(inp)
    out, lse = abi.forward(d["q"], d["k"], d["v"], d["offsets"], dims, window)
    ref = abi.backward(d["q"], d["k"], d["v"], d["offsets"], lse, d["dout"], dims, window)
    torch.cuda.synchronize()
    for _ in range(2):
        got = _noalloc(d, lse, dims, window, abi.DSA3D_BF16)
        for name, a, b in zip(("dq", "dk", "dv", "doffsets"), got, ref):
            err = (a.float() - b.float()).abs().max().item()
            assert err <= TOL["bf16"], f"{name}: {err:.3e}"


def test_noalloc_refuses_problem_larger_than_its_scratch():
    # 720p at dh 128 with a 3x9x9 window: one head's stored splats alone take 138 MB and its fp32
    # accumulators 118 MB, so neither path fits the 64 MiB scratch
    dims, heads, dh, window = (32, 45, 80), 2, 128, (3, 9, 9)
    N = dims[0] * dims[1] * dims[2]
    assert 2 * N * dh * 4 > (64 << 20)
    assert abi.dsa3d_backward_workspace_bytes(*dims, 1, dh, *window, abi.DSA3D_BF16) > (64 << 20)
    t = torch.zeros(16, dtype=torch.uint8, device="cuda")  # never dereferenced: refused on the host
    p = t.data_ptr()
    st = abi.dsa3d_backward_noalloc(p, p + 1024, p + 2048, p + 3072, p + 4096, p + 5120, p + 6144,
                                    p + 7168, p + 8192, p + 9216, *dims, heads, dh,
                                    *window, abi.DSA3D_BF16, torch.cuda.current_stream().cuda_stream)
    assert st == 3  # DSA3D_ERR_WORKSPACE_TOO_SMALL
