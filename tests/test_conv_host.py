"""The depthwise-convolution kernels' per-thread routines (conv_strip2, dw_walk in
csrc/dsa3d_conv.cuh) and the offset network's pointwise routine (pw_tile in
csrc/dsa3d_pointwise.cuh), run on the CPU by a host harness over every work item the GPU kernels
process, against the oracle's convolution (reading R9).  The forward runs as the library launches
it: the staged kernel's blocks (channel group, run of units, weights copied tap-major) or, past
the staged tap limit, the global kernel's items.  This checks their indexing, boundary handling,
kernel flip and weight-gradient accumulation without a GPU; the GPU parity tests call the same
code through the C ABI.

Tolerances: the routines accumulate in fp32 (the oracle in fp64): max-abs 1e-4 relative to the
output scale for the forward and dX, 1e-4 relative for dW and db (sums over all tokens).
"""
import ctypes
import math
import os
import subprocess

import numpy as np
import pytest
import torch

import oracle

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
SRC = os.path.join(HERE, "conv_host", "conv_host_harness.cu")
CSRC = os.path.join(ROOT, "deformable_slide_attention_b200", "csrc")
LIB = os.path.join(HERE, "conv_host", "_build", "libconvhost.so")


@pytest.fixture(scope="module")
def harness():
    deps = [SRC, os.path.join(CSRC, "dsa3d_conv.cuh"), os.path.join(CSRC, "dsa3d_pointwise.cuh")]
    if not os.path.exists(LIB) or os.path.getmtime(LIB) < max(os.path.getmtime(d) for d in deps):
        os.makedirs(os.path.dirname(LIB), exist_ok=True)
        subprocess.run(["/usr/local/cuda/bin/nvcc", "-O2", "-std=c++17", "-x", "cu",
                        "-gencode", "arch=compute_100a,code=sm_100a", "-Xcompiler", "-fPIC",
                        "-shared", "-I", CSRC, "-o", LIB + ".tmp", SRC], check=True)
        os.replace(LIB + ".tmp", LIB)
    lib = ctypes.CDLL(LIB)
    I, P = ctypes.c_int, ctypes.c_void_p
    lib.conv_host_forward.argtypes = [I, P, P, P] + [I] * 7 + [I, P]
    lib.conv_host_dw.argtypes = [I, P, P] + [I] * 7 + [I, P, P]
    lib.pw_host_offsets.argtypes = [P, P, P, I, I, I, ctypes.c_longlong, P]
    lib.conv_host_dw_mixed.argtypes = [I, P, P] + [I] * 7 + [I, P, P]
    L = ctypes.c_longlong
    lib.pw_host_backward.argtypes = [P, P, P, I, I, I, L, L, P, P, P]
    return lib


def _io(x):
    x = x.contiguous()
    if x.dtype == torch.bfloat16:
        return 1, x.view(torch.int16).numpy()
    return 0, x.numpy()


def _ptr(a):
    return ctypes.c_void_p(a.ctypes.data) if a is not None else None


def host_forward(lib, x, w, b, dims, flip=False):
    io, xa = _io(x)
    C = x.shape[1]
    wa = w.float().contiguous().numpy()
    ba = None if b is None else b.float().contiguous().numpy()
    y = np.zeros((x.shape[0], C), np.float32)
    rc = lib.conv_host_forward(io, _ptr(xa), _ptr(wa), _ptr(ba), *dims, C, *w.shape[1:], int(flip),
                               _ptr(y))
    assert rc == 0
    return y


def host_dw(lib, x, dy, dims, window, frames_per_item):
    io, xa = _io(x)
    _, da = _io(dy)
    C = x.shape[1]
    dw = np.zeros((C, *window), np.float32)
    db = np.zeros(C, np.float32)
    rc = lib.conv_host_dw(io, _ptr(xa), _ptr(da), *dims, C, *window, frames_per_item, _ptr(dw), _ptr(db))
    assert rc == 0
    return dw, db


CASES = [((3, 5, 6), 4, (3, 3, 3)), ((2, 7, 19), 6, (3, 5, 9)), ((4, 3, 11), 2, (1, 1, 15)),
         ((1, 4, 9), 8, (1, 3, 1)), ((5, 2, 17), 4, (5, 3, 7)), ((2, 3, 8), 2, (3, 3, 13))]


# The forward's staged kernel: two runs of units and a last channel group of one pair (C = 66);
# the strip-pair kernel over five groups (C = 160); and 405 taps, past the staged limit (the
# global kernel).
FWD_CASES = CASES + [((4, 7, 40), 66, (3, 5, 9)), ((3, 5, 6), 160, (3, 3, 3)), ((3, 5, 12), 4, (5, 9, 9)),
                     # C a multiple of 32 (the strip-pair kernel): a ragged last strip pair, k_w = 15
                     ((4, 9, 21), 64, (3, 9, 9)), ((2, 7, 40), 32, (1, 5, 15))]
# dW's kernel-row groups of three: kh = 7 (3 + 3 + 1) and kh = 9 as well; C a multiple of 64 (the
# warp-cooperative copies), with a ragged last strip
DW_CASES = FWD_CASES + [((3, 4, 10), 4, (3, 7, 3)), ((3, 5, 12), 128, (3, 9, 9)), ((2, 4, 19), 64, (1, 3, 5))]


@pytest.mark.parametrize("dims,C,window", FWD_CASES)
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_forward_and_dx_match_oracle(harness, dims, C, window, dtype):
    g = torch.Generator().manual_seed(sum(dims) + C)
    N = math.prod(dims)
    x = torch.randn(N, C, generator=g).to(dtype)
    w = torch.randn(C, *window, generator=g)
    b = torch.randn(C, generator=g)
    y = host_forward(harness, x, w, b, dims)
    ref = oracle.dwconv3d(x, w, b, dims)
    assert np.abs(y - ref).max() <= 1e-4 * max(1.0, np.abs(ref).max())
    # dX = the forward on dY with the kernel flipped (no bias)
    dy = torch.randn(N, C, generator=g).to(dtype)
    dx = host_forward(harness, dy, w, None, dims, flip=True)
    ref_dx, _, _ = oracle.dwconv3d_backward(x, w, dy.double().numpy(), dims)
    assert np.abs(dx - ref_dx).max() <= 1e-4 * max(1.0, np.abs(ref_dx).max())


@pytest.mark.parametrize("dims,C,window", DW_CASES)
@pytest.mark.parametrize("frames_per_item", [1, 2, 64])
def test_weight_gradient_matches_oracle(harness, dims, C, window, frames_per_item):
    g = torch.Generator().manual_seed(7 + sum(window))
    N = math.prod(dims)
    x = torch.randn(N, C, generator=g).to(torch.bfloat16)
    dy = torch.randn(N, C, generator=g).to(torch.bfloat16)
    w = torch.randn(C, *window, generator=g)
    dw, db = host_dw(harness, x, dy, dims, window, frames_per_item)
    _, ref_dw, ref_db = oracle.dwconv3d_backward(x, w, dy.double().numpy(), dims)
    assert np.abs(dw - ref_dw).max() <= 1e-4 * max(1.0, np.abs(ref_dw).max())
    assert np.abs(db - ref_db).max() <= 1e-4 * max(1.0, np.abs(ref_db).max())


def test_unsupported_width_is_refused(harness):
    x = torch.zeros(6, 2)
    y = np.zeros((6, 2), np.float32)
    w = np.zeros((2, 1, 1, 17), np.float32)
    io, xa = _io(x)
    assert harness.conv_host_forward(io, _ptr(xa), _ptr(w), None, 1, 1, 6, 2, 1, 1, 17, 0, _ptr(y)) == -1


@pytest.mark.parametrize("taps", [None, 9])
@pytest.mark.parametrize("dims,heads,dh,window", [((2, 5, 6), 2, 8, (1, 3, 3)),
                                                  ((3, 4, 9), 3, 4, (3, 3, 5))])
def test_offset_network_matches_oracle(harness, dims, heads, dh, window, taps):
    """Z = the conv routine in fp32 (as the GPU writes it to its workspace), then the pointwise
    routine into the attention's offset layout, against oracle.offset_head."""
    if taps is not None:
        taps = math.prod(window)
    C, N = heads * dh, math.prod(dims)
    g = torch.Generator().manual_seed(C + N)
    x = torch.randn(N, C, generator=g).to(torch.bfloat16)
    dw_w, dw_b = torch.randn(C, *window, generator=g), torch.randn(C, generator=g)
    width = heads * 3 * (taps or 1)
    pw_w = torch.randn(C, width, generator=g) * 0.2
    pw_b = torch.randn(width, generator=g)
    z = host_forward(harness, x, dw_w, dw_b, dims)
    off = np.zeros((heads, N, taps, 3) if taps else (heads, N, 3), np.float32)
    wa, ba = pw_w.contiguous().numpy(), pw_b.contiguous().numpy()
    rc = harness.pw_host_offsets(_ptr(np.ascontiguousarray(z)), _ptr(wa), _ptr(ba), C, width,
                                 3 * (taps or 1), N, _ptr(off))
    assert rc == 0
    ref = oracle.offset_head(x, dw_w, dw_b, pw_w, pw_b, dims, heads, taps)
    assert np.abs(off - ref).max() <= 1e-4 * max(1.0, np.abs(ref).max())


@pytest.mark.parametrize("taps", [None, 9])
@pytest.mark.parametrize("tokens_per_item", [7, 1000])
def test_offset_network_backward_matches_oracle(harness, taps, tokens_per_item):
    """The backward's pieces in the order the library runs them: Z (conv, fp32), dZ and dWp/dbp
    (pointwise), dX (conv of the fp32 dZ with the flipped kernel), dW/db (x in bf16, dZ in fp32),
    against oracle.offset_head_backward."""
    dims, heads, dh, window = (2, 5, 6), 2, 16, (1, 3, 3)
    if taps is not None:
        taps = math.prod(window)
    C, N = heads * dh, math.prod(dims)
    g = torch.Generator().manual_seed(5 + C)
    x = torch.randn(N, C, generator=g).to(torch.bfloat16)
    dw_w, dw_b = torch.randn(C, *window, generator=g), torch.randn(C, generator=g)
    width = heads * 3 * (taps or 1)
    pw_w = torch.randn(C, width, generator=g) * 0.2
    doff = torch.randn((heads, N, taps, 3) if taps else (heads, N, 3), generator=g)
    z = np.ascontiguousarray(host_forward(harness, x, dw_w, dw_b, dims))
    dz = np.zeros((N, C), np.float32)
    dwp = np.zeros((C, width), np.float32)
    dbp = np.zeros(width, np.float32)
    wa, da = pw_w.contiguous().numpy(), doff.contiguous().numpy()
    assert harness.pw_host_backward(_ptr(z), _ptr(da), _ptr(wa), C, width, 3 * (taps or 1), N,
                                    tokens_per_item, _ptr(dz), _ptr(dwp), _ptr(dbp)) == 0
    dx = host_forward(harness, torch.from_numpy(dz), dw_w, None, dims, flip=True)
    ddw = np.zeros((C, *window), np.float32)
    ddb = np.zeros(C, np.float32)
    io, xa = _io(x)
    assert harness.conv_host_dw_mixed(io, _ptr(xa), _ptr(dz), *dims, C, *window, 3, _ptr(ddw),
                                      _ptr(ddb)) == 0
    ref = oracle.offset_head_backward(x, dw_w, dw_b, pw_w, doff.double().numpy(), dims)
    for name, got, want in (("dx", dx, ref[0]), ("d dw_weight", ddw, ref[1]), ("d dw_bias", ddb, ref[2]),
                            ("d pw_weight", dwp, ref[3]), ("d pw_bias", dbp, ref[4])):
        err = np.abs(got - want).max()
        assert err <= 1e-4 * max(1.0, np.abs(want).max()), (name, err)


@pytest.mark.parametrize("frames_per_item", [1, 3])
def test_weight_gradient_fp32_dy_cooperative(harness, frames_per_item):
    """dW with x in bf16 and dY in fp32 (the offset network's backward) at C = 64, where the
    library takes the warp-cooperative copies: a token's 32 fp32 pairs are 16 chunks, so a lane's
    chunks are two tokens apart (eight for bf16)."""
    dims, C, window = (3, 6, 19), 64, (3, 5, 7)
    g = torch.Generator().manual_seed(19)
    N = math.prod(dims)
    x = torch.randn(N, C, generator=g).to(torch.bfloat16)
    dy = torch.randn(N, C, generator=g)
    w = torch.randn(C, *window, generator=g)
    io, xa = _io(x)
    dya = dy.contiguous().numpy()
    dw = np.zeros((C, *window), np.float32)
    db = np.zeros(C, np.float32)
    assert harness.conv_host_dw_mixed(io, _ptr(xa), _ptr(dya), *dims, C, *window, frames_per_item,
                                      _ptr(dw), _ptr(db)) == 0
    _, ref_dw, ref_db = oracle.dwconv3d_backward(x, w, dy.double().numpy(), dims)
    assert np.abs(dw - ref_dw).max() <= 1e-4 * max(1.0, np.abs(ref_dw).max())
    assert np.abs(db - ref_db).max() <= 1e-4 * max(1.0, np.abs(ref_db).max())
