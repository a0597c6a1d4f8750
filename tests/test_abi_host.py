"""Host-side checks of the C ABI that need no GPU: the library loads, exports every function the
header declares, and rejects bad arguments before touching the device."""
import ctypes
import os
import re

import pytest

from deformable_slide_attention_b200 import abi, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    build.build()
    return ctypes.CDLL(abi.library_path())


def declared_functions():
    names = []
    for h in os.listdir(os.path.join(ROOT, "include")):
        if h.endswith(".h"):
            text = open(os.path.join(ROOT, "include", h)).read()
            text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
            names += re.findall(r"\b(dsa3d_\w+)\s*\(", text)
    return sorted(set(names))


def test_every_declared_symbol_is_exported(lib):
    names = declared_functions()
    assert {"dsa3d_forward", "dsa3d_backward", "dsa3d_backward_workspace_bytes",
            "dsa3d_abi_version", "dsa3d_status_string", "dsa3d_check_device"} <= set(names)
    for n in names:
        assert hasattr(lib, n), n


def test_abi_version_and_status_strings():
    assert abi.dsa3d_abi_version() == 3
    for s in range(6):
        assert abi.dsa3d_status_string(s)
    assert abi.dsa3d_status_string(0) == "ok"


ARGS = dict(F=4, Hp=8, Wp=8, heads=2, dh=64, kt=3, kh=3, kw=3)
P = 1 << 20  # a fake 16-byte-aligned address; validation fails before any device access


def fwd(**kw):
    a = {**ARGS, **kw}
    ptrs = [kw.get(n, P * (i + 1)) for i, n in enumerate(["q", "k", "v", "off", "out", "lse"])]
    return abi.dsa3d_forward(*ptrs, kw.get("ws", 0), kw.get("wsb", 0), a["F"], a["Hp"], a["Wp"],
                             a["heads"], a["dh"], a["kt"], a["kh"], a["kw"],
                             kw.get("dtype", abi.DSA3D_BF16), 0)


def test_forward_rejects_bad_arguments():
    INV, UNS = 1, 2
    assert fwd(q=0) == INV
    assert fwd(out=P + 8) == INV  # misaligned
    assert fwd(kt=2) == INV       # even window
    assert fwd(kw=0) == INV
    assert fwd(F=0) == INV
    assert fwd(heads=0) == INV
    assert fwd(dtype=7) == INV
    assert fwd(dh=48) == UNS
    assert fwd(kh=17) == UNS      # larger than 2*Hp-1
    # out overlapping q
    assert fwd(q=P, out=P + 4096) == INV
    # a workspace smaller than one head's sort, and one overlapping an input
    assert fwd(ws=P * 64, wsb=1024) == 3
    need = abi.dsa3d_forward_workspace_bytes(4, 8, 8, 1, 64, 3, 3, 3, abi.DSA3D_BF16)
    assert fwd(ws=P, wsb=need) == INV


def test_forward_accepts_a_null_workspace():
    """The forward's workspace is optional (a departure from the survey's workspace-free forward
    signature, made because the library allocates nothing and the sort needs scratch): a NULL
    workspace passes validation and runs the general CUDA-core kernels, a non-NULL one smaller than
    one head's need is refused, and a large enough one selects the sorted tensor-core path.  Here,
    without a GPU, a call that passes validation ends at the device with DSA3D_ERR_CUDA (the fake
    pointers are never dereferenced); on a machine with a GPU the call would launch on them, so
    the test does not run there."""
    import torch
    if torch.cuda.is_available():
        pytest.skip("would launch kernels on fake device pointers")
    assert fwd(ws=0, wsb=0) == 4          # validated, then no device: DSA3D_ERR_CUDA
    assert fwd(ws=0, wsb=0, dtype=abi.DSA3D_F32) == 4
    need = abi.dsa3d_forward_workspace_bytes(4, 8, 8, 1, 64, 3, 3, 3, abi.DSA3D_BF16)
    assert need > 0
    assert fwd(ws=P * 64, wsb=need - 16) == 3   # DSA3D_ERR_WORKSPACE_TOO_SMALL, before any launch
    assert fwd(ws=P * 64, wsb=need) == 4        # the tensor-core path, then no device


def test_forward_workspace_bytes():
    # the sort's arrays (buckets, then key, rank, sorted token and x-origin per query, then the
    # scan's block sums) and the paired value rows: F Hp ceil(Wp/2) pairs x heads x dh words
    a16 = lambda b: (b + 15) // 16 * 16
    for (F, Hp, Wp, H, dh, kt, kh, kw) in ((4, 8, 8, 1, 64, 3, 3, 3), (4, 8, 9, 2, 128, 3, 5, 7)):
        N = F * Hp * Wp
        E1 = (F + kt) * (Hp + kh) * (Wp + kw) + 1
        nb = (H * E1 + 2047) // 2048
        sort = a16(4 * H * E1) + 4 * a16(4 * H * N) + a16(4 * nb)
        pairs = a16(F * Hp * ((Wp + 1) // 2) * H * dh * 4)
        assert abi.dsa3d_forward_workspace_bytes(F, Hp, Wp, H, dh, kt, kh, kw, abi.DSA3D_BF16) == sort + pairs
    one = abi.dsa3d_forward_workspace_bytes(4, 8, 8, 1, 64, 3, 3, 3, abi.DSA3D_BF16)
    assert abi.dsa3d_forward_workspace_bytes(4, 8, 8, 2, 64, 3, 3, 3, abi.DSA3D_BF16) > one
    # no tensor-core path: fp32, dh 32, kw > 15
    assert abi.dsa3d_forward_workspace_bytes(4, 8, 8, 2, 64, 3, 3, 3, abi.DSA3D_F32) == 0
    assert abi.dsa3d_forward_workspace_bytes(4, 8, 8, 2, 32, 3, 3, 3, abi.DSA3D_BF16) == 0
    assert abi.dsa3d_forward_workspace_bytes(4, 8, 16, 2, 64, 3, 3, 17, abi.DSA3D_BF16) == 0


def test_backward_workspace_bytes():
    a16 = lambda b: (b + 15) // 16 * 16
    F, Hp, Wp, H, kt, kh, kw = 4, 8, 8, 2, 3, 3, 3
    N = F * Hp * Wp
    # tensor-core backward (bf16, dh 64/128, kw <= 15): the sort's arrays, the bf16 splats of P and
    # P dP per query and tap plane (kt (kh+1) (kw+1) each), and (D, f_t) per query
    E1 = (F + kt) * (Hp + kh) * (Wp + kw) + 1
    nb = (H * E1 + 2047) // 2048
    sort = a16(4 * H * E1) + 4 * a16(4 * H * N) + a16(4 * nb)
    splats = 2 * a16(H * N * kt * (kh + 1) * (kw + 1) * 2) + a16(H * N * 8)
    assert abi.dsa3d_backward_workspace_bytes(F, Hp, Wp, H, 64, kt, kh, kw, abi.DSA3D_BF16) == sort + splats
    # CUDA-core backward (bf16, dh 32): fp32 dK and dV accumulators of every head
    assert abi.dsa3d_backward_workspace_bytes(F, Hp, Wp, H, 32, kt, kh, kw, abi.DSA3D_BF16) == 2 * N * 32 * 4 * H
    assert abi.dsa3d_backward_workspace_bytes(F, Hp, Wp, H, 64, kt, kh, kw, abi.DSA3D_F32) == 0
    assert abi.dsa3d_backward_workspace_bytes(F, Hp, Wp, H, 48, kt, kh, kw, abi.DSA3D_BF16) == 0


def test_backward_rejects_bad_arguments():
    ptr = [P * (i + 1) for i in range(11)]
    a = ARGS
    call = lambda ptrs, wsb=0, dtype=abi.DSA3D_BF16, **kw: abi.dsa3d_backward(
        *ptrs, wsb, kw.get("F", a["F"]), a["Hp"], a["Wp"], a["heads"], a["dh"], a["kt"], a["kh"],
        a["kw"], dtype, 0)
    bad = list(ptr)
    bad[2] = 0
    assert call(bad) == 1
    # workspace too small for one head
    assert call(ptr, wsb=1000) == 3
    # dk aliasing q
    alias = list(ptr)
    alias[7] = ptr[0]
    assert call(alias, wsb=1 << 30) == 1


def fwd_taps(**kw):
    a = {**ARGS, **kw}
    ptrs = [kw.get(n, P * (i + 1)) for i, n in enumerate(["q", "k", "v", "off", "out", "lse"])]
    return abi.dsa3d_forward_taps(*ptrs, a["F"], a["Hp"], a["Wp"], a["heads"], a["dh"], a["kt"],
                                  a["kh"], a["kw"], kw.get("dtype", abi.DSA3D_BF16), 0)


def test_forward_taps_rejects_bad_arguments():
    INV, UNS = 1, 2
    assert fwd_taps(v=0) == INV
    assert fwd_taps(off=P * 4 + 4) == INV   # misaligned
    assert fwd_taps(kh=4) == INV            # even window
    assert fwd_taps(dtype=3) == INV
    assert fwd_taps(dh=96) == UNS
    assert fwd_taps(kw=17) == UNS           # larger than 2*Wp-1
    # the per-tap offsets are K = 27 times the per-token size (2 * 256 * 27 * 12 bytes): an
    # output placed 100 KB after their start overlaps them
    assert fwd_taps(off=P * 8, out=P * 8 + 100_000) == INV


def test_backward_taps_workspace_bytes_and_rejections():
    F, Hp, Wp, H, kt, kh, kw = 4, 8, 8, 2, 3, 3, 3
    N = F * Hp * Wp
    # fp32 dK/dV accumulators of every head with bf16 I/O (no tensor-core path for per-tap
    # offsets), none with fp32 I/O
    for dh in (32, 64, 128):
        assert abi.dsa3d_backward_taps_workspace_bytes(F, Hp, Wp, H, dh, kt, kh, kw, abi.DSA3D_BF16) == 2 * N * dh * 4 * H
        assert abi.dsa3d_backward_taps_workspace_bytes(F, Hp, Wp, H, dh, kt, kh, kw, abi.DSA3D_F32) == 0
    assert abi.dsa3d_backward_taps_workspace_bytes(F, Hp, Wp, H, 48, kt, kh, kw, abi.DSA3D_BF16) == 0
    # q, k, v, offsets, lse, dout, dq, dk, dv, doffsets, workspace
    ptr = [P * (i + 1) for i in range(11)]
    a = ARGS
    call = lambda ptrs, wsb=0, dtype=abi.DSA3D_BF16: abi.dsa3d_backward_taps(
        *ptrs, wsb, a["F"], a["Hp"], a["Wp"], a["heads"], a["dh"], a["kt"], a["kh"], a["kw"], dtype, 0)
    for i in (4, 5):  # lse, dout
        bad = list(ptr)
        bad[i] = 0
        assert call(bad, wsb=1 << 30) == 1
    misaligned = list(ptr)
    misaligned[5] += 8
    assert call(misaligned, wsb=1 << 30) == 1
    assert call(ptr, wsb=1000) == 3  # smaller than one head's accumulators
    alias = list(ptr)
    alias[9] = ptr[3] + 16 * 4096  # doffsets inside the per-tap offsets
    assert call(alias, wsb=1 << 30) == 1
    alias = list(ptr)
    alias[6] = ptr[5]  # dq on top of dout
    assert call(alias, wsb=1 << 30) == 1
    overlap_ws = list(ptr)
    overlap_ws[10] = ptr[2]  # workspace on top of v
    assert call(overlap_ws, wsb=1 << 20) == 1


def test_offset_head_rejections():
    a = dict(F=2, Hp=4, Wp=4, C=8, heads=2, kt=3, kh=3, kw=3)
    need = abi.dsa3d_offset_head_workspace_bytes(a["F"], a["Hp"], a["Wp"], a["C"])
    assert need == 2 * 4 * 4 * 8 * 4

    def call(taps=1, C=8, wsb=need, ws=P * 20, x=P):
        return abi.dsa3d_offset_head(x, P * 2, None, P * 4, P * 6, P * 8, ws, wsb, a["F"], a["Hp"],
                                     a["Wp"], C, a["heads"], taps, a["kt"], a["kh"], a["kw"],
                                     abi.DSA3D_BF16, 0)
    assert call(taps=5) == 1          # neither 1 nor kt*kh*kw
    assert call(C=6) == 2             # the pointwise layer reads 4 channels at a time
    assert call(wsb=need - 16) == 3   # workspace too small
    assert call(x=0) == 1
    assert call(ws=P * 8) == 1        # workspace on top of the offsets


def test_offset_head_backward_rejections():
    F, Hp, Wp, C, heads = 2, 4, 4, 16, 2
    need = abi.dsa3d_offset_head_backward_workspace_bytes(F, Hp, Wp, C)
    assert need == 2 * F * Hp * Wp * C * 4
    ptr = [P * (i + 1) for i in range(11)]  # x, dw_w, dw_b, pw_w, doff, dx, ddw, ddb, dpw, dpb, ws

    def call(p=ptr, C=C, taps=1, wsb=need):
        return abi.dsa3d_offset_head_backward(*p, wsb, F, Hp, Wp, C, heads, taps, 3, 3, 3,
                                              abi.DSA3D_BF16, 0)
    assert call(C=8) == 2          # 16-channel groups in the weight gradient
    assert call(taps=4) == 1
    assert call(wsb=need - 16) == 3
    bad = list(ptr)
    bad[5] = 0                     # dx
    assert call(bad) == 1
    alias = list(ptr)
    alias[5] = ptr[0]              # dx on top of x
    assert call(alias) == 1
