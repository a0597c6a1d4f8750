"""The torch conveniences of the binding (abi.forward, backward, forward_taps, backward_taps,
dwconv3d, dwconv3d_backward) check every tensor they hand to the C ABI, which takes plain pointers
and trusts the extents.  On the CPU: the C calls, the stream lookup and the device check are
replaced by stand-ins, so the call patterns of the GPU tests and bench.py run with CPU tensors,
and mismatched tensors must be refused before any C call."""
import math

import pytest
import torch

from deformable_slide_attention_b200 import abi

DIMS, WINDOW, HEADS, DH = (2, 3, 4), (1, 3, 3), 2, 32
N, K = math.prod(DIMS), math.prod(WINDOW)


@pytest.fixture()
def calls(monkeypatch):
    log = []

    def fake(name):
        def f(*args):
            log.append(name)
            return 0
        return f

    for name in ("dsa3d_forward", "dsa3d_backward", "dsa3d_forward_taps", "dsa3d_backward_taps",
                 "dsa3d_dwconv3d", "dsa3d_dwconv3d_backward", "dsa3d_offset_head"):
        monkeypatch.setattr(abi, name, fake(name))
    for name in ("dsa3d_forward_workspace_bytes", "dsa3d_backward_workspace_bytes",
                 "dsa3d_backward_taps_workspace_bytes", "dsa3d_offset_head_workspace_bytes"):
        monkeypatch.setattr(abi, name, lambda *a: 64)
    monkeypatch.setattr(abi, "_on_device", lambda *a: None)
    monkeypatch.setattr(abi, "_stream_handle", lambda s: 0)
    return log


def _inputs(dtype=torch.bfloat16, taps=False):
    q, k, v, dout = (torch.zeros(N, HEADS, DH, dtype=dtype) for _ in range(4))
    off = torch.zeros((HEADS, N, K, 3) if taps else (HEADS, N, 3))
    lse = torch.zeros(HEADS, N)
    return q, k, v, off, lse, dout


def test_call_patterns_of_the_tests_and_the_bench_are_accepted(calls):
    q, k, v, off, lse, dout = _inputs()
    out, l2 = abi.forward(q, k, v, off, DIMS, WINDOW)
    abi.forward(q, k, v, off, DIMS, WINDOW, out=out, lse=l2, workspace=torch.empty(64, dtype=torch.uint8))
    abi.forward(q, k, v, off, DIMS, WINDOW, workspace=None, want_lse=False)
    grads = abi.backward(q, k, v, off, lse, dout, DIMS, WINDOW)
    abi.backward(q, k, v, off, lse, dout, DIMS, WINDOW, workspace=torch.empty(8, dtype=torch.uint8),
                 grads=grads)
    q, k, v, off, lse, dout = _inputs(torch.float32, taps=True)
    out, l2 = abi.forward_taps(q, k, v, off, DIMS, WINDOW)
    abi.forward_taps(q, k, v, off, DIMS, WINDOW, out=out, lse=l2)
    g = abi.backward_taps(q, k, v, off, lse, dout, DIMS, WINDOW)
    abi.backward_taps(q, k, v, off, lse, dout, DIMS, WINDOW, workspace=torch.empty(8, dtype=torch.uint8),
                      grads=g)
    x = torch.zeros(N, HEADS * DH, dtype=torch.bfloat16)
    w, b = torch.zeros(HEADS * DH, *WINDOW), torch.zeros(HEADS * DH)
    y = abi.dwconv3d(x, w, b, DIMS)
    abi.dwconv3d(x, w, None, DIMS, add=y, out=y)  # in place into the attention output
    abi.dwconv3d_backward(x, w, y, DIMS)
    off = abi.offset_head(x, w, b, torch.zeros(HEADS * DH, HEADS * 3), torch.zeros(HEADS * 3), DIMS, HEADS)
    assert off.shape == (HEADS, N, 3)
    off = abi.offset_head(x, w, None, torch.zeros(HEADS * DH, HEADS * K * 3), torch.zeros(HEADS * K * 3),
                          DIMS, HEADS, per_tap=True)
    assert off.shape == (HEADS, N, K, 3)
    assert calls == ["dsa3d_forward"] * 3 + ["dsa3d_backward"] * 2 + ["dsa3d_forward_taps"] * 2 + \
        ["dsa3d_backward_taps"] * 2 + ["dsa3d_dwconv3d"] * 2 + ["dsa3d_dwconv3d_backward"] + \
        ["dsa3d_offset_head"] * 2


def test_mismatched_tensors_are_refused_before_any_call(calls):
    q, k, v, off, lse, dout = _inputs()
    bad = [
        lambda: abi.forward(q, k[:-1], v, off, DIMS, WINDOW),                         # k rows
        lambda: abi.forward(q, k, v.float(), off, DIMS, WINDOW),                      # v dtype
        lambda: abi.forward(q, k, v, off.double(), DIMS, WINDOW),                     # offsets dtype
        lambda: abi.forward(q, k, v, off, DIMS, WINDOW, out=torch.empty(N, HEADS, DH)),  # out dtype
        lambda: abi.forward(q, k, v, off, DIMS, WINDOW, lse=torch.empty(HEADS, N + 1)),
        lambda: abi.forward(q, k, v, off, DIMS, WINDOW, workspace=torch.empty(8)),    # not uint8
        lambda: abi.forward(q, k.transpose(1, 2).contiguous().transpose(1, 2), v, off, DIMS, WINDOW),
        lambda: abi.backward(q, k, v, off, lse[:, :-1], dout, DIMS, WINDOW),          # lse
        lambda: abi.backward(q, k, v, off, lse, dout[:, :1], DIMS, WINDOW),           # dout heads
        lambda: abi.backward(q, k, v, off, lse, dout, DIMS, WINDOW,
                             grads=(q.clone(), k.clone(), v.clone(), off[:1].clone())),
        lambda: abi.forward_taps(q, k, v, off, DIMS, WINDOW),                         # per-token offsets
        lambda: abi.backward_taps(q, k, v, torch.zeros(HEADS, N, K, 3), lse, dout.float(), DIMS, WINDOW),
        lambda: abi.dwconv3d(torch.zeros(N, 8), torch.zeros(4, *WINDOW), None, DIMS),  # weight rows
        lambda: abi.dwconv3d(torch.zeros(N, 8), torch.zeros(8, *WINDOW, dtype=torch.float64), None, DIMS),
        lambda: abi.dwconv3d(torch.zeros(N, 8), torch.zeros(8, *WINDOW), torch.zeros(7), DIMS),
        lambda: abi.dwconv3d(torch.zeros(N + 1, 8), torch.zeros(8, *WINDOW), None, DIMS),
        lambda: abi.dwconv3d(torch.zeros(N, 8), torch.zeros(8, *WINDOW), None, DIMS,
                             add=torch.zeros(N, 8, dtype=torch.bfloat16)),
        lambda: abi.dwconv3d_backward(torch.zeros(N, 8), torch.zeros(8, *WINDOW), torch.zeros(N, 4), DIMS),
        lambda: abi.offset_head(torch.zeros(N, 8), torch.zeros(8, *WINDOW), None, torch.zeros(8, 5),
                                torch.zeros(6), DIMS, 2),                             # pw width
        lambda: abi.offset_head(torch.zeros(N, 8), torch.zeros(8, *WINDOW), None, torch.zeros(8, 6),
                                torch.zeros(6, dtype=torch.float64), DIMS, 2),        # pw bias dtype
    ]
    for i, f in enumerate(bad):
        with pytest.raises(ValueError):
            f()
        assert calls == [], i
