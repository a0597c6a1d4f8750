"""CPU oracle for 3D Deformable Slide Attention (3D-DSA).

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline
leg may import this package; the product path never does.  It shares no code with the CUDA path.

The arithmetic lives in ``dsa3d_oracle.c`` (plain C, double precision, one tap at a time).  This
module compiles it with gcc on first use and marshals numpy/torch CPU arrays through ctypes.

Source of the operator: MegaSlide-DiT (arXiv 2607.22696), the 3D-DSA definition (Eq. 1 and the
softmax over the k_t x k_h x k_w neighbourhood that follows it).  The readings the paper leaves
open are listed in the C file's header (R1..R10).  Besides the attention term, the module holds
the other two parts of Eq. 1's layer: the DWConv3D term (a depthwise 3-D convolution, R9) and the
offset network (a depthwise 3-D convolution and a pointwise linear layer, R10).

Parity pins: every routine here is pinned, the attention by ``tests/test_oracle_pins.py``
against brute-force dense attention, torch's ``grid_sample``, finite differences and an
independent torch autograd restatement, and the convolution and offset network by
``tests/test_oracle_layer_pins.py`` against torch's conv3d and autograd, closed forms and
finite differences through the whole layer.  The one unpinned reading is the score scale (R3,
1/sqrt(dh)); the convolution's kernel extent (R9, R10) is a reading the pins take as given.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "dsa3d_oracle.c")
_LIB_PATH = os.path.join(_HERE, "libdsa3d_oracle.so")
_lib = None
_lock = threading.Lock()

IO_F32 = 0
IO_BF16 = 1


def build(force: bool = False) -> str:
    """Compile the oracle shared library with gcc (OpenMP, strict IEEE arithmetic)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-ffp-contract=off", "-fno-fast-math",
               "-std=c11", "-Wall", "-o", tmp, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is None:
            # DSA3D_ORACLE_LIB lets the oracle's own mutation test load a deliberately broken copy
            path = os.environ.get("DSA3D_ORACLE_LIB") or build()
            lib = ctypes.CDLL(path)
            i64p = ctypes.POINTER(ctypes.c_int64)
            vp = ctypes.c_void_p
            dims = [ctypes.c_int] * 8
            lib.dsa3d_oracle_forward.restype = ctypes.c_int64
            lib.dsa3d_oracle_forward.argtypes = [ctypes.c_int, vp, vp, vp, vp, *dims, i64p,
                                                 ctypes.c_int64, vp, vp, ctypes.c_int]
            lib.dsa3d_oracle_backward.restype = ctypes.c_int
            lib.dsa3d_oracle_backward.argtypes = [ctypes.c_int, vp, vp, vp, vp, vp, *dims, i64p,
                                                  ctypes.c_int64, vp, vp, i64p, ctypes.c_int64,
                                                  vp, vp, ctypes.c_int]
            lib.dsa3d_oracle_forward_taps.restype = ctypes.c_int64
            lib.dsa3d_oracle_forward_taps.argtypes = lib.dsa3d_oracle_forward.argtypes
            lib.dsa3d_oracle_backward_taps.restype = ctypes.c_int
            lib.dsa3d_oracle_backward_taps.argtypes = lib.dsa3d_oracle_backward.argtypes
            cdims = [ctypes.c_int] * 7  # F, Hp, Wp, C, kt, kh, kw
            lib.dsa3d_oracle_dwconv3d.restype = ctypes.c_int
            lib.dsa3d_oracle_dwconv3d.argtypes = [ctypes.c_int, vp, vp, vp, *cdims, vp, ctypes.c_int]
            lib.dsa3d_oracle_dwconv3d_backward.restype = ctypes.c_int
            lib.dsa3d_oracle_dwconv3d_backward.argtypes = [ctypes.c_int, vp, vp, vp, *cdims, vp,
                                                           vp, vp, ctypes.c_int]
            lib.dsa3d_oracle_tap.restype = ctypes.c_int
            lib.dsa3d_oracle_tap.argtypes = [ctypes.c_int, vp, vp, *dims, ctypes.c_int,
                                             ctypes.c_int64, ctypes.c_int, i64p, vp, vp, vp]
            _lib = lib
    return _lib


def _as_io(x):
    """Return (contiguous numpy array, io code) for an fp32 or bf16 array (numpy or torch)."""
    try:
        import torch
        if isinstance(x, torch.Tensor):
            x = x.detach().cpu().contiguous()
            if x.dtype == torch.bfloat16:
                return x.view(torch.int16).numpy().view(np.uint16), IO_BF16
            if x.dtype == torch.float32:
                return x.numpy(), IO_F32
            raise TypeError(f"oracle inputs must be float32 or bfloat16, got {x.dtype}")
    except ImportError:  # pragma: no cover
        pass
    x = np.ascontiguousarray(x)
    if x.dtype == np.float32:
        return x, IO_F32
    if x.dtype == np.uint16:
        return x, IO_BF16
    raise TypeError(f"oracle inputs must be float32 or bf16 bits (uint16), got {x.dtype}")


def _f32(x):
    try:
        import torch
        if isinstance(x, torch.Tensor):
            x = x.detach().cpu().contiguous().numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.ascontiguousarray(x, dtype=np.float32)


def _ptr(a):
    return ctypes.c_void_p(a.ctypes.data) if a is not None and a.size else ctypes.c_void_p(0)


def _items(items, total):
    if items is None:
        items = np.arange(total, dtype=np.int64)
    items = np.ascontiguousarray(items, dtype=np.int64)
    return items, items.ctypes.data_as(ctypes.POINTER(ctypes.c_int64))


def _threads(n):
    return int(n) if n else (os.cpu_count() or 1)


def forward(q, k, v, offsets, dims, window, items=None, threads=None, return_reads=False,
            per_tap=False):
    """Forward of 3D-DSA.

    q, k, v: [N][heads][dh] (fp32 or bf16); offsets: [heads][N][3] fp32, or with ``per_tap``
    [heads][N][K][3] (one offset per window tap, K = kt*kh*kw, reading R8); dims = (F, Hp, Wp);
    window = (kt, kh, kw).  ``items`` lists h*N + n; None means every (h, n), head-major.
    Returns (out [n_items][dh] float64, lse [n_items] float64).
    """
    qa, io = _as_io(q)
    ka, io_k = _as_io(k)
    va, io_v = _as_io(v)
    if not (io == io_k == io_v):
        raise TypeError("q, k, v must share one dtype")
    off = _f32(offsets)
    N = dims[0] * dims[1] * dims[2]
    heads, dh = qa.shape[-2], qa.shape[-1]
    it, itp = _items(items, N * heads)
    out = np.zeros((len(it), dh), np.float64)
    lse = np.zeros(len(it), np.float64)
    _check_offsets(off, heads, N, window, per_tap)
    fn = _load().dsa3d_oracle_forward_taps if per_tap else _load().dsa3d_oracle_forward
    reads = fn(io, _ptr(qa), _ptr(ka), _ptr(va), _ptr(off), *dims, heads, dh, *window, itp, len(it),
               _ptr(out), _ptr(lse), _threads(threads))
    if reads < 0:
        raise ValueError("oracle forward rejected its arguments")
    return (out, lse, reads) if return_reads else (out, lse)


def backward(q, k, v, offsets, dout, dims, window, q_items=None, k_items=None, threads=None,
             per_tap=False):
    """Backward of 3D-DSA.

    Returns (dq [n_q][dh], doff [n_q][3], dk [n_k][dh], dv [n_k][dh]) in float64; with
    ``per_tap`` (offsets [heads][N][K][3]) doff is [n_q][K][3].  ``q_items`` and ``k_items`` list
    h*N + n; None means every item.  dk/dv at a key gather the contributions of every query of
    that head.
    """
    qa, io = _as_io(q)
    ka, _ = _as_io(k)
    va, _ = _as_io(v)
    da, io_d = _as_io(dout)
    if io_d != io:
        raise TypeError("dout must share the dtype of q")
    off = _f32(offsets)
    N = dims[0] * dims[1] * dims[2]
    heads, dh = qa.shape[-2], qa.shape[-1]
    qi, qip = _items(q_items, N * heads)
    ki, kip = _items(k_items, N * heads)
    _check_offsets(off, heads, N, window, per_tap)
    K = window[0] * window[1] * window[2]
    dq = np.zeros((len(qi), dh), np.float64)
    doff = np.zeros((len(qi), K, 3) if per_tap else (len(qi), 3), np.float64)
    dk = np.zeros((len(ki), dh), np.float64)
    dv = np.zeros((len(ki), dh), np.float64)
    fn = _load().dsa3d_oracle_backward_taps if per_tap else _load().dsa3d_oracle_backward
    rc = fn(io, _ptr(qa), _ptr(ka), _ptr(va), _ptr(off), _ptr(da), *dims, heads, dh, *window, qip,
            len(qi), _ptr(dq), _ptr(doff), kip, len(ki), _ptr(dk), _ptr(dv), _threads(threads))
    if rc != 0:
        raise ValueError("oracle backward rejected its arguments")
    return dq, doff, dk, dv


def _check_offsets(off, heads, N, window, per_tap):
    K = window[0] * window[1] * window[2]
    want = heads * N * (K if per_tap else 1) * 3
    if off.size != want:
        raise ValueError(f"offsets hold {off.size} values, expected {want}")


def tap(src, offsets, dims, window, h, n, tau):
    """One tap: (valid, base[3] int64, frac[3] float32, sample[dh], dsample[3][dh])."""
    sa, io = _as_io(src)
    off = _f32(offsets)
    heads, dh = sa.shape[-2], sa.shape[-1]
    base = np.zeros(3, np.int64)
    frac = np.zeros(3, np.float32)
    samp = np.zeros(dh, np.float64)
    dsamp = np.zeros((3, dh), np.float64)
    rc = _load().dsa3d_oracle_tap(io, _ptr(sa), _ptr(off), *dims, heads, dh, *window, h, n, tau,
                                  base.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)), _ptr(frac),
                                  _ptr(samp), _ptr(dsamp))
    if rc < 0:
        raise ValueError("oracle tap rejected its arguments")
    return bool(rc), base, frac, samp, dsamp


def full_forward(q, k, v, offsets, dims, window, threads=None, per_tap=False):
    """Forward over every (n, h), returned in the [N][heads][dh] / [heads][N] layouts."""
    N = dims[0] * dims[1] * dims[2]
    heads, dh = q.shape[-2], q.shape[-1]
    out, lse = forward(q, k, v, offsets, dims, window, None, threads, per_tap=per_tap)
    out = out.reshape(heads, N, dh).transpose(1, 0, 2).copy()
    return out, lse.reshape(heads, N)


def full_backward(q, k, v, offsets, dout, dims, window, threads=None, per_tap=False):
    """Backward over every item, returned as dq/dk/dv [N][heads][dh] and doff [heads][N][3]
    (per_tap: [heads][N][K][3])."""
    N = dims[0] * dims[1] * dims[2]
    heads, dh = q.shape[-2], q.shape[-1]
    dq, doff, dk, dv = backward(q, k, v, offsets, dout, dims, window, None, None, threads,
                                per_tap=per_tap)
    r = lambda a: a.reshape(heads, N, dh).transpose(1, 0, 2).copy()
    return r(dq), doff.reshape((heads, N, -1, 3) if per_tap else (heads, N, 3)), r(dk), r(dv)


# --- the DWConv3D term and the offset network (R9, R10) ----------------------------------------
def _conv_args(x, weight, bias, dims):
    xa, io = _as_io(x)
    F, Hp, Wp = dims
    N = F * Hp * Wp
    if xa.ndim != 2 or xa.shape[0] != N:
        raise ValueError(f"x must be [N={N}][C], got {xa.shape}")
    C = xa.shape[1]
    w = _f32(weight)
    if w.ndim != 4 or w.shape[0] != C:
        raise ValueError(f"weight must be [C={C}][kt][kh][kw], got {w.shape}")
    b = None if bias is None else _f32(bias).reshape(C)
    return xa, io, w, b, C, w.shape[1:]


def dwconv3d(x, weight, bias, dims, threads=None):
    """Depthwise 3-D convolution (R9): x [N][C] (fp32 or bf16), weight [C][kt][kh][kw] fp32,
    bias [C] fp32 or None.  Returns Y [N][C] float64 (zero padding, output grid = token grid)."""
    xa, io, w, b, C, (kt, kh, kw) = _conv_args(x, weight, bias, dims)
    y = np.zeros((xa.shape[0], C), np.float64)
    rc = _load().dsa3d_oracle_dwconv3d(io, _ptr(xa), _ptr(w), _ptr(b), *dims, C, kt, kh, kw,
                                       _ptr(y), _threads(threads))
    if rc != 0:
        raise ValueError("dsa3d_oracle_dwconv3d: bad arguments")
    return y


def dwconv3d_backward(x, weight, dy, dims, threads=None):
    """Gradients of sum(Y * dy) for Y = dwconv3d(x, weight, bias): (dx [N][C], dweight
    [C][kt][kh][kw], dbias [C]), all float64."""
    xa, io, w, _, C, (kt, kh, kw) = _conv_args(x, weight, None, dims)
    g = np.ascontiguousarray(dy, dtype=np.float64).reshape(xa.shape[0], C)
    dx = np.zeros((xa.shape[0], C), np.float64)
    dw = np.zeros(w.shape, np.float64)
    db = np.zeros(C, np.float64)
    rc = _load().dsa3d_oracle_dwconv3d_backward(io, _ptr(xa), _ptr(w), _ptr(g), *dims, C, kt, kh,
                                                kw, _ptr(dx), _ptr(dw), _ptr(db), _threads(threads))
    if rc != 0:
        raise ValueError("dsa3d_oracle_dwconv3d_backward: bad arguments")
    return dx, dw, db


def _offset_layout(flat, heads, taps):
    """[N][heads * (taps) * 3] -> [heads][N][3] or [heads][N][taps][3]."""
    N = flat.shape[0]
    if taps is None:
        return np.ascontiguousarray(flat.reshape(N, heads, 3).transpose(1, 0, 2))
    return np.ascontiguousarray(flat.reshape(N, heads, taps, 3).transpose(1, 0, 2, 3))


def offset_head(x, dw_weight, dw_bias, pw_weight, pw_bias, dims, heads, taps=None, threads=None):
    """The offset network (R10): Z = dwconv3d(x, dw_weight, dw_bias), then the pointwise layer
    O = Z @ pw_weight + pw_bias with pw_weight [C][heads * 3] (per token) or [C][heads * taps * 3]
    (per tap).  Returns the offsets in the attention's layout, [heads][N][3] or
    [heads][N][taps][3], float64 (the attention takes them rounded to fp32)."""
    z = dwconv3d(x, dw_weight, dw_bias, dims, threads)
    pw = np.asarray(_f32(pw_weight), np.float64)
    width = heads * 3 * (1 if taps is None else taps)
    if pw.shape != (z.shape[1], width):
        raise ValueError(f"pw_weight must be [C][{width}], got {pw.shape}")
    flat = z @ pw + np.asarray(_f32(pw_bias), np.float64).reshape(width)
    return _offset_layout(flat, heads, taps)


def offset_head_backward(x, dw_weight, dw_bias, pw_weight, doffsets, dims, threads=None):
    """Gradients of sum(offsets * doffsets) for offsets = offset_head(...): (dx [N][C],
    d dw_weight, d dw_bias, d pw_weight [C][width], d pw_bias [width]), float64.  doffsets is in
    the attention's layout ([heads][N][3] or [heads][N][taps][3])."""
    z = dwconv3d(x, dw_weight, dw_bias, dims, threads)
    g = np.asarray(doffsets, np.float64)
    N = z.shape[0]
    # back to the pointwise layer's [N][heads * (taps) * 3] order
    g_flat = np.ascontiguousarray(np.moveaxis(g, 1, 0)).reshape(N, -1)
    pw = np.asarray(_f32(pw_weight), np.float64)
    d_pw = z.T @ g_flat
    d_pb = g_flat.sum(axis=0)
    dz = g_flat @ pw.T
    dx, d_dw, d_db = dwconv3d_backward(x, dw_weight, dz, dims, threads)
    return dx, d_dw, d_db, d_pw, d_pb
