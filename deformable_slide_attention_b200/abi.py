"""ctypes binding over ``libdsa3d.so`` (declared in ``include/dsa3d.h``).

The ``dsa3d_*`` functions here carry the C names and take plain integers for pointers and the
stream; they only marshal arguments.  :func:`forward` and :func:`backward` are conveniences for
torch CUDA tensors: they validate shapes, allocate the outputs (and the backward workspace) with
torch's caching allocator and call the C entry points on the current stream.

There is no fallback: if the library is missing, or no CUDA device is present, every call raises.
"""
from __future__ import annotations

import ctypes
import os
import threading

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_NAME = "libdsa3d.so"
_lib = None
_lock = threading.Lock()

DSA3D_F32 = 0
DSA3D_BF16 = 1

_STATUS = {0: "DSA3D_OK", 1: "DSA3D_ERR_INVALID_ARGUMENT", 2: "DSA3D_ERR_UNSUPPORTED",
           3: "DSA3D_ERR_WORKSPACE_TOO_SMALL", 4: "DSA3D_ERR_CUDA", 5: "DSA3D_ERR_DEVICE_CHECK"}


class Dsa3dError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {_STATUS.get(status, status)} ({dsa3d_status_string(status)})")


def library_path() -> str:
    return os.path.join(_HERE, _LIB_NAME)


def _load():
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        path = library_path()
        if not os.path.exists(path):
            raise RuntimeError(f"{path} is missing: build it with `python -m "
                               "deformable_slide_attention_b200.build` (there is no CPU fallback)")
        lib = ctypes.CDLL(path)
        I, Z, P = ctypes.c_int, ctypes.c_size_t, ctypes.c_void_p
        dims = [I] * 8
        lib.dsa3d_abi_version.restype = I
        lib.dsa3d_abi_version.argtypes = []
        lib.dsa3d_status_string.restype = ctypes.c_char_p
        lib.dsa3d_status_string.argtypes = [I]
        lib.dsa3d_forward.restype = I
        lib.dsa3d_forward.argtypes = [P, P, P, P, P, P, P, Z, *dims, I, P]
        lib.dsa3d_forward_workspace_bytes.restype = Z
        lib.dsa3d_forward_workspace_bytes.argtypes = [*dims, I]
        lib.dsa3d_backward_workspace_bytes.restype = Z
        lib.dsa3d_backward_workspace_bytes.argtypes = [*dims, I]
        lib.dsa3d_backward.restype = I
        lib.dsa3d_backward.argtypes = [P, P, P, P, P, P, P, P, P, P, P, Z, *dims, I, P]
        lib.dsa3d_backward_noalloc.restype = I
        lib.dsa3d_backward_noalloc.argtypes = [P, P, P, P, P, P, P, P, P, P, *dims, I, P]
        lib.dsa3d_forward_taps.restype = I
        lib.dsa3d_forward_taps.argtypes = [P, P, P, P, P, P, *dims, I, P]
        lib.dsa3d_backward_taps_workspace_bytes.restype = Z
        lib.dsa3d_backward_taps_workspace_bytes.argtypes = [*dims, I]
        lib.dsa3d_backward_taps.restype = I
        lib.dsa3d_backward_taps.argtypes = [P, P, P, P, P, P, P, P, P, P, P, Z, *dims, I, P]
        cdims = [I] * 7  # F, Hp, Wp, C, kt, kh, kw
        lib.dsa3d_dwconv3d.restype = I
        lib.dsa3d_dwconv3d.argtypes = [P, P, P, P, P, *cdims, I, P]
        lib.dsa3d_dwconv3d_backward.restype = I
        lib.dsa3d_dwconv3d_backward.argtypes = [P, P, P, P, P, P, *cdims, I, P]
        lib.dsa3d_offset_head_workspace_bytes.restype = Z
        lib.dsa3d_offset_head_workspace_bytes.argtypes = [I, I, I, I]
        lib.dsa3d_offset_head.restype = I
        lib.dsa3d_offset_head.argtypes = [P, P, P, P, P, P, P, Z, I, I, I, I, I, I, I, I, I, I, P]
        lib.dsa3d_offset_head_backward_workspace_bytes.restype = Z
        lib.dsa3d_offset_head_backward_workspace_bytes.argtypes = [I, I, I, I]
        lib.dsa3d_offset_head_backward.restype = I
        lib.dsa3d_offset_head_backward.argtypes = [P] * 11 + [Z] + [I] * 10 + [P]
        lib.dsa3d_check_device.restype = I
        lib.dsa3d_check_device.argtypes = [P]
        lib.dsa3d_timing_enable.restype = I
        lib.dsa3d_timing_enable.argtypes = [I]
        lib.dsa3d_timing_read.restype = I
        lib.dsa3d_timing_read.argtypes = [ctypes.POINTER(KernelTime), I]
        lib.dsa3d_timing_reset.restype = None
        lib.dsa3d_timing_reset.argtypes = []
        _lib = lib
        return lib


class KernelTime(ctypes.Structure):
    _fields_ = [("kernel", ctypes.c_char_p), ("launches", ctypes.c_longlong),
                ("total_ms", ctypes.c_double)]


# --- the C entry points, one to one -----------------------------------------------------------
def dsa3d_abi_version() -> int:
    return _load().dsa3d_abi_version()


def dsa3d_status_string(status: int) -> str:
    try:
        return _load().dsa3d_status_string(int(status)).decode()
    except RuntimeError:
        return _STATUS.get(status, "unknown status")


def dsa3d_forward(q, k, v, offsets, out, lse, workspace, workspace_bytes, F, Hp, Wp, heads, dh,
                  kt, kh, kw, dtype, stream) -> int:
    return _load().dsa3d_forward(q, k, v, offsets, out, lse, workspace, workspace_bytes, F, Hp, Wp,
                                 heads, dh, kt, kh, kw, dtype, stream)


def dsa3d_forward_workspace_bytes(F, Hp, Wp, heads, dh, kt, kh, kw, dtype) -> int:
    return _load().dsa3d_forward_workspace_bytes(F, Hp, Wp, heads, dh, kt, kh, kw, dtype)


def dsa3d_backward_workspace_bytes(F, Hp, Wp, heads, dh, kt, kh, kw, dtype) -> int:
    return _load().dsa3d_backward_workspace_bytes(F, Hp, Wp, heads, dh, kt, kh, kw, dtype)


def dsa3d_backward(q, k, v, offsets, lse, dout, dq, dk, dv, doffsets, workspace, workspace_bytes,
                   F, Hp, Wp, heads, dh, kt, kh, kw, dtype, stream) -> int:
    return _load().dsa3d_backward(q, k, v, offsets, lse, dout, dq, dk, dv, doffsets, workspace,
                                  workspace_bytes, F, Hp, Wp, heads, dh, kt, kh, kw, dtype, stream)


def dsa3d_backward_noalloc(q, k, v, offsets, lse, dout, dq, dk, dv, doffsets, F, Hp, Wp, heads,
                           dh, kt, kh, kw, dtype, stream) -> int:
    """The backward for callers that cannot allocate: its scratch is a fixed device array inside
    the library (see include/dsa3d.h)."""
    return _load().dsa3d_backward_noalloc(q, k, v, offsets, lse, dout, dq, dk, dv, doffsets,
                                          F, Hp, Wp, heads, dh, kt, kh, kw, dtype, stream)


def dsa3d_forward_taps(q, k, v, offsets, out, lse, F, Hp, Wp, heads, dh, kt, kh, kw, dtype,
                       stream) -> int:
    """Forward with per-tap offsets ([heads][N][K][3])."""
    return _load().dsa3d_forward_taps(q, k, v, offsets, out, lse, F, Hp, Wp, heads, dh, kt, kh, kw,
                                      dtype, stream)


def dsa3d_backward_taps_workspace_bytes(F, Hp, Wp, heads, dh, kt, kh, kw, dtype) -> int:
    return _load().dsa3d_backward_taps_workspace_bytes(F, Hp, Wp, heads, dh, kt, kh, kw, dtype)


def dsa3d_backward_taps(q, k, v, offsets, lse, dout, dq, dk, dv, doffsets, workspace,
                        workspace_bytes, F, Hp, Wp, heads, dh, kt, kh, kw, dtype, stream) -> int:
    """Backward with per-tap offsets; doffsets is [heads][N][K][3]."""
    return _load().dsa3d_backward_taps(q, k, v, offsets, lse, dout, dq, dk, dv, doffsets, workspace,
                                       workspace_bytes, F, Hp, Wp, heads, dh, kt, kh, kw, dtype,
                                       stream)


def dsa3d_dwconv3d(x, weight, bias, add, y, F, Hp, Wp, C, kt, kh, kw, dtype, stream) -> int:
    """The DWConv3D term of Eq. 1 (depthwise 3-D convolution, optional fused add)."""
    return _load().dsa3d_dwconv3d(x, weight, bias, add, y, F, Hp, Wp, C, kt, kh, kw, dtype, stream)


def dsa3d_dwconv3d_backward(x, weight, dy, dx, dweight, dbias, F, Hp, Wp, C, kt, kh, kw, dtype,
                            stream) -> int:
    return _load().dsa3d_dwconv3d_backward(x, weight, dy, dx, dweight, dbias, F, Hp, Wp, C, kt, kh,
                                           kw, dtype, stream)


def dsa3d_offset_head_workspace_bytes(F, Hp, Wp, C) -> int:
    return _load().dsa3d_offset_head_workspace_bytes(F, Hp, Wp, C)


def dsa3d_offset_head(x, dw_weight, dw_bias, pw_weight, pw_bias, offsets, workspace,
                      workspace_bytes, F, Hp, Wp, C, heads, taps, kt, kh, kw, dtype, stream) -> int:
    """The offset network's forward: depthwise conv then the pointwise layer, into offsets."""
    return _load().dsa3d_offset_head(x, dw_weight, dw_bias, pw_weight, pw_bias, offsets, workspace,
                                     workspace_bytes, F, Hp, Wp, C, heads, taps, kt, kh, kw, dtype,
                                     stream)


def dsa3d_offset_head_backward_workspace_bytes(F, Hp, Wp, C) -> int:
    return _load().dsa3d_offset_head_backward_workspace_bytes(F, Hp, Wp, C)


def dsa3d_offset_head_backward(x, dw_weight, dw_bias, pw_weight, doffsets, dx, d_dw_weight,
                               d_dw_bias, d_pw_weight, d_pw_bias, workspace, workspace_bytes, F,
                               Hp, Wp, C, heads, taps, kt, kh, kw, dtype, stream) -> int:
    return _load().dsa3d_offset_head_backward(x, dw_weight, dw_bias, pw_weight, doffsets, dx,
                                              d_dw_weight, d_dw_bias, d_pw_weight, d_pw_bias,
                                              workspace, workspace_bytes, F, Hp, Wp, C, heads, taps,
                                              kt, kh, kw, dtype, stream)


def dsa3d_check_device(stream) -> int:
    return _load().dsa3d_check_device(stream)


def dsa3d_timing_enable(enable: bool) -> int:
    return _load().dsa3d_timing_enable(1 if enable else 0)


def dsa3d_timing_read() -> dict:
    """{kernel name: (launches, total ms)} accumulated since the last reset."""
    buf = (KernelTime * 16)()
    n = _load().dsa3d_timing_read(buf, 16)
    return {buf[i].kernel.decode(): (int(buf[i].launches), float(buf[i].total_ms)) for i in range(min(n, 16))}


def dsa3d_timing_reset() -> None:
    _load().dsa3d_timing_reset()


# --- torch conveniences -----------------------------------------------------------------------
def _torch():
    import torch
    return torch


def _dtype_code(t):
    torch = _torch()
    if t.dtype == torch.float32:
        return DSA3D_F32
    if t.dtype == torch.bfloat16:
        return DSA3D_BF16
    raise TypeError(f"3D-DSA takes float32 or bfloat16 tensors, got {t.dtype}")


def _stream_handle(stream):
    torch = _torch()
    s = torch.cuda.current_stream() if stream is None else stream
    return s.cuda_stream


def _check(status, what):
    if status != 0:
        raise Dsa3dError(status, what)


def _need(t, name, shape, dtype):
    """t must be a contiguous tensor of exactly this shape and dtype: the C ABI takes plain
    pointers and reads sizes from the extents, so a mismatched tensor would be read past its end."""
    if t is None:
        raise ValueError(f"{name} is required")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _on_device(ref, *ts):
    """Every tensor given must be a CUDA tensor on ref's device."""
    for t in (ref, *ts):
        if t is not None and (not t.is_cuda or t.device != ref.device):
            raise ValueError("tensors must be CUDA tensors on one device")


def _workspace(ws):
    if ws is not None:
        torch = _torch()
        if ws.dtype != torch.uint8 or not ws.is_contiguous() or ws.dim() != 1:
            raise ValueError("workspace must be a contiguous 1-D uint8 tensor")
    return ws


def _shapes(q, offsets, dims, taps=None):
    """N, heads, dh; offsets must be [heads][N][3], or [heads][N][taps][3] when taps is given."""
    F, Hp, Wp = dims
    N = F * Hp * Wp
    if q.dim() != 3 or q.shape[0] != N:
        raise ValueError(f"q must be [N={N}][heads][dh], got {tuple(q.shape)}")
    heads, dh = q.shape[1], q.shape[2]
    want = (heads, N, 3) if taps is None else (heads, N, taps, 3)
    if tuple(offsets.shape) != want:
        raise ValueError(f"offsets must be {want}, got {tuple(offsets.shape)}")
    return N, heads, dh


def forward(q, k, v, offsets, dims, window, out=None, lse=None, stream=None, want_lse=True,
            workspace="auto"):
    """3D-DSA forward on CUDA tensors.  Returns (out [N][heads][dh], lse [heads][N] or None).

    workspace: "auto" allocates what dsa3d_forward_workspace_bytes asks for (the sorted
    tensor-core path where the shape has one); None runs the general CUDA-core kernel; a uint8
    CUDA tensor is used as given.
    """
    torch = _torch()
    N, heads, dh = _shapes(q, offsets, dims)
    code = _dtype_code(q)
    for name, t in (("q", q), ("k", k), ("v", v)):
        _need(t, name, q.shape, q.dtype)
    _need(offsets, "offsets", offsets.shape, torch.float32)
    if out is None:
        out = torch.empty_like(q)
    _need(out, "out", q.shape, q.dtype)
    if lse is None and want_lse:
        lse = torch.empty((heads, N), dtype=torch.float32, device=q.device)
    if lse is not None:
        _need(lse, "lse", (heads, N), torch.float32)
    if isinstance(workspace, str):
        need = dsa3d_forward_workspace_bytes(*dims, heads, dh, *window, code)
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device) if need else None
    _on_device(q, k, v, offsets, out, lse, _workspace(workspace))
    ws_ptr = workspace.data_ptr() if workspace is not None else None
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check(dsa3d_forward(q.data_ptr(), k.data_ptr(), v.data_ptr(), offsets.data_ptr(), out.data_ptr(),
                         lse.data_ptr() if lse is not None else None, ws_ptr, ws_bytes, *dims, heads,
                         dh, *window, code, _stream_handle(stream)), "dsa3d_forward")
    return out, lse


def backward(q, k, v, offsets, lse, dout, dims, window, workspace=None, stream=None, grads=None):
    """3D-DSA backward on CUDA tensors.  Returns (dq, dk, dv, doffsets)."""
    torch = _torch()
    N, heads, dh = _shapes(q, offsets, dims)
    code = _dtype_code(q)
    _check_backward_tensors(q, k, v, offsets, lse, dout, heads, N)
    if grads is None:
        grads = (torch.empty_like(q), torch.empty_like(k), torch.empty_like(v),
                 torch.empty_like(offsets))
    dq, dk, dv, doff = grads
    for name, t in (("dq", dq), ("dk", dk), ("dv", dv)):
        _need(t, name, q.shape, q.dtype)
    _need(doff, "doffsets", offsets.shape, torch.float32)
    need = dsa3d_backward_workspace_bytes(*dims, heads, dh, *window, code)
    if workspace is None and need:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    _on_device(q, k, v, offsets, lse, dout, dq, dk, dv, doff, _workspace(workspace))
    ws_ptr = workspace.data_ptr() if workspace is not None else None
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check(dsa3d_backward(q.data_ptr(), k.data_ptr(), v.data_ptr(), offsets.data_ptr(),
                          lse.data_ptr(), dout.data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(),
                          doff.data_ptr(), ws_ptr, ws_bytes, *dims, heads, dh, *window, code,
                          _stream_handle(stream)), "dsa3d_backward")
    return dq, dk, dv, doff


def _check_backward_tensors(q, k, v, offsets, lse, dout, heads, N):
    torch = _torch()
    for name, t in (("q", q), ("k", k), ("v", v), ("dout", dout)):
        _need(t, name, q.shape, q.dtype)
    _need(offsets, "offsets", offsets.shape, torch.float32)
    _need(lse, "lse", (heads, N), torch.float32)


def _taps(window):
    kt, kh, kw = window
    return kt * kh * kw


def forward_taps(q, k, v, offsets, dims, window, out=None, lse=None, stream=None, want_lse=True):
    """3D-DSA forward with per-tap offsets ([heads][N][kt*kh*kw][3]) on CUDA tensors.
    Returns (out [N][heads][dh], lse [heads][N] or None)."""
    torch = _torch()
    N, heads, dh = _shapes(q, offsets, dims, _taps(window))
    code = _dtype_code(q)
    for name, t in (("q", q), ("k", k), ("v", v)):
        _need(t, name, q.shape, q.dtype)
    _need(offsets, "offsets", offsets.shape, torch.float32)
    if out is None:
        out = torch.empty_like(q)
    _need(out, "out", q.shape, q.dtype)
    if lse is None and want_lse:
        lse = torch.empty((heads, N), dtype=torch.float32, device=q.device)
    if lse is not None:
        _need(lse, "lse", (heads, N), torch.float32)
    _on_device(q, k, v, offsets, out, lse)
    _check(dsa3d_forward_taps(q.data_ptr(), k.data_ptr(), v.data_ptr(), offsets.data_ptr(),
                              out.data_ptr(), lse.data_ptr() if lse is not None else None, *dims,
                              heads, dh, *window, code, _stream_handle(stream)), "dsa3d_forward_taps")
    return out, lse


def backward_taps(q, k, v, offsets, lse, dout, dims, window, workspace=None, stream=None, grads=None):
    """3D-DSA backward with per-tap offsets.  Returns (dq, dk, dv, doffsets [heads][N][K][3])."""
    torch = _torch()
    N, heads, dh = _shapes(q, offsets, dims, _taps(window))
    code = _dtype_code(q)
    _check_backward_tensors(q, k, v, offsets, lse, dout, heads, N)
    if grads is None:
        grads = (torch.empty_like(q), torch.empty_like(k), torch.empty_like(v),
                 torch.empty_like(offsets))
    dq, dk, dv, doff = grads
    for name, t in (("dq", dq), ("dk", dk), ("dv", dv)):
        _need(t, name, q.shape, q.dtype)
    _need(doff, "doffsets", offsets.shape, torch.float32)
    need = dsa3d_backward_taps_workspace_bytes(*dims, heads, dh, *window, code)
    if workspace is None and need:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    _on_device(q, k, v, offsets, lse, dout, dq, dk, dv, doff, _workspace(workspace))
    ws_ptr = workspace.data_ptr() if workspace is not None else None
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check(dsa3d_backward_taps(q.data_ptr(), k.data_ptr(), v.data_ptr(), offsets.data_ptr(),
                               lse.data_ptr(), dout.data_ptr(), dq.data_ptr(), dk.data_ptr(),
                               dv.data_ptr(), doff.data_ptr(), ws_ptr, ws_bytes, *dims, heads, dh,
                               *window, code, _stream_handle(stream)), "dsa3d_backward_taps")
    return dq, dk, dv, doff


def _conv_shapes(x, weight, dims):
    """(C, kt, kh, kw) of a convolution call; x must be [N][C] with N = F*Hp*Wp and weight
    [C][kt][kh][kw] fp32, both contiguous."""
    torch = _torch()
    N = dims[0] * dims[1] * dims[2]
    if x.dim() != 2 or x.shape[0] != N:
        raise ValueError(f"x must be [N={N}][C], got {tuple(x.shape)}")
    _need(x, "x", x.shape, x.dtype)
    C = x.shape[1]
    if weight.dim() != 4 or weight.shape[0] != C:
        raise ValueError(f"weight must be [C={C}][kt][kh][kw], got {tuple(weight.shape)}")
    _need(weight, "weight", weight.shape, torch.float32)
    return (C, *weight.shape[1:])


def dwconv3d(x, weight, bias, dims, add=None, out=None, stream=None):
    """Depthwise 3-D convolution of x [N][C] with weight [C][kt][kh][kw] (fp32) and bias [C]
    (fp32 or None), plus add [N][C] if given (the attention output viewed as [N][C]; out may be
    add itself).  Returns out [N][C]."""
    torch = _torch()
    code = _dtype_code(x)
    C, kt, kh, kw = _conv_shapes(x, weight, dims)
    if bias is not None:
        _need(bias, "bias", (C,), torch.float32)
    if add is not None:
        _need(add, "add", x.shape, x.dtype)
    if out is None:
        out = torch.empty_like(x)
    _need(out, "out", x.shape, x.dtype)
    _on_device(x, weight, bias, add, out)
    _check(dsa3d_dwconv3d(x.data_ptr(), weight.data_ptr(), bias.data_ptr() if bias is not None else None,
                          add.data_ptr() if add is not None else None, out.data_ptr(), *dims, C, kt,
                          kh, kw, code, _stream_handle(stream)), "dsa3d_dwconv3d")
    return out


def dwconv3d_backward(x, weight, dy, dims, stream=None):
    """Gradients of sum(dwconv3d(x, weight, bias) * dy): (dx [N][C], dweight, dbias [C] fp32)."""
    torch = _torch()
    code = _dtype_code(x)
    C, kt, kh, kw = _conv_shapes(x, weight, dims)
    _need(dy, "dy", x.shape, x.dtype)
    _on_device(x, weight, dy)
    dx = torch.empty_like(x)
    dw = torch.empty_like(weight, dtype=torch.float32)
    db = torch.empty(x.shape[1], dtype=torch.float32, device=x.device)
    _check(dsa3d_dwconv3d_backward(x.data_ptr(), weight.data_ptr(), dy.data_ptr(), dx.data_ptr(),
                                   dw.data_ptr(), db.data_ptr(), *dims, C, kt, kh, kw, code,
                                   _stream_handle(stream)), "dsa3d_dwconv3d_backward")
    return dx, dw, db


def offset_head(x, dw_weight, dw_bias, pw_weight, pw_bias, dims, heads, per_tap=False, stream=None):
    """The offset network's forward on CUDA tensors: offsets [heads][N][3] (or [heads][N][K][3]
    with per_tap) from x [N][C], dw_weight [C][kt][kh][kw], dw_bias [C] or None, pw_weight
    [C][heads * (K) * 3] and pw_bias (fp32)."""
    torch = _torch()
    code = _dtype_code(x)
    C, kt, kh, kw = _conv_shapes(x, dw_weight, dims)
    taps = kt * kh * kw if per_tap else 1
    width = heads * taps * 3
    if dw_bias is not None:
        _need(dw_bias, "dw_bias", (C,), torch.float32)
    _need(pw_weight, "pw_weight", (C, width), torch.float32)
    _need(pw_bias, "pw_bias", (width,), torch.float32)
    N = x.shape[0]
    offsets = torch.empty((heads, N, taps, 3) if per_tap else (heads, N, 3), dtype=torch.float32,
                          device=x.device)
    ws = torch.empty(dsa3d_offset_head_workspace_bytes(*dims, C), dtype=torch.uint8, device=x.device)
    _on_device(x, dw_weight, dw_bias, pw_weight, pw_bias)
    _check(dsa3d_offset_head(x.data_ptr(), dw_weight.data_ptr(),
                             dw_bias.data_ptr() if dw_bias is not None else None,
                             pw_weight.data_ptr(), pw_bias.data_ptr(), offsets.data_ptr(),
                             ws.data_ptr(), ws.numel(), *dims, C, heads, taps, kt, kh, kw, code,
                             _stream_handle(stream)), "dsa3d_offset_head")
    return offsets


def offset_head_backward(x, dw_weight, dw_bias, pw_weight, doffsets, dims, heads, per_tap=False,
                         stream=None):
    """Gradients of sum(offsets * doffsets) for offsets = offset_head(...): (dx [N][C] in x's
    dtype, d dw_weight, d dw_bias, d pw_weight, d pw_bias, all fp32 but dx)."""
    torch = _torch()
    code = _dtype_code(x)
    C, kt, kh, kw = _conv_shapes(x, dw_weight, dims)
    taps = kt * kh * kw if per_tap else 1
    width = heads * taps * 3
    N = x.shape[0]
    if dw_bias is not None:
        _need(dw_bias, "dw_bias", (C,), torch.float32)
    _need(pw_weight, "pw_weight", (C, width), torch.float32)
    _need(doffsets, "doffsets", (heads, N, taps, 3) if per_tap else (heads, N, 3), torch.float32)
    _on_device(x, dw_weight, dw_bias, pw_weight, doffsets)
    dx = torch.empty_like(x)
    grads = (torch.empty_like(dw_weight), torch.empty(C, dtype=torch.float32, device=x.device),
             torch.empty_like(pw_weight), torch.empty(width, dtype=torch.float32, device=x.device))
    ws = torch.empty(dsa3d_offset_head_backward_workspace_bytes(*dims, C), dtype=torch.uint8,
                     device=x.device)
    _check(dsa3d_offset_head_backward(x.data_ptr(), dw_weight.data_ptr(),
                                      dw_bias.data_ptr() if dw_bias is not None else None,
                                      pw_weight.data_ptr(), doffsets.data_ptr(), dx.data_ptr(),
                                      *(t.data_ptr() for t in grads), ws.data_ptr(), ws.numel(), *dims,
                                      C, heads, taps, kt, kh, kw, code, _stream_handle(stream)),
           "dsa3d_offset_head_backward")
    return (dx, *grads)
