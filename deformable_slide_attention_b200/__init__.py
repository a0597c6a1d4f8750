"""B200-native 3D Deformable Slide Attention (3D-DSA).

The operator is the motion-adaptive local attention of MegaSlide-DiT (arXiv 2607.22696, the
3D-DSA definition, Eq. 1): every query token attends to a k_t x k_h x k_w window of keys and
values, slid by a per-(token, head) offset and sampled by trilinear interpolation.

The compute runs in hand-written sm_100a CUDA kernels behind a C ABI (``include/dsa3d.h``,
``libdsa3d.so``); :mod:`deformable_slide_attention_b200.abi` is the thin ctypes binding over it.
Importing this package does not load the library; the first call does, and fails loudly if the
library is missing.  There is no CPU fallback.
"""
from .abi import (  # noqa: F401
    DSA3D_BF16,
    DSA3D_F32,
    Dsa3dError,
    dsa3d_abi_version,
    dsa3d_backward,
    dsa3d_backward_workspace_bytes,
    dsa3d_check_device,
    dsa3d_forward,
    dsa3d_forward_workspace_bytes,
    dsa3d_status_string,
    dsa3d_timing_enable,
    dsa3d_timing_read,
    dsa3d_timing_reset,
    backward,
    forward,
    library_path,
)
