/*
 * dsa3d.h -- C ABI of the B200 (sm_100a) 3D Deformable Slide Attention library (libdsa3d.so).
 *
 * Operator: 3D-DSA from MegaSlide-DiT, "Memory-Centric Adaptation and Deformable Local Attention
 * for Efficient Video Diffusion" (arXiv 2607.22696), the 3D-DSA definition: Eq. 1's attention
 * term and the softmax over the k_t x k_h x k_w neighbourhood that follows it.  For every head h
 * and query token p = (t, y, x) of a T x H' x W' token grid:
 *
 *   out[p,h] = sum_tau alpha_tau * Trilinear(V[.,h], p + tau + delta[h,p])
 *   alpha    = softmax_tau( q[p,h] . Trilinear(K[.,h], p + tau + delta[h,p]) / sqrt(dh) )
 *
 * with tau over the centred window [-r_t..r_t] x [-r_h..r_h] x [-r_w..r_w], r = (k-1)/2, and one
 * offset 3-vector delta = (dt, dy, dx) per (token, head).  Positions follow grid_sample's
 * align_corners=True convention (integer coordinate = token centre).  The offset is decoded in
 * single precision: i = floor(delta), f = delta - i (round to nearest), f == 1 carries into i.
 * A tap whose sample position leaves the closed box [0, dim-1] on any axis is masked out of the
 * softmax; trilinear corners outside the volume read as zero.  A query with no valid tap, or with
 * a non-finite offset or |offset| > 2^24, gets out = 0 and lse = -inf and has zero gradient.
 * No causal mask.  The DWConv3D term of Eq. 1 is not computed here: the caller adds it.
 *
 * Layouts (row-major, token n = (t*H' + y)*W' + x, N = T*H'*W'):
 *   q, k, v, out, dout, dq, dk, dv : [N][heads][dh]   in the I/O type (fp32 or bf16)
 *   offsets, doffsets              : [heads][N][3]    fp32, order (dt, dy, dx)
 *   lse                            : [heads][N]       fp32, natural log of the softmax sum
 *
 * Conventions for every entry point:
 *   - All tensor pointers are DEVICE pointers owned by the caller, 16-byte aligned.  Outputs are
 *     fully overwritten (never accumulated) and must not overlap any input or each other.
 *   - Work is enqueued asynchronously on `stream` (a cudaStream_t; 0 = the legacy default
 *     stream).  The returned status covers argument validation and launch errors only; a later
 *     device-side failure surfaces through CUDA's own error reporting or dsa3d_check_device.
 *   - The library allocates no device memory.  The forward (for its tensor-core path) and the
 *     backward take a caller-owned workspace.
 *   - Supported: dh in {32, 64, 128}; odd window sizes 1 <= k <= 2*dim - 1 on each axis;
 *     every extent >= 1; N*heads*dh < 2^62.  Other shapes return DSA3D_ERR_UNSUPPORTED.
 *   - Thread safety: calls on different streams may run concurrently.
 */
#ifndef DSA3D_H
#define DSA3D_H

#include <stddef.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

#define DSA3D_ABI_VERSION 3

typedef enum {
    DSA3D_OK = 0,
    DSA3D_ERR_INVALID_ARGUMENT = 1,   /* null/misaligned pointer, bad extent, aliasing, bad dtype */
    DSA3D_ERR_UNSUPPORTED = 2,        /* valid arguments this library does not handle (dh, window) */
    DSA3D_ERR_WORKSPACE_TOO_SMALL = 3,
    DSA3D_ERR_CUDA = 4,               /* a CUDA runtime call or kernel launch failed */
    DSA3D_ERR_DEVICE_CHECK = 5        /* a kernel recorded a failed internal check */
} dsa3d_status_t;

typedef enum { DSA3D_F32 = 0, DSA3D_BF16 = 1 } dsa3d_dtype_t;

/* DSA3D_ABI_VERSION of the loaded library. */
int dsa3d_abi_version(void);

/* Static, human-readable name of a status code (never NULL). */
const char *dsa3d_status_string(dsa3d_status_t status);

/*
 * Forward: out (and lse, if non-NULL) for every (token, head).
 *   q, k, v  [N][heads][dh] I/O type;  offsets [heads][N][3] fp32;
 *   out      [N][heads][dh] I/O type (written);  lse [heads][N] fp32 (written; may be NULL).
 *   workspace: device scratch of workspace_bytes bytes (contents on entry ignored), or NULL.
 *   F, Hp, Wp: frames and token grid (T, H', W');  kt, kh, kw: window (odd).
 * With bf16 I/O, dh in {64, 128}, kw <= 15 and a workspace of at least
 * dsa3d_forward_workspace_bytes(..., heads = 1, ...) bytes, the forward sorts each head's
 * queries by window origin and runs the tensor-core kernel (heads in groups that fit the
 * workspace).  Otherwise (no workspace, fp32, other shapes) it runs the general CUDA-core kernel;
 * both compute the same function.  A non-NULL workspace smaller than one head's need is
 * DSA3D_ERR_WORKSPACE_TOO_SMALL.  The backward needs lse; pass NULL only for inference.
 * The workspace pair is an addition to the operator's plain signature (tensors, extents, window,
 * dtype, stream): the library allocates no device memory, and the tensor-core path sorts the
 * queries by window origin into caller-owned scratch.  A caller that cannot provide it passes
 * NULL, 0 and gets the same results from the general kernel, several times slower on large
 * problems (the sorted tensor-core forward is the fast path).
 */
dsa3d_status_t dsa3d_forward(const void *q, const void *k, const void *v, const float *offsets,
                             void *out, float *lse, void *workspace, size_t workspace_bytes,
                             int F, int Hp, int Wp, int heads, int dh, int kt, int kh, int kw,
                             dsa3d_dtype_t dtype, cudaStream_t stream);

/*
 * Bytes of forward workspace for all heads in one pass (0 if the shape has no tensor-core path,
 * or is invalid).  Per head: 4 * ((F+kt)(Hp+kh)(Wp+kw) + 1 + 4N) bytes for the sort, plus scan
 * scratch, plus 4 * F * Hp * ceil(Wp/2) * dh bytes for a copy of the head's value rows arranged
 * in pairs of adjacent keys (the operand form of the tensor-core value products).
 */
size_t dsa3d_forward_workspace_bytes(int F, int Hp, int Wp, int heads, int dh, int kt, int kh,
                                     int kw, dsa3d_dtype_t dtype);

/*
 * Bytes of workspace dsa3d_backward needs to process all heads in one pass.  Any workspace of at
 * least the size returned for heads = 1 works (heads are then processed in groups that fit);
 * larger is faster.  Returns 0 when no workspace is needed (fp32 I/O), and 0 for unsupported or
 * invalid shapes (the backward call itself then reports the error).
 */
size_t dsa3d_backward_workspace_bytes(int F, int Hp, int Wp, int heads, int dh, int kt, int kh,
                                      int kw, dsa3d_dtype_t dtype);

/*
 * Backward: gradients of sum(out * dout) with respect to q, k, v and the offsets.
 *   q, k, v, offsets: the forward's inputs;  lse: the forward's lse output (required);
 *   dout [N][heads][dh] I/O type;
 *   dq, dk, dv [N][heads][dh] I/O type (written);  doffsets [heads][N][3] fp32 (written);
 *   workspace: device scratch of workspace_bytes bytes (contents on entry are ignored).
 * The offset gradient is the derivative of the trilinear weights within the cell [i, i+1]; the
 * mask and the integer part of the offset are held fixed.  The softmax Jacobian's row term
 * D = sum_tau P_tau dP_tau is recomputed (it equals dout . out for the unrounded out), so the
 * forward's out is not an input.
 */
dsa3d_status_t dsa3d_backward(const void *q, const void *k, const void *v, const float *offsets,
                              const float *lse, const void *dout, void *dq,
                              void *dk, void *dv, float *doffsets, void *workspace,
                              size_t workspace_bytes, int F, int Hp, int Wp, int heads, int dh,
                              int kt, int kh, int kw, dsa3d_dtype_t dtype, cudaStream_t stream);

/*
 * Backward without a caller workspace (the paper has no counterpart: this is a library-usage
 * entry point).  For callers that cannot allocate device memory or pass a workspace: plugin hosts
 * that own every device allocation and hand the operator only its tensors, fixed call signatures
 * with no workspace argument, and steps that must not pay cudaMalloc's device-wide
 * synchronisation.  Arguments, results and errors are those of dsa3d_backward.
 *
 * Its scratch is a file-scope device array of DSA3D_NOALLOC_SCRATCH_BYTES inside the library,
 * which every GPU that loads the library holds until the process exits, passed to dsa3d_backward
 * as the workspace: the tensor-core path runs when one head's sort and stored splats fit it, the
 * general path when one head's fp32 dK/dV accumulators fit; heads are processed in groups that
 * fit.  A bf16 problem whose single head fits neither -- not the tensor-core path's workspace
 * (dsa3d_backward_workspace_bytes with heads = 1, where that path applies) and not the fp32
 * accumulators (2 * N * dh * 4 bytes) -- is rejected with DSA3D_ERR_WORKSPACE_TOO_SMALL before
 * anything is launched; fp32 I/O needs no scratch.
 * The first call on each device looks up the array's device address (on the current device) and
 * caches it for the life of the process; make that first call before any stream capture.  The
 * cached address belongs to the device's primary context (the one the CUDA runtime uses): after
 * cudaDeviceReset, or under a different context, it is no longer valid.  The array is shared by every call
 * and keeps the previous call's contents (the accumulators are cleared before use): calls that
 * overlap on the GPU -- on different streams, or from different threads -- race on it.
 * The function calls no cudaMalloc, cudaFree or other allocating routine.
 */
#define DSA3D_NOALLOC_SCRATCH_BYTES ((size_t)64 << 20)

dsa3d_status_t dsa3d_backward_noalloc(const void *q, const void *k, const void *v,
                                      const float *offsets, const float *lse,
                                      const void *dout, void *dq, void *dk, void *dv,
                                      float *doffsets, int F, int Hp, int Wp, int heads, int dh,
                                      int kt, int kh, int kw, dsa3d_dtype_t dtype,
                                      cudaStream_t stream);

/*
 * Per-tap offsets: the offset tensor of the 3D-DSA definition (MegaSlide-DiT, Eq. 1) taken
 * literally, one 3-vector per (head, query, window tap) instead of one per (head, query).
 *   offsets, doffsets: [heads][N][K][3] fp32, K = kt*kh*kw, taps in (u, v, w) order with u (the
 *   temporal tap) outermost and w fastest; components (dt, dy, dx).
 * Tap tau of query p samples K and V at p + tau + delta[h,p,tau] (trilinear, align_corners=True).
 * Each tap's offset is decoded on its own as above (floor, fp32 fraction, carry); a non-finite
 * component or |component| > 2^24 masks that tap only, and a tap whose sample position leaves the
 * closed box [0, dim-1] is masked.  A query with no valid tap gets out = 0, lse = -inf and zero
 * gradients.  With every tap's offset equal to one per-token offset the results equal those of
 * dsa3d_forward / dsa3d_backward.  The other arguments, layouts and errors are those of
 * dsa3d_forward and dsa3d_backward.  These entry points always run the general CUDA-core kernels
 * (every tap reads its own 8 corners, so the shared-box tensor-core form does not apply).
 */
dsa3d_status_t dsa3d_forward_taps(const void *q, const void *k, const void *v,
                                  const float *offsets, void *out, float *lse, int F, int Hp,
                                  int Wp, int heads, int dh, int kt, int kh, int kw,
                                  dsa3d_dtype_t dtype, cudaStream_t stream);

/*
 * Workspace of dsa3d_backward_taps for all heads in one pass: the fp32 dK/dV accumulators,
 * 2 * N * dh * 4 bytes per head with bf16 I/O (any multiple of one head's share works; heads are
 * then processed in groups), 0 with fp32 I/O (the gradients accumulate in dk/dv themselves) and
 * for invalid shapes.
 */
size_t dsa3d_backward_taps_workspace_bytes(int F, int Hp, int Wp, int heads, int dh, int kt,
                                           int kh, int kw, dsa3d_dtype_t dtype);

/*
 * Backward with per-tap offsets: gradients of sum(out * dout) with respect to q, k, v and the
 * per-tap offsets (doffsets [heads][N][K][3], the derivative of each tap's trilinear weights
 * within its cell, masks and integer parts held fixed).  Needs the lse of dsa3d_forward_taps;
 * the softmax Jacobian's row term D = sum_tau P dP is recomputed exactly, as in dsa3d_backward.
 * The other arguments and errors are those of dsa3d_backward, with offsets and doffsets
 * [heads][N][K][3].  Its shared memory grows with the tap count (20 bytes per tap per warp):
 * windows of more than about 11,000 taps return DSA3D_ERR_UNSUPPORTED.
 */
dsa3d_status_t dsa3d_backward_taps(const void *q, const void *k, const void *v,
                                   const float *offsets, const float *lse, const void *dout,
                                   void *dq, void *dk, void *dv, float *doffsets, void *workspace,
                                   size_t workspace_bytes, int F, int Hp, int Wp, int heads,
                                   int dh, int kt, int kh, int kw, dsa3d_dtype_t dtype,
                                   cudaStream_t stream);

/*
 * The DWConv3D term of Eq. 1 (MegaSlide-DiT, the 3D-DSA definition): a depthwise 3-D convolution
 * of the layer input X, added to the attention output.
 *   x    [N][C] I/O type (C = heads * dh in the layer; any even C >= 2 here);
 *   weight [C][kt][kh][kw] fp32, bias [C] fp32 (may be NULL);
 *   add  [N][C] I/O type or NULL: added element by element (the attention output
 *        [N][heads][dh] viewed as [N][C]); may equal y (in place);
 *   y    [N][C] I/O type (written):
 *        y[(t,y,x)][c] = bias[c] + sum_{u,v,w} weight[c][u][v][w] * x[(t+u-r_t, y+v-r_h, x+w-r_w)][c]
 *                        (+ add), with x = 0 outside the volume (zero padding, same grid).
 * Cross-correlation (PyTorch's conv3d with groups = C and padding k // 2).  Kernel extents are
 * odd, at most 2 * dim - 1, and kw <= 15.  y must not overlap x, weight or bias.
 */
dsa3d_status_t dsa3d_dwconv3d(const void *x, const float *weight, const float *bias,
                              const void *add, void *y, int F, int Hp, int Wp, int C, int kt,
                              int kh, int kw, dsa3d_dtype_t dtype, cudaStream_t stream);

/*
 * Backward of dsa3d_dwconv3d for the upstream gradient dy [N][C]: dx [N][C] I/O type (the
 * convolution of dy with the flipped kernel), dweight [C][kt][kh][kw] and dbias [C] fp32 (both
 * overwritten; summed over all tokens in fp32).  Outputs must not overlap the inputs or each other.
 */
dsa3d_status_t dsa3d_dwconv3d_backward(const void *x, const float *weight, const void *dy,
                                       void *dx, float *dweight, float *dbias, int F, int Hp,
                                       int Wp, int C, int kt, int kh, int kw, dsa3d_dtype_t dtype,
                                       cudaStream_t stream);

/*
 * The offset network of 3D-DSA (MegaSlide-DiT, the 3D-DSA definition: offsets are predicted by a
 * depthwise 3-D convolution followed by a linear layer), forward:
 *   Z = depthwise conv of x (as dsa3d_dwconv3d, kernel dw_weight [C][kt][kh][kw], bias dw_bias or
 *       NULL), in fp32 in the workspace (N * C * 4 bytes, dsa3d_offset_head_workspace_bytes);
 *   O[n][o] = pw_bias[o] + sum_c Z[n][c] * pw_weight[c][o],  pw_weight [C][heads*taps*3] fp32;
 *   offsets [heads][N][3] (taps = 1) or [heads][N][K][3] (taps = K = kt*kh*kw) fp32 (written),
 *   element (h, n, tau, a) = O[n][(h*taps + tau)*3 + a]: the layouts dsa3d_forward and
 *   dsa3d_forward_taps take.
 * C must be a multiple of 4; the other shape rules are dsa3d_dwconv3d's.  Everything is fp32
 * after the input, since the offsets' integer parts are taken by a floor.
 */
size_t dsa3d_offset_head_workspace_bytes(int F, int Hp, int Wp, int C);

/*
 * Backward of dsa3d_offset_head for the offsets' gradient doffsets (the layout of the offsets;
 * dsa3d_backward / dsa3d_backward_taps write it): dx [N][C] I/O type (the offset network's part
 * of the layer input's gradient), d_dw_weight [C][kt][kh][kw], d_dw_bias [C], d_pw_weight
 * [C][heads*taps*3], d_pw_bias [heads*taps*3], all fp32 and overwritten.  The workspace holds Z
 * (recomputed) and dZ in fp32: dsa3d_offset_head_backward_workspace_bytes = 2 N C 4 bytes.
 * C must be a multiple of 16; the other rules are dsa3d_offset_head's.
 */
size_t dsa3d_offset_head_backward_workspace_bytes(int F, int Hp, int Wp, int C);
dsa3d_status_t dsa3d_offset_head_backward(const void *x, const float *dw_weight,
                                          const float *dw_bias, const float *pw_weight,
                                          const float *doffsets, void *dx, float *d_dw_weight,
                                          float *d_dw_bias, float *d_pw_weight, float *d_pw_bias,
                                          void *workspace, size_t workspace_bytes, int F, int Hp,
                                          int Wp, int C, int heads, int taps, int kt, int kh,
                                          int kw, dsa3d_dtype_t dtype, cudaStream_t stream);
dsa3d_status_t dsa3d_offset_head(const void *x, const float *dw_weight, const float *dw_bias,
                                 const float *pw_weight, const float *pw_bias, float *offsets,
                                 void *workspace, size_t workspace_bytes, int F, int Hp, int Wp,
                                 int C, int heads, int taps, int kt, int kh, int kw,
                                 dsa3d_dtype_t dtype, cudaStream_t stream);

/*
 * Synchronises `stream` and reports DSA3D_ERR_DEVICE_CHECK if any kernel of this library on the
 * current device recorded a failed internal check since the last call (the record is then
 * cleared), DSA3D_ERR_CUDA if the stream reports an error, else DSA3D_OK.
 */
dsa3d_status_t dsa3d_check_device(cudaStream_t stream);

/*
 * Per-kernel timing (profiling aid; off by default).  While enabled, every kernel this library
 * launches is bracketed by two CUDA events recorded on the launch's own stream.
 * dsa3d_timing_read waits for the pending events, adds each launch's duration to the totals of
 * its kernel, and copies up to max_entries totals (kernel name, launch count, total ms) into
 * out; it returns the number of kernels with totals.  dsa3d_timing_reset clears the totals.
 * Host-side state is process-wide and mutex-protected.
 */
typedef struct {
    const char *kernel;  /* static string */
    long long launches;
    double total_ms;
} dsa3d_kernel_time_t;

dsa3d_status_t dsa3d_timing_enable(int enable);
int dsa3d_timing_read(dsa3d_kernel_time_t *out, int max_entries);
void dsa3d_timing_reset(void);

#ifdef __cplusplus
}
#endif

#endif /* DSA3D_H */
