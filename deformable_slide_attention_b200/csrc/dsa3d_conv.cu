// dsa3d_conv.cu -- C ABI of the DWConv3D term of Eq. 1 (MegaSlide-DiT, the 3D-DSA definition):
// argument validation, launch configuration and the extern "C" entry points dsa3d_dwconv3d and
// dsa3d_dwconv3d_backward declared in include/dsa3d.h.  The kernels are in dsa3d_conv.cuh.  A
// translation unit of its own, next to dsa3d.cu; this file allocates no device memory.
#include <cuda_runtime.h>

#include <algorithm>
#include <climits>
#include <cstdint>

#include "dsa3d.h"
#include "dsa3d_conv.cuh"
#include "dsa3d_pointwise.cuh"
#include "dsa3d_timing.cuh"

namespace dsa3d {
namespace {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

struct Range {
  uintptr_t lo, hi;
};
Range range_of(const void* p, size_t bytes) {
  const uintptr_t a = reinterpret_cast<uintptr_t>(p);
  return {a, a + bytes};
}
bool overlap(Range a, Range b) { return a.lo < b.hi && b.lo < a.hi; }

size_t elem_size(dsa3d_dtype_t t) { return t == DSA3D_F32 ? 4 : 2; }

struct DeviceInfo {
  int sms = 0;
};
DeviceInfo device_info() {
  DeviceInfo d;
  int dev = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev);
  return d;
}

// Blocks of `threads` for `work` items, at most per_sm_cap per SM (the kernels stride the rest).
int grid_for(int64_t work, int threads, int per_sm_cap) {
  const DeviceInfo d = device_info();
  int64_t grid = (work + threads - 1) / threads;
  const int64_t cap = (int64_t)(d.sms > 0 ? d.sms : 1) * per_sm_cap;
  if (grid > cap) grid = cap;
  if (grid < 1) grid = 1;
  return (int)grid;
}

// --- depthwise 3-D convolution (the DWConv3D term of Eq. 1) -----------------------------------------
ConvGeo make_conv_geo(int F, int Hp, int Wp, int C, int kt, int kh, int kw) {
  ConvGeo g;
  g.F = F; g.Hp = Hp; g.Wp = Wp; g.C = C; g.kt = kt; g.kh = kh; g.kw = kw;
  g.N = (int64_t)F * Hp * Wp;
  return g;
}

dsa3d_status_t check_conv_shape(int F, int Hp, int Wp, int C, int kt, int kh, int kw,
                                dsa3d_dtype_t dtype) {
  if (dtype != DSA3D_F32 && dtype != DSA3D_BF16) return DSA3D_ERR_INVALID_ARGUMENT;
  if (F < 1 || Hp < 1 || Wp < 1 || C < 2) return DSA3D_ERR_INVALID_ARGUMENT;
  const int dims[3] = {F, Hp, Wp}, win[3] = {kt, kh, kw};
  for (int a = 0; a < 3; a++) {
    if (win[a] < 1 || (win[a] & 1) == 0) return DSA3D_ERR_INVALID_ARGUMENT;
    if ((int64_t)win[a] > 2 * (int64_t)dims[a] - 1) return DSA3D_ERR_UNSUPPORTED;
  }
  if (kw > 15 || (C & 1)) return DSA3D_ERR_UNSUPPORTED;  // kernel rows are unrolled; channel pairs
  if ((int64_t)F * Hp * Wp >= (int64_t(1) << 31)) return DSA3D_ERR_UNSUPPORTED;
  return DSA3D_OK;
}

// The forward (and dX, flip = 1): when the kernel's taps fit in shared memory and the grid in one
// dimension, the strip-pair kernel for C a multiple of 32 and the staged kernel for the other
// channel counts; else the global-memory one.
template <typename T, int KW, typename OutT = T>
dsa3d_status_t dwconv_launch_kw(const ConvGeo& g, const void* x, const float* w, const float* b,
                                const void* add, void* y, int flip, cudaStream_t st) {
  const int64_t units = (int64_t)g.F * ((g.Hp + 1) / 2) * ((g.Wp + kConvStrip - 1) / kConvStrip);
  const int64_t groups = (g.C / 2 + kConvGroupPairs - 1) / kConvGroupPairs;
  const int64_t sw_blocks = (units + kConvSwUnits - 1) / kConvSwUnits * groups;
  const int K = g.kt * g.kh * KW;
  const T* xt = static_cast<const T*>(x);
  const OutT* at = static_cast<const OutT*>(add);
  OutT* yt = static_cast<OutT*>(y);
  const int64_t sw2_units =
      (int64_t)g.F * ((g.Hp + kSw2Rows - 1) / kSw2Rows) * ((g.Wp + 2 * kConvStrip - 1) / (2 * kConvStrip));
  const int64_t sw2_grid = (sw2_units + kSw2Units - 1) / kSw2Units * (g.C / (2 * kSw2Pairs));
  if (K <= kConvSwMaxTaps && g.C % (2 * kSw2Pairs) == 0 && sw2_grid <= INT_MAX) {
    // strip pairs with a warp-shared row ring
    const size_t smem = conv_sw2_weight_bytes(K) + kConvSwWarps * Sw2Ring<T, KW>::warp_bytes();
    if (cudaFuncSetAttribute(dsa3d_dwconv3d_sw2_kernel<T, KW, OutT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem) != cudaSuccess)
      return DSA3D_ERR_CUDA;
    TimedLaunch tl(kKernDwconvSw2, st);
    dsa3d_dwconv3d_sw2_kernel<T, KW, OutT><<<(unsigned)sw2_grid, kConvSwWarps * 32, smem, st>>>(
        xt, w, b, at, yt, g, flip);
    const bool launched = cudaGetLastError() == cudaSuccess;
    return (tl.finish() && launched) ? DSA3D_OK : DSA3D_ERR_CUDA;
  }
  if (K <= kConvSwMaxTaps && sw_blocks <= INT_MAX) {
    // the staged kernel may take up to conv_sw_bytes(kConvSwMaxTaps) of dynamic shared memory
    if (cudaFuncSetAttribute(dsa3d_dwconv3d_sw_kernel<T, KW, OutT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)conv_sw_bytes(kConvSwMaxTaps)) != cudaSuccess)
      return DSA3D_ERR_CUDA;
    TimedLaunch tl(kKernDwconvSw, st);
    dsa3d_dwconv3d_sw_kernel<T, KW, OutT><<<(unsigned)sw_blocks, kConvSwWarps * 32, conv_sw_bytes(K), st>>>(
        xt, w, b, at, yt, g, flip);
    const bool launched = cudaGetLastError() == cudaSuccess;
    return (tl.finish() && launched) ? DSA3D_OK : DSA3D_ERR_CUDA;
  }
  const int64_t items = units * (g.C / 2);
  TimedLaunch tl(kKernDwconv, st);
  dsa3d_dwconv3d_kernel<T, KW, OutT><<<grid_for(items, kConvFwdThreads, 8), kConvFwdThreads, 0, st>>>(
      xt, w, b, at, yt, g, flip);
  const bool launched = cudaGetLastError() == cudaSuccess;
  return (tl.finish() && launched) ? DSA3D_OK : DSA3D_ERR_CUDA;
}

template <typename T, typename OutT = T>
dsa3d_status_t dwconv_launch(const ConvGeo& g, const void* x, const float* w, const float* b,
                             const void* add, void* y, int flip, cudaStream_t st) {
  switch (g.kw) {
    case 1: return dwconv_launch_kw<T, 1, OutT>(g, x, w, b, add, y, flip, st);
    case 3: return dwconv_launch_kw<T, 3, OutT>(g, x, w, b, add, y, flip, st);
    case 5: return dwconv_launch_kw<T, 5, OutT>(g, x, w, b, add, y, flip, st);
    case 7: return dwconv_launch_kw<T, 7, OutT>(g, x, w, b, add, y, flip, st);
    case 9: return dwconv_launch_kw<T, 9, OutT>(g, x, w, b, add, y, flip, st);
    case 11: return dwconv_launch_kw<T, 11, OutT>(g, x, w, b, add, y, flip, st);
    case 13: return dwconv_launch_kw<T, 13, OutT>(g, x, w, b, add, y, flip, st);
    case 15: return dwconv_launch_kw<T, 15, OutT>(g, x, w, b, add, y, flip, st);
    default: return DSA3D_ERR_UNSUPPORTED;
  }
}

// dY frames per dW work item: about 8 items per resident thread (resident = the threads the GPU
// holds at once), so that the items' last round leaves little of the GPU idle, each item long
// enough that its final atomics are a small share of its work.
int dw_frames_per_item(const ConvGeo& g, int64_t resident) {
  const int64_t per_run = dw_items(g, g.F);  // items when one run covers every frame
  int64_t runs = resident * 8 / (per_run > 0 ? per_run : 1);
  if (runs < 1) runs = 1;
  if (runs > g.F) runs = g.F;
  return (int)((g.F + runs - 1) / runs);
}

// dW and db: a grid of at most the blocks the GPU holds at once, striding over the items.
template <typename T, int KW, typename TD, bool Coop>
dsa3d_status_t dwconv_dw_launch_kernel(const ConvGeo& g, const void* x, const void* dy, float* dw,
                                       float* db, cudaStream_t st) {
  auto* kern = dsa3d_dwconv3d_dw_kernel<T, KW, TD, Coop>;
  // a staging ring per warp
  const size_t smem = (size_t)(kConvDwThreads / 32) * DwRing<T, TD, KW>::warp_bytes();
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
    return DSA3D_ERR_CUDA;
  int per_sm = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kConvDwThreads, smem) != cudaSuccess)
    return DSA3D_ERR_CUDA;
  if (per_sm < 1) per_sm = 1;
  const int sms = std::max(device_info().sms, 1);
  const int fpi = dw_frames_per_item(g, (int64_t)sms * per_sm * kConvDwThreads);
  const int64_t items = dw_items(g, fpi);
  TimedLaunch tl(kKernDwconvDw, st);
  kern<<<grid_for(items, kConvDwThreads, per_sm), kConvDwThreads, smem, st>>>(
      static_cast<const T*>(x), static_cast<const TD*>(dy), dw, db, g, fpi);
  const bool launched = cudaGetLastError() == cudaSuccess;
  return (tl.finish() && launched) ? DSA3D_OK : DSA3D_ERR_CUDA;
}

// The warp-cooperative copies when every warp is 32 aligned channel pairs of one work item: C a
// multiple of 64 (the items run channel pairs fastest, and blocks and the grid stride are whole
// warps).
template <typename T, int KW, typename TD = T>
dsa3d_status_t dwconv_dw_launch_kw(const ConvGeo& g, const void* x, const void* dy, float* dw,
                                   float* db, cudaStream_t st) {
  static_assert(kConvDwThreads % 32 == 0, "whole warps");
  if (g.C % 64 == 0) return dwconv_dw_launch_kernel<T, KW, TD, true>(g, x, dy, dw, db, st);
  return dwconv_dw_launch_kernel<T, KW, TD, false>(g, x, dy, dw, db, st);
}

template <typename T, typename TD = T>
dsa3d_status_t dwconv_dw_launch(const ConvGeo& g, const void* x, const void* dy, float* dw,
                                float* db, cudaStream_t st) {
  switch (g.kw) {
    case 1: return dwconv_dw_launch_kw<T, 1, TD>(g, x, dy, dw, db, st);
    case 3: return dwconv_dw_launch_kw<T, 3, TD>(g, x, dy, dw, db, st);
    case 5: return dwconv_dw_launch_kw<T, 5, TD>(g, x, dy, dw, db, st);
    case 7: return dwconv_dw_launch_kw<T, 7, TD>(g, x, dy, dw, db, st);
    case 9: return dwconv_dw_launch_kw<T, 9, TD>(g, x, dy, dw, db, st);
    case 11: return dwconv_dw_launch_kw<T, 11, TD>(g, x, dy, dw, db, st);
    case 13: return dwconv_dw_launch_kw<T, 13, TD>(g, x, dy, dw, db, st);
    case 15: return dwconv_dw_launch_kw<T, 15, TD>(g, x, dy, dw, db, st);
    default: return DSA3D_ERR_UNSUPPORTED;
  }
}

size_t offset_head_ws_bytes(int F, int Hp, int Wp, int C) {
  return ((size_t)F * Hp * Wp * C * 4 + 15) & ~size_t(15);
}

}  // namespace
}  // namespace dsa3d

using namespace dsa3d;

extern "C" {

dsa3d_status_t dsa3d_dwconv3d(const void* x, const float* weight, const float* bias,
                              const void* add, void* y, int F, int Hp, int Wp, int C, int kt, int kh,
                              int kw, dsa3d_dtype_t dtype, cudaStream_t stream) {
  dsa3d_status_t rc = check_conv_shape(F, Hp, Wp, C, kt, kh, kw, dtype);
  if (rc != DSA3D_OK) return rc;
  if (!x || !weight || !y) return DSA3D_ERR_INVALID_ARGUMENT;
  const void* al[] = {x, y};
  for (const void* p : al)
    if (!aligned16(p)) return DSA3D_ERR_INVALID_ARGUMENT;
  if ((add && !aligned16(add)) || (reinterpret_cast<uintptr_t>(weight) & 3u) ||
      (bias && (reinterpret_cast<uintptr_t>(bias) & 7u)))
    return DSA3D_ERR_INVALID_ARGUMENT;
  const ConvGeo g = make_conv_geo(F, Hp, Wp, C, kt, kh, kw);
  const size_t tb = (size_t)g.N * C * elem_size(dtype);
  const Range ry = range_of(y, tb);
  // y is written while neighbouring rows of x are still read; add may be y itself
  if (overlap(range_of(x, tb), ry) || overlap(range_of(weight, (size_t)C * kt * kh * kw * 4), ry) ||
      (bias && overlap(range_of(bias, (size_t)C * 4), ry)))
    return DSA3D_ERR_INVALID_ARGUMENT;
  if (add && add != y && overlap(range_of(add, tb), ry)) return DSA3D_ERR_INVALID_ARGUMENT;
  if (dtype == DSA3D_F32) return dwconv_launch<float>(g, x, weight, bias, add, y, 0, stream);
  return dwconv_launch<__nv_bfloat16>(g, x, weight, bias, add, y, 0, stream);
}

dsa3d_status_t dsa3d_dwconv3d_backward(const void* x, const float* weight, const void* dy, void* dx,
                                       float* dweight, float* dbias, int F, int Hp, int Wp, int C,
                                       int kt, int kh, int kw, dsa3d_dtype_t dtype,
                                       cudaStream_t stream) {
  dsa3d_status_t rc = check_conv_shape(F, Hp, Wp, C, kt, kh, kw, dtype);
  if (rc != DSA3D_OK) return rc;
  if (!x || !weight || !dy || !dx || !dweight || !dbias) return DSA3D_ERR_INVALID_ARGUMENT;
  const void* al[] = {x, dy, dx};
  for (const void* p : al)
    if (!aligned16(p)) return DSA3D_ERR_INVALID_ARGUMENT;
  if ((reinterpret_cast<uintptr_t>(weight) & 3u) || (reinterpret_cast<uintptr_t>(dweight) & 3u) ||
      (reinterpret_cast<uintptr_t>(dbias) & 7u))
    return DSA3D_ERR_INVALID_ARGUMENT;
  const ConvGeo g = make_conv_geo(F, Hp, Wp, C, kt, kh, kw);
  const size_t tb = (size_t)g.N * C * elem_size(dtype), wb = (size_t)C * kt * kh * kw * 4;
  const Range ins[] = {range_of(x, tb), range_of(weight, wb), range_of(dy, tb)};
  const Range outs[] = {range_of(dx, tb), range_of(dweight, wb), range_of(dbias, (size_t)C * 4)};
  for (int i = 0; i < 3; i++) {
    for (const Range& r : ins)
      if (overlap(r, outs[i])) return DSA3D_ERR_INVALID_ARGUMENT;
    for (int j = i + 1; j < 3; j++)
      if (overlap(outs[i], outs[j])) return DSA3D_ERR_INVALID_ARGUMENT;
  }
  if (cudaMemsetAsync(dweight, 0, wb, stream) != cudaSuccess ||
      cudaMemsetAsync(dbias, 0, (size_t)C * 4, stream) != cudaSuccess)
    return DSA3D_ERR_CUDA;
  if (dtype == DSA3D_F32) {
    if ((rc = dwconv_launch<float>(g, dy, weight, nullptr, nullptr, dx, 1, stream)) != DSA3D_OK) return rc;
    return dwconv_dw_launch<float>(g, x, dy, dweight, dbias, stream);
  }
  if ((rc = dwconv_launch<__nv_bfloat16>(g, dy, weight, nullptr, nullptr, dx, 1, stream)) != DSA3D_OK)
    return rc;
  return dwconv_dw_launch<__nv_bfloat16>(g, x, dy, dweight, dbias, stream);
}

size_t dsa3d_offset_head_workspace_bytes(int F, int Hp, int Wp, int C) {
  if (F < 1 || Hp < 1 || Wp < 1 || C < 1) return 0;
  return offset_head_ws_bytes(F, Hp, Wp, C);
}

dsa3d_status_t dsa3d_offset_head(const void* x, const float* dw_weight, const float* dw_bias,
                                 const float* pw_weight, const float* pw_bias, float* offsets,
                                 void* workspace, size_t workspace_bytes, int F, int Hp, int Wp,
                                 int C, int heads, int taps, int kt, int kh, int kw,
                                 dsa3d_dtype_t dtype, cudaStream_t stream) {
  dsa3d_status_t rc = check_conv_shape(F, Hp, Wp, C, kt, kh, kw, dtype);
  if (rc != DSA3D_OK) return rc;
  if (heads < 1 || (taps != 1 && taps != kt * kh * kw)) return DSA3D_ERR_INVALID_ARGUMENT;
  if (C % 4) return DSA3D_ERR_UNSUPPORTED;  // the pointwise layer reads 4 channels at a time
  if (!x || !dw_weight || !pw_weight || !pw_bias || !offsets || !workspace)
    return DSA3D_ERR_INVALID_ARGUMENT;
  if (!aligned16(x) || !aligned16(workspace) || (reinterpret_cast<uintptr_t>(offsets) & 3u) ||
      (reinterpret_cast<uintptr_t>(dw_weight) & 3u) || (reinterpret_cast<uintptr_t>(pw_weight) & 3u) ||
      (reinterpret_cast<uintptr_t>(pw_bias) & 3u) || (dw_bias && (reinterpret_cast<uintptr_t>(dw_bias) & 7u)))
    return DSA3D_ERR_INVALID_ARGUMENT;
  if (workspace_bytes < offset_head_ws_bytes(F, Hp, Wp, C)) return DSA3D_ERR_WORKSPACE_TOO_SMALL;
  const ConvGeo g = make_conv_geo(F, Hp, Wp, C, kt, kh, kw);
  const int width = heads * taps * 3;
  const size_t tb = (size_t)g.N * C * elem_size(dtype);
  const size_t ob = (size_t)g.N * width * 4;
  const Range ins[] = {range_of(x, tb), range_of(dw_weight, (size_t)C * kt * kh * kw * 4),
                       range_of(dw_bias, dw_bias ? (size_t)C * 4 : 0),
                       range_of(pw_weight, (size_t)C * width * 4), range_of(pw_bias, (size_t)width * 4)};
  const Range ro = range_of(offsets, ob), rw = range_of(workspace, workspace_bytes);
  for (const Range& r : ins)
    if (overlap(r, ro) || overlap(r, rw)) return DSA3D_ERR_INVALID_ARGUMENT;
  if (overlap(ro, rw)) return DSA3D_ERR_INVALID_ARGUMENT;
  float* z = static_cast<float*>(workspace);
  rc = (dtype == DSA3D_F32)
           ? dwconv_launch<float, float>(g, x, dw_weight, dw_bias, nullptr, z, 0, stream)
           : dwconv_launch<__nv_bfloat16, float>(g, x, dw_weight, dw_bias, nullptr, z, 0, stream);
  if (rc != DSA3D_OK) return rc;
  const int64_t items = (g.N + kPwTokens - 1) / kPwTokens * width;
  TimedLaunch tl(kKernPointwise, stream);
  dsa3d_pointwise_offsets_kernel<<<grid_for(items, 256, 8), 256, 0, stream>>>(
      z, pw_weight, pw_bias, offsets, C, width, taps * 3, g.N);
  const bool launched = cudaGetLastError() == cudaSuccess;
  return (tl.finish() && launched) ? DSA3D_OK : DSA3D_ERR_CUDA;
}

size_t dsa3d_offset_head_backward_workspace_bytes(int F, int Hp, int Wp, int C) {
  if (F < 1 || Hp < 1 || Wp < 1 || C < 1) return 0;
  return 2 * offset_head_ws_bytes(F, Hp, Wp, C);
}

dsa3d_status_t dsa3d_offset_head_backward(const void* x, const float* dw_weight, const float* dw_bias,
                                          const float* pw_weight, const float* doffsets, void* dx,
                                          float* d_dw_weight, float* d_dw_bias, float* d_pw_weight,
                                          float* d_pw_bias, void* workspace, size_t workspace_bytes,
                                          int F, int Hp, int Wp, int C, int heads, int taps, int kt,
                                          int kh, int kw, dsa3d_dtype_t dtype, cudaStream_t stream) {
  dsa3d_status_t rc = check_conv_shape(F, Hp, Wp, C, kt, kh, kw, dtype);
  if (rc != DSA3D_OK) return rc;
  if (heads < 1 || (taps != 1 && taps != kt * kh * kw)) return DSA3D_ERR_INVALID_ARGUMENT;
  if (C % kPwChannels) return DSA3D_ERR_UNSUPPORTED;  // 16-channel groups in the weight gradient
  if (!x || !dw_weight || !pw_weight || !doffsets || !dx || !d_dw_weight || !d_dw_bias ||
      !d_pw_weight || !d_pw_bias || !workspace)
    return DSA3D_ERR_INVALID_ARGUMENT;
  const void* al16[] = {x, dx, workspace};
  for (const void* p : al16)
    if (!aligned16(p)) return DSA3D_ERR_INVALID_ARGUMENT;
  const void* al4[] = {dw_weight, pw_weight, doffsets, d_dw_weight, d_pw_weight, d_pw_bias};
  for (const void* p : al4)
    if (reinterpret_cast<uintptr_t>(p) & 3u) return DSA3D_ERR_INVALID_ARGUMENT;
  if ((reinterpret_cast<uintptr_t>(d_dw_bias) & 7u) || (dw_bias && (reinterpret_cast<uintptr_t>(dw_bias) & 7u)))
    return DSA3D_ERR_INVALID_ARGUMENT;
  const size_t zb = offset_head_ws_bytes(F, Hp, Wp, C);
  if (workspace_bytes < 2 * zb) return DSA3D_ERR_WORKSPACE_TOO_SMALL;
  const ConvGeo g = make_conv_geo(F, Hp, Wp, C, kt, kh, kw);
  const int width = heads * taps * 3;
  const size_t tb = (size_t)g.N * C * elem_size(dtype), wb = (size_t)C * kt * kh * kw * 4;
  const size_t pwb = (size_t)C * width * 4, ob = (size_t)g.N * width * 4;
  const Range ins[] = {range_of(x, tb), range_of(dw_weight, wb), range_of(dw_bias, dw_bias ? (size_t)C * 4 : 0),
                       range_of(pw_weight, pwb), range_of(doffsets, ob)};
  const Range outs[] = {range_of(dx, tb), range_of(d_dw_weight, wb), range_of(d_dw_bias, (size_t)C * 4),
                        range_of(d_pw_weight, pwb), range_of(d_pw_bias, (size_t)width * 4),
                        range_of(workspace, workspace_bytes)};
  for (int i = 0; i < 6; i++) {
    for (const Range& r : ins)
      if (overlap(r, outs[i])) return DSA3D_ERR_INVALID_ARGUMENT;
    for (int j = i + 1; j < 6; j++)
      if (overlap(outs[i], outs[j])) return DSA3D_ERR_INVALID_ARGUMENT;
  }
  float* z = static_cast<float*>(workspace);
  float* dz = reinterpret_cast<float*>(static_cast<char*>(workspace) + zb);
  if (cudaMemsetAsync(d_dw_weight, 0, wb, stream) != cudaSuccess ||
      cudaMemsetAsync(d_dw_bias, 0, (size_t)C * 4, stream) != cudaSuccess ||
      cudaMemsetAsync(d_pw_weight, 0, pwb, stream) != cudaSuccess ||
      cudaMemsetAsync(d_pw_bias, 0, (size_t)width * 4, stream) != cudaSuccess)
    return DSA3D_ERR_CUDA;
  const bool f32 = dtype == DSA3D_F32;
  // Z again (the forward's convolution), then the pointwise layer's dZ and weight gradient
  rc = f32 ? dwconv_launch<float, float>(g, x, dw_weight, dw_bias, nullptr, z, 0, stream)
           : dwconv_launch<__nv_bfloat16, float>(g, x, dw_weight, dw_bias, nullptr, z, 0, stream);
  if (rc != DSA3D_OK) return rc;
  {
    const int64_t items = (g.N + kPwTokens - 1) / kPwTokens * C;
    TimedLaunch tl(kKernPointwiseDz, stream);
    dsa3d_pointwise_dz_kernel<<<grid_for(items, 256, 8), 256, 0, stream>>>(doffsets, pw_weight, dz, C,
                                                                          width, taps * 3, g.N);
    if (cudaGetLastError() != cudaSuccess || !tl.finish()) return DSA3D_ERR_CUDA;
  }
  {
    const int64_t per_item = 256;
    const int64_t items = (g.N + per_item - 1) / per_item * (C / kPwChannels) * width;
    TimedLaunch tl(kKernPointwiseDw, stream);
    dsa3d_pointwise_dw_kernel<<<grid_for(items, 256, 8), 256, 0, stream>>>(
        z, doffsets, d_pw_weight, d_pw_bias, C, width, taps * 3, g.N, per_item);
    if (cudaGetLastError() != cudaSuccess || !tl.finish()) return DSA3D_ERR_CUDA;
  }
  // the depthwise convolution's backward for the fp32 dZ
  rc = f32 ? dwconv_launch<float, float>(g, dz, dw_weight, nullptr, nullptr, dx, 1, stream)
           : dwconv_launch<float, __nv_bfloat16>(g, dz, dw_weight, nullptr, nullptr, dx, 1, stream);
  if (rc != DSA3D_OK) return rc;
  return f32 ? dwconv_dw_launch<float, float>(g, x, dz, d_dw_weight, d_dw_bias, stream)
             : dwconv_dw_launch<__nv_bfloat16, float>(g, x, dz, d_dw_weight, d_dw_bias, stream);
}

}  // extern "C"
