// dsa3d_conv.cuh -- the DWConv3D term of Eq. 1 (MegaSlide-DiT, arXiv 2607.22696, the 3D-DSA
// definition) and the first layer of the offset network: a depthwise 3-D convolution of the layer
// input X [N][C] (token n = (t*Hp + y)*Wp + x, channels fastest) with a kernel W [C][kt][kh][kw]
// (fp32), a bias per channel, stride 1 and zero padding to the same token grid:
//
//   Y[(t, y, x)][c] = b[c] + sum_{u,v,w} W[c][u][v][w] * X[(t + u - r_t, y + v - r_h, x + w - r_w)][c]
//
// (cross-correlation; X = 0 outside the volume).  The backward's dX is the same operation on dY
// with the kernel flipped on every axis; dW[c][u][v][w] = sum_p dY[p][c] X[p + tap offset][c].
//
// At the window's extent (3 x 9 x 9) the convolution does 2 C K flop per token for 4 C bytes of
// bf16 traffic: about 120 flop per byte, so it is bound by the fp32 FMA pipes, not by HBM.  The
// kernels block registers along x: a thread owns one channel pair (a 4-byte bf16x2 or 8-byte
// float2 load, consecutive threads on consecutive pairs, so a warp's loads are one coalesced
// 128- or 256-byte row segment) and a strip of kConvStrip outputs along x.  Per kernel row
// (u, v) it loads the kConvStrip + KW - 1 input values of the row once and the KW weights of
// the row once, and does kConvStrip * KW FMAs per channel from registers.
//
// The per-thread arithmetic (conv_strip, dw_row) is __host__ __device__ code so that a host
// harness can run exactly these routines on the CPU.
#pragma once

#include <cuda_bf16.h>
#include <stdint.h>

// Threads per block of the convolution kernels and, if DSA3D_CONV_MINB is defined, the minimum
// resident blocks per SM asked of the compiler (a register cap).  Without it the launch bounds
// name the block size alone (the compiler's own register choice).
#ifndef DSA3D_CONV_THREADS
#define DSA3D_CONV_THREADS 256
#endif
#ifdef DSA3D_CONV_MINB
#define DSA3D_CONV_BOUNDS __launch_bounds__(DSA3D_CONV_THREADS, DSA3D_CONV_MINB)
#else
#define DSA3D_CONV_BOUNDS __launch_bounds__(DSA3D_CONV_THREADS)
#endif

namespace dsa3d {

constexpr int kConvStrip = 8;  // outputs along x per thread
constexpr int kConvThreads = DSA3D_CONV_THREADS;
static_assert(kConvThreads % 32 == 0 && kConvThreads >= 32 && kConvThreads <= 1024,
              "DSA3D_CONV_THREADS: whole warps, at most 1024 threads per block");

struct ConvGeo {
  int F, Hp, Wp, C;
  int kt, kh, kw;
  int64_t N;
};

// Two adjacent channels of one token row, as fp32.
__host__ __device__ __forceinline__ void conv_load2(const float* p, float& a, float& b) {
#ifdef __CUDA_ARCH__
  const float2 v = __ldg(reinterpret_cast<const float2*>(p));
#else
  const float2 v = *reinterpret_cast<const float2*>(p);
#endif
  a = v.x;
  b = v.y;
}
__host__ __device__ __forceinline__ void conv_load2(const __nv_bfloat16* p, float& a, float& b) {
#ifdef __CUDA_ARCH__
  const unsigned u = __ldg(reinterpret_cast<const unsigned*>(p));
#else
  const unsigned u = *reinterpret_cast<const unsigned*>(p);
#endif
  union {
    unsigned i;
    float f;
  } lo, hi;
  lo.i = u << 16;
  hi.i = u & 0xffff0000u;
  a = lo.f;
  b = hi.f;
}
__host__ __device__ __forceinline__ void conv_store2(float* p, float a, float b) {
  *reinterpret_cast<float2*>(p) = make_float2(a, b);
}
__host__ __device__ __forceinline__ void conv_store2(__nv_bfloat16* p, float a, float b) {
  *reinterpret_cast<__nv_bfloat162*>(p) = __floats2bfloat162_rn(a, b);
}
__host__ __device__ __forceinline__ float conv_ldw(const float* p) {
#ifdef __CUDA_ARCH__
  return __ldg(p);
#else
  return *p;
#endif
}

// Convolution sums of channel pair c2 (channels 2 c2 and 2 c2 + 1) for the outputs
// (t, y, x0 + i), i < kConvStrip, added into acc[i][0..1].  flip: use W[c][kt-1-u][kh-1-v][kw-1-w]
// (the backward's dX).  KW = the kernel's width kw (a compile-time constant).
template <typename T, int KW>
__host__ __device__ __forceinline__ void conv_strip(const T* __restrict__ x, const float* __restrict__ w,
                                                    const ConvGeo& g, int t, int y, int x0, int c2,
                                                    bool flip, float (&acc)[kConvStrip][2]) {
  const int rt = (g.kt - 1) / 2, rh = (g.kh - 1) / 2, rw = (KW - 1) / 2;
  const int64_t K = (int64_t)g.kt * g.kh * KW;
  const float* w0 = w + (int64_t)(2 * c2) * K;
  const float* w1 = w0 + K;
  for (int u = 0; u < g.kt; u++) {
    const int ts = t + u - rt;
    if (ts < 0 || ts >= g.F) continue;
    for (int v = 0; v < g.kh; v++) {
      const int ys = y + v - rh;
      if (ys < 0 || ys >= g.Hp) continue;
      // the kernel row's weights (flipped for the transposed convolution)
      const int64_t wrow = flip ? ((int64_t)(g.kt - 1 - u) * g.kh + (g.kh - 1 - v)) * KW
                                : ((int64_t)u * g.kh + v) * KW;
      float wa[KW], wb[KW];
#pragma unroll
      for (int j = 0; j < KW; j++) {
        const int jj = flip ? KW - 1 - j : j;
        wa[j] = conv_ldw(w0 + wrow + jj);
        wb[j] = conv_ldw(w1 + wrow + jj);
      }
      const T* row = x + ((int64_t)ts * g.Hp + ys) * g.Wp * g.C + 2 * c2;
      // input column x0 - rw + j feeds output x0 + i through tap j - i
#pragma unroll
      for (int j = 0; j < kConvStrip + KW - 1; j++) {
        const int xs = x0 - rw + j;
        float a = 0.f, b = 0.f;
        if (xs >= 0 && xs < g.Wp) conv_load2(row + (int64_t)xs * g.C, a, b);
#pragma unroll
        for (int i = 0; i < kConvStrip; i++) {
          if (j - i >= 0 && j - i < KW) {
            acc[i][0] = fmaf(wa[j - i], a, acc[i][0]);
            acc[i][1] = fmaf(wb[j - i], b, acc[i][1]);
          }
        }
      }
    }
  }
}

// The contribution of one output strip (t, y, x0 .. x0 + kConvStrip - 1) to the weight gradient
// of kernel row (u, v) of channel pair c2: dwr[j][k] += sum_i dY[(t, y, x0 + i)][2 c2 + k] *
// X[(t + u - r_t, y + v - r_h, x0 + i + j - r_w)][2 c2 + k]; and, with db != nullptr, the bias
// gradient db[k] += sum_i dY[...].  Outputs past the volume's last column are skipped.  TD: the
// type of dY (the input's, or fp32 for the offset network's backward).
template <typename T, int KW, typename TD = T>
__host__ __device__ __forceinline__ void dw_row(const T* __restrict__ x, const TD* __restrict__ dy,
                                                const ConvGeo& g, int t, int y, int x0, int c2, int u,
                                                int v, float (&dwr)[KW][2], float* db) {
  const int rt = (g.kt - 1) / 2, rh = (g.kh - 1) / 2, rw = (KW - 1) / 2;
  float ga[kConvStrip], gb[kConvStrip];
  const TD* dyrow = dy + ((int64_t)t * g.Hp + y) * g.Wp * g.C + 2 * c2;
#pragma unroll
  for (int i = 0; i < kConvStrip; i++) {
    ga[i] = gb[i] = 0.f;
    if (x0 + i < g.Wp) conv_load2(dyrow + (int64_t)(x0 + i) * g.C, ga[i], gb[i]);
    if (db) {
      db[0] += ga[i];
      db[1] += gb[i];
    }
  }
  const int ts = t + u - rt, ys = y + v - rh;
  if (ts < 0 || ts >= g.F || ys < 0 || ys >= g.Hp) return;
  const T* row = x + ((int64_t)ts * g.Hp + ys) * g.Wp * g.C + 2 * c2;
#pragma unroll
  for (int j = 0; j < kConvStrip + KW - 1; j++) {
    const int xs = x0 - rw + j;
    float a = 0.f, b = 0.f;
    if (xs >= 0 && xs < g.Wp) conv_load2(row + (int64_t)xs * g.C, a, b);
#pragma unroll
    for (int i = 0; i < kConvStrip; i++) {
      if (j - i >= 0 && j - i < KW) {
        dwr[j - i][0] = fmaf(ga[i], a, dwr[j - i][0]);
        dwr[j - i][1] = fmaf(gb[i], b, dwr[j - i][1]);
      }
    }
  }
}

#ifdef __CUDACC__
// Y = conv(X) (+ bias) (+ add): one thread per (strip, channel pair), channel pairs fastest.
// add (nullable) is added element by element (the attention output of Eq. 1; may equal y).
// OutT: the output type (the input's, or fp32 for the offset network's first layer).
template <typename T, int KW, typename OutT = T>
__global__ void DSA3D_CONV_BOUNDS
    dsa3d_dwconv3d_kernel(const T* __restrict__ x, const float* __restrict__ w,
                          const float* __restrict__ bias, const OutT* add, OutT* y,
                          const ConvGeo g, const int flip) {
  const int pairs = g.C / 2;
  const int nxs = (g.Wp + kConvStrip - 1) / kConvStrip;
  const int64_t items = (int64_t)g.F * g.Hp * nxs * pairs;
  for (int64_t it = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; it < items;
       it += (int64_t)gridDim.x * blockDim.x) {
    const int c2 = (int)(it % pairs);
    const int64_t s = it / pairs;
    const int x0 = (int)(s % nxs) * kConvStrip;
    const int yy = (int)((s / nxs) % g.Hp);
    const int t = (int)(s / ((int64_t)nxs * g.Hp));
    float acc[kConvStrip][2];
    const float b0 = bias ? __ldg(bias + 2 * c2) : 0.f, b1 = bias ? __ldg(bias + 2 * c2 + 1) : 0.f;
#pragma unroll
    for (int i = 0; i < kConvStrip; i++) {
      acc[i][0] = b0;
      acc[i][1] = b1;
    }
    conv_strip<T, KW>(x, w, g, t, yy, x0, c2, flip != 0, acc);
    const int64_t base = (((int64_t)t * g.Hp + yy) * g.Wp + x0) * g.C + 2 * c2;
#pragma unroll
    for (int i = 0; i < kConvStrip; i++) {
      if (x0 + i >= g.Wp) break;
      const int64_t o = base + (int64_t)i * g.C;
      float a = acc[i][0], b = acc[i][1];
      if (add) {
        float p, q;
        conv_load2(add + o, p, q);
        a += p;
        b += q;
      }
      conv_store2(y + o, a, b);
    }
  }
}

// dW (and db): one thread per (channel pair, kernel row (u, v), range of strips); fp32 partial
// sums reduced with atomics into dweight [C][kt][kh][kw] and dbias [C] (both zeroed before).
template <typename T, int KW, typename TD = T>
__global__ void DSA3D_CONV_BOUNDS
    dsa3d_dwconv3d_dw_kernel(const T* __restrict__ x, const TD* __restrict__ dy, float* dweight,
                             float* dbias, const ConvGeo g, const int strips_per_item) {
  const int pairs = g.C / 2;
  const int rows = g.kt * g.kh;
  const int nxs = (g.Wp + kConvStrip - 1) / kConvStrip;
  const int64_t strips = (int64_t)g.F * g.Hp * nxs;
  const int64_t chunks = (strips + strips_per_item - 1) / strips_per_item;
  const int64_t items = chunks * rows * pairs;
  for (int64_t it = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; it < items;
       it += (int64_t)gridDim.x * blockDim.x) {
    const int c2 = (int)(it % pairs);
    const int r = (int)((it / pairs) % rows);
    const int64_t chunk = it / ((int64_t)pairs * rows);
    const int u = r / g.kh, v = r % g.kh;
    float dwr[KW][2];
#pragma unroll
    for (int j = 0; j < KW; j++) dwr[j][0] = dwr[j][1] = 0.f;
    float db[2] = {0.f, 0.f};
    const int64_t s_end = (chunk + 1) * strips_per_item < strips ? (chunk + 1) * strips_per_item : strips;
    for (int64_t s = chunk * strips_per_item; s < s_end; s++) {
      const int x0 = (int)(s % nxs) * kConvStrip;
      const int yy = (int)((s / nxs) % g.Hp);
      const int t = (int)(s / ((int64_t)nxs * g.Hp));
      dw_row<T, KW, TD>(x, dy, g, t, yy, x0, c2, u, v, dwr, r == 0 ? db : nullptr);
    }
    const int64_t K = (int64_t)rows * KW;
    float* d0 = dweight + (int64_t)(2 * c2) * K + (int64_t)r * KW;
#pragma unroll
    for (int j = 0; j < KW; j++) {
      atomicAdd(d0 + j, dwr[j][0]);
      atomicAdd(d0 + K + j, dwr[j][1]);
    }
    if (r == 0) {
      atomicAdd(dbias + 2 * c2, db[0]);
      atomicAdd(dbias + 2 * c2 + 1, db[1]);
    }
  }
}
#endif  // __CUDACC__

}  // namespace dsa3d
