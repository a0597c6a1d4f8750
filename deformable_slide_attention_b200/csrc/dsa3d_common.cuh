// dsa3d_common.cuh -- device helpers shared by the 3D-DSA kernels (sm_100a).
//
// Geometry of one query (MegaSlide-DiT, arXiv 2607.22696, 3D-DSA definition, Eq. 1): the taps of
// a query at p with integer offset part i and fractional part f sample positions
// p + tau + i + f, tau in the centred window.  All taps share f, so their trilinear corners all
// fall on one integer "box" of (k_t+1) x (k_h+1) x (k_w+1) tokens whose origin is p + i - r.
// The kernels therefore dot q with each box token once and combine the results per tap with the
// 8 trilinear weights, instead of sampling every tap separately.
#pragma once

#include <cuda_bf16.h>
#include <stdint.h>

// Minimum resident CTAs per SM requested from the compiler for the tensor-core kernels
// (trades registers for occupancy).
#ifndef DSA3D_MMA_MINB
#define DSA3D_MMA_MINB 3
#endif
#ifndef DSA3D_BWDQ_MINB
#define DSA3D_BWDQ_MINB 6  // the query side's CTAs are one warp pair (64 threads)
#endif
#ifndef DSA3D_DQ_MINB
#define DSA3D_DQ_MINB 3
#endif
#ifndef DSA3D_KV_MINB
#define DSA3D_KV_MINB 2
#endif

namespace dsa3d {

constexpr unsigned kFull = 0xffffffffu;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

// Launch-wide geometry.
struct Geo {
  int F, Hp, Wp, heads;
  int kt, kh, kw;  // window
  int Bt, Bh, Bw;  // box = window + 1 on each axis
  int B, K;        // box tokens, taps
  int HW;          // Hp * Wp
  int64_t N;       // tokens
  float scale;     // 1/sqrt(dh)
};

// One decoded query.
struct Query {
  bool ok;     // false: no valid tap, or an invalid offset
  int o[3];    // box origin p + i - r (may lie outside the volume)
  float f[3];  // fractional offset parts in [0, 1)
  int lo[3];   // valid taps: tap coordinate in [lo, hi] on each axis (coordinates 0..k-1)
  int hi[3];
  int nhi[3];  // box coordinates the query reads: [lo, nhi] on each axis (see decode_query)
};

__device__ __forceinline__ int dim_of(const Geo& g, int a) { return a == 0 ? g.F : (a == 1 ? g.Hp : g.Wp); }
__device__ __forceinline__ int win_of(const Geo& g, int a) { return a == 0 ? g.kt : (a == 1 ? g.kh : g.kw); }

// One offset component: i = floor(delta), f = delta - i in fp32 round-to-nearest, f == 1 carries
// into i.  Returns false (i = 0, f = 0) for a non-finite delta or |delta| > 2^24.
__device__ __forceinline__ bool decode_delta(float d, int& ii, float& fr) {
  ii = 0;
  fr = 0.f;
  if (!(fabsf(d) <= 16777216.f)) return false;  // also false for NaN
  const float fl = floorf(d);
  fr = __fsub_rn(d, fl);
  ii = (int)fl;
  if (fr == 1.0f) {
    ii += 1;
    fr = 0.f;
  }
  return true;
}

// Offset decode of a per-token offset (decode_delta on each axis; an invalid component makes
// the query invalid), then the per-axis tap and corner ranges.
// The forward reads only corners with a nonzero weight (the +1 plane only when f != 0).  With
// for_grad the +1 plane is read whenever it lies in the volume: at f == 0 its weight is zero but
// the derivative of the weight along that axis is not.
__device__ __forceinline__ Query decode_query(const Geo& g, const float* __restrict__ off, int h,
                                              int64_t n, bool for_grad = false) {
  Query Q;
  Q.ok = true;
  const float* o = off + ((int64_t)h * g.N + n) * 3;
  const int x = (int)(n % g.Wp);
  const int y = (int)((n / g.Wp) % g.Hp);
  const int t = (int)(n / g.HW);
  const int p[3] = {t, y, x};
#pragma unroll
  for (int a = 0; a < 3; a++) {
    int ii;
    float fr;
    if (!decode_delta(__ldg(o + a), ii, fr)) Q.ok = false;
    const int k = win_of(g, a), D = dim_of(g, a);
    const int org = p[a] + ii - (k - 1) / 2;
    const int up = (fr != 0.f) ? 1 : 0;
    Q.o[a] = org;
    Q.f[a] = fr;
    Q.lo[a] = max(0, -org);
    Q.hi[a] = min(k - 1, D - 1 - org - up);
    Q.nhi[a] = for_grad ? min(Q.hi[a] + 1, D - 1 - org) : Q.hi[a] + up;
    if (Q.lo[a] > Q.hi[a]) Q.ok = false;
  }
  return Q;
}

// 8 trilinear weights, corner c = (ct << 2) | (cy << 1) | cx.
__device__ __forceinline__ void corner_weights(const float f[3], float w[8]) {
#pragma unroll
  for (int c = 0; c < 8; c++) {
    const float wt = (c & 4) ? f[0] : 1.f - f[0];
    const float wy = (c & 2) ? f[1] : 1.f - f[1];
    const float wx = (c & 1) ? f[2] : 1.f - f[2];
    w[c] = wt * wy * wx;
  }
}

// d w_c / d f_a for the three axes.
__device__ __forceinline__ void corner_dweights(const float f[3], float dw[3][8]) {
#pragma unroll
  for (int c = 0; c < 8; c++) {
    const float wt = (c & 4) ? f[0] : 1.f - f[0];
    const float wy = (c & 2) ? f[1] : 1.f - f[1];
    const float wx = (c & 1) ? f[2] : 1.f - f[2];
    const float st = (c & 4) ? 1.f : -1.f, sy = (c & 2) ? 1.f : -1.f, sx = (c & 1) ? 1.f : -1.f;
    dw[0][c] = st * wy * wx;
    dw[1][c] = wt * sy * wx;
    dw[2][c] = wt * wy * sx;
  }
}

// --- 16-byte row chunks -------------------------------------------------------------------------
template <typename T>
struct Elems;
template <>
struct Elems<float> {
  static constexpr int kPerLoad = 4;
};
template <>
struct Elems<__nv_bfloat16> {
  static constexpr int kPerLoad = 8;
};

__device__ __forceinline__ void load16(const float* p, float* x) {
  const float4 v = __ldg(reinterpret_cast<const float4*>(p));
  x[0] = v.x; x[1] = v.y; x[2] = v.z; x[3] = v.w;
}
__device__ __forceinline__ void load16(const __nv_bfloat16* p, float* x) {
  const uint4 v = __ldg(reinterpret_cast<const uint4*>(p));
  const unsigned w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; i++) {
    x[2 * i] = __uint_as_float(w[i] << 16);
    x[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
  }
}
__device__ __forceinline__ void store16(float* p, const float* x) {
  *reinterpret_cast<float4*>(p) = make_float4(x[0], x[1], x[2], x[3]);
}
__device__ __forceinline__ void store16(__nv_bfloat16* p, const float* x) {
  uint4 v;
  unsigned* w = reinterpret_cast<unsigned*>(&v);
#pragma unroll
  for (int i = 0; i < 4; i++) {
    const __nv_bfloat162 b = __floats2bfloat162_rn(x[2 * i], x[2 * i + 1]);
    w[i] = *reinterpret_cast<const unsigned*>(&b);
  }
  *reinterpret_cast<uint4*>(p) = v;
}

// Reduce L partial sums across the L lanes of an aligned lane group (L a power of two <= 32):
// on entry v[i] is this lane's partial for item i; on exit v[0] holds the full sum for item
// (lane % L).  L-1 shuffles per L items instead of log2(L) per item.
template <int L>
__device__ __forceinline__ float group_transpose_sum(float (&v)[L], int lane) {
#pragma unroll
  for (int w = L / 2; w >= 1; w >>= 1) {
    const bool up = (lane & w) != 0;
#pragma unroll
    for (int i = 0; i < w; i++) {
      const float send = up ? v[i] : v[i + w];
      const float keep = up ? v[i + w] : v[i];
      v[i] = keep + __shfl_xor_sync(kFull, send, w);
    }
  }
  return v[0];
}

__device__ __forceinline__ float warp_max(float x) {
#pragma unroll
  for (int w = 16; w >= 1; w >>= 1) x = fmaxf(x, __shfl_xor_sync(kFull, x, w));
  return x;
}
__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int w = 16; w >= 1; w >>= 1) x += __shfl_xor_sync(kFull, x, w);
  return x;
}

// Box/tap coordinate packing for the per-CTA tables (each coordinate < 1024).
__device__ __forceinline__ int pack3(int a, int b, int c) { return (a << 20) | (b << 10) | c; }
__device__ __forceinline__ void unpack3(int r, int& a, int& b, int& c) {
  a = r >> 20;
  b = (r >> 10) & 1023;
  c = r & 1023;
}

// Device-side check record (set by kernels built with DSA3D_DEBUG, read by dsa3d_check_device).
// Of the library's two translation units only dsa3d.cu includes this header (the convolution's
// dsa3d_conv.cu does not), so this is its only definition.
__device__ int g_dsa3d_check;

#ifdef DSA3D_DEBUG
#define DSA3D_DEVICE_CHECK(cond) \
  do {                           \
    if (!(cond)) atomicExch(&::dsa3d::g_dsa3d_check, 1); \
  } while (0)
#else
#define DSA3D_DEVICE_CHECK(cond) \
  do {                           \
  } while (0)
#endif

}  // namespace dsa3d
