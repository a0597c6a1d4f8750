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
// bf16 traffic: about 120 flop per byte, so it is bound by the fp32 FMA pipes, not by HBM.  Every
// kernel gives a thread one channel pair (consecutive lanes on consecutive pairs, so a warp's
// loads of one token are one coalesced 128- or 256-byte run) and blocks registers along x (strips
// of kConvStrip outputs) and y; the pair's two channels share one packed fp32x2 FMA (conv_fma2).
//
//   forward and dX, at most kConvSwMaxTaps taps:
//     dsa3d_dwconv3d_sw2_kernel (C a multiple of 32): units of two neighbouring strips on
//       kSw2Rows rows; the block's weights staged tap-major in shared memory, the input rows
//       copied by the warp into a ring in shared memory (16-byte cp.async chunks, two rows ahead);
//     dsa3d_dwconv3d_sw_kernel (other C): one strip on two rows per thread, the weights staged,
//       the rows loaded one row ahead into registers;
//   forward and dX, larger kernels: dsa3d_dwconv3d_kernel, the weights read from global memory;
//   dW and db: dsa3d_dwconv3d_dw_kernel, a thread on three kernel rows of a plane walking a strip
//     column down the input rows, the rows and dY strips through a per-warp cp.async ring.
//
// The per-thread arithmetic (conv_strip2, conv_strips_ring, dw_walk and their copy routines) is
// __host__ __device__ code so that a host harness can run exactly these routines on the CPU.
#pragma once

#include <cuda_bf16.h>
#include <stdint.h>

// Threads per block of the global-memory forward kernel and of the dW kernel (the staged forward
// has its own, kConvSwWarps warps).  Both hold many accumulators per thread (about 165 and 235
// registers): 128-thread blocks let the SM hold three and two of them.  At 1080p (256 x 68 x 120
// tokens, 4096 channels, 3 x 9 x 9) the global-memory forward took 326 ms at 128 threads and 412
// ms at 256.
#ifndef DSA3D_CONV_FWD_THREADS
#define DSA3D_CONV_FWD_THREADS 128
#endif
#ifndef DSA3D_CONV_DW_THREADS
#define DSA3D_CONV_DW_THREADS 128
#endif

namespace dsa3d {

constexpr int kConvStrip = 8;  // outputs along x per thread
constexpr int kConvFwdThreads = DSA3D_CONV_FWD_THREADS;
constexpr int kConvDwThreads = DSA3D_CONV_DW_THREADS;
static_assert(kConvFwdThreads % 32 == 0 && kConvFwdThreads >= 32 && kConvFwdThreads <= 1024 &&
                  kConvDwThreads % 32 == 0 && kConvDwThreads >= 32 && kConvDwThreads <= 1024,
              "convolution blocks: whole warps, at most 1024 threads");

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
template <typename T>
__host__ __device__ __forceinline__ float2 conv_load2v(const T* p) {
  float2 v;
  conv_load2(p, v.x, v.y);
  return v;
}

// acc += w * x on both channels of a pair: on the GPU one fma.rn.f32x2 (one issue slot for the
// two FMAs), each lane rounded as fmaf rounds it.
__host__ __device__ __forceinline__ void conv_fma2(float2& acc, const float2 w, const float2 x) {
#ifdef __CUDA_ARCH__
  acc = __ffma2_rn(w, x, acc);
#else
  acc.x = fmaf(w.x, x.x, acc.x);
  acc.y = fmaf(w.y, x.y, acc.y);
#endif
}

// Where conv_strip2 reads the kernel: tap k (flattened (u, v, w)) of channel pair c2's two
// channels.  ConvWGlobal reads W [C][kt][kh][kw] where it lies; its channels are K floats apart,
// so a warp's 32 pairs touch 32 cache lines per tap.  ConvWShared reads a block's staged copy of
// its channel group, tap-major (conv_sw_index), where a warp's pairs read one 256-byte row.
struct ConvWGlobal {
  const float* w0;  // W[2 c2][0][0][0]
  int64_t K;        // taps per channel
  __host__ __device__ __forceinline__ float2 operator()(int64_t k) const {
    return make_float2(conv_ldw(w0 + k), conv_ldw(w0 + K + k));
  }
};

constexpr int kConvGroupPairs = 32;                        // channel pairs per staged group: one per lane
constexpr int kConvGroupStride = 2 * kConvGroupPairs + 2;  // floats per staged tap row (2 of padding)
constexpr int kConvSwWarps = 4;                            // warps per block of the staged kernel
constexpr int kConvSwUnits = 32;                           // (t, row pair, strip) units per block
// Most taps staged: 387 x 66 x 4 B = 102 KB, two blocks per SM (3 x 9 x 9 = 243 taps take 64 KB:
// three).  A larger kernel runs from global memory.
constexpr int kConvSwMaxTaps = 387;
static_assert(kConvSwUnits % kConvSwWarps == 0, "whole steps of the staged kernel's warps");

// Channel cc (of the group's 2 kConvGroupPairs) at tap k in the staged copy.
__host__ __device__ __forceinline__ int conv_sw_index(int k, int cc) { return k * kConvGroupStride + cc; }
__host__ __device__ __forceinline__ size_t conv_sw_bytes(int K) {
  return (size_t)K * kConvGroupStride * sizeof(float);
}
struct ConvWShared {
  const float* s;  // the staged group + 2 * lane (8-byte aligned: the stride is even)
  __host__ __device__ __forceinline__ float2 operator()(int64_t k) const {
    return *reinterpret_cast<const float2*>(s + (int)k * kConvGroupStride);
  }
};

// Unit (t, y0, x0) of the forward's work: output rows y0, y0 + 1 from column x0, strips fastest,
// then row pairs, then frames.
__host__ __device__ __forceinline__ void conv_unit(int64_t unit, int nxs, int nyp, int& t, int& y0,
                                                   int& x0) {
  x0 = (int)(unit % nxs) * kConvStrip;
  const int64_t r = unit / nxs;
  y0 = 2 * (int)(r % nyp);
  t = (int)(r / nyp);
}

// The i-th unit (i < units per block / kConvSwWarps) of warp `warp` in a staged kernel's block
// slot `slot` of `slots` (= ceil(units / units per block)).  The slots' units interleave: at step i
// the resident blocks, whose slots are consecutive, work on one run of consecutive units (the
// rows they read stay in L2), and every unit below slots * kConvSwUnits is visited once.
__host__ __device__ __forceinline__ int64_t conv_sw_unit(int64_t slot, int64_t slots, int warp, int i) {
  return ((int64_t)i * slots + slot) * kConvSwWarps + warp;
}

// The raw channel pair of T as loaded (4 bytes for bf16, 8 for fp32), and its fp32 values.
template <typename T>
struct ConvRaw;
template <>
struct ConvRaw<float> {
  using type = float2;
};
template <>
struct ConvRaw<__nv_bfloat16> {
  using type = unsigned;
};
__host__ __device__ __forceinline__ float2 conv_unpack(float2 r) { return r; }
__host__ __device__ __forceinline__ float2 conv_unpack(unsigned u) {
  union {
    unsigned i;
    float f;
  } lo, hi;
  lo.i = u << 16;
  hi.i = u & 0xffff0000u;
  return make_float2(lo.f, hi.f);
}

// Convolution sums of channel pair c2 (channels 2 c2 and 2 c2 + 1) for the two output strips
// (t, y0 + r, x0 + i), r < 2, i < kConvStrip, added into acc[r][i] (.x: channel 2 c2, .y: 2 c2 +
// 1).  For kernel plane u the input rows y0 - r_h .. y0 + 1 + r_h are loaded once each, and
// kernel row v's weights once for both outputs: output row y0 takes input row y0 + v - r_h,
// output row y0 + 1 the next one, so the row loaded for one v is carried to the next.  flip: use
// W[c][kt-1-u][kh-1-v][kw-1-w] (the backward's dX).  An output row past the volume (y0 + 1 =
// Hp) is computed and not stored.  KW = the kernel's width kw (a compile-time constant); wget:
// where the weights are read (ConvWGlobal, ConvWShared).
template <typename T, int KW>
__host__ __device__ __forceinline__ void conv_load_row(const T* __restrict__ row, const ConvGeo& g, int x0,
                                                       float2 (&a)[kConvStrip + KW - 1]) {
  const int rw = (KW - 1) / 2;
#pragma unroll
  for (int j = 0; j < kConvStrip + KW - 1; j++) {
    const int xs = x0 - rw + j;
    a[j] = make_float2(0.f, 0.f);
    if (xs >= 0 && xs < g.Wp) a[j] = conv_load2v(row + (int64_t)xs * g.C);
  }
}

// The same row as raw pairs (zero past the volume's edges, and all zero when !in).
template <typename T, int KW>
__host__ __device__ __forceinline__ void conv_load_row_raw(const T* __restrict__ row, bool in, const ConvGeo& g,
                                                           int x0,
                                                           typename ConvRaw<T>::type (&r)[kConvStrip + KW - 1]) {
  using R = typename ConvRaw<T>::type;
  const int rw = (KW - 1) / 2;
#pragma unroll
  for (int j = 0; j < kConvStrip + KW - 1; j++) {
    const int xs = x0 - rw + j;
    r[j] = R{};
    if (in && xs >= 0 && xs < g.Wp) {
#ifdef __CUDA_ARCH__
      r[j] = __ldg(reinterpret_cast<const R*>(row + (int64_t)xs * g.C));
#else
      r[j] = *reinterpret_cast<const R*>(row + (int64_t)xs * g.C);
#endif
    }
  }
}

template <typename T, int KW, typename WGet>
__host__ __device__ __forceinline__ void conv_strip2(const T* __restrict__ x, const WGet& wget,
                                                     const ConvGeo& g, int t, int y0, int x0, int c2,
                                                     bool flip, float2 (&acc)[2][kConvStrip]) {
  constexpr int NJ = kConvStrip + KW - 1;
  using R = typename ConvRaw<T>::type;
  const int rt = (g.kt - 1) / 2, rh = (g.kh - 1) / 2;
  const int64_t rstride = (int64_t)g.Wp * g.C;  // one token row
  // The input rows in order: plane u = 0 .. kt - 1, rows y0 - r_h + r, r = 0 .. kh; each row is
  // loaded (raw) one row ahead of its use.  Row r = 0 of a plane is kernel row 0's input for
  // output row y0; row r >= 1 is kernel row r - 1's input for output row y0 + 1 and kernel row r's
  // for y0 (carried in pr).  Rows outside the volume are zeros (plane u outside it: all its rows).
  const T* xc = x + 2 * c2;
  auto row_at = [&](int u, int r, bool& in) {
    const int ts = t + u - rt, ys = y0 - rh + r;
    in = ts >= 0 && ts < g.F && ys >= 0 && ys < g.Hp;
    return xc + ((int64_t)(in ? ts : 0) * g.Hp + (in ? ys : 0)) * rstride;
  };
  R nxt[NJ];
  {
    bool in;
    const T* row = row_at(0, 0, in);
    conv_load_row_raw<T, KW>(row, in, g, x0, nxt);
  }
  float2 pr[NJ];
  for (int u = 0; u < g.kt; u++) {
    for (int r = 0; r <= g.kh; r++) {
      float2 cr[NJ];
#pragma unroll
      for (int j = 0; j < NJ; j++) cr[j] = conv_unpack(nxt[j]);
      // the next row: r + 1 of this plane, or row 0 of the next plane
      if (r < g.kh || u + 1 < g.kt) {
        bool in;
        const T* row = r < g.kh ? row_at(u, r + 1, in) : row_at(u + 1, 0, in);
        conv_load_row_raw<T, KW>(row, in, g, x0, nxt);
      }
      if (r > 0) {
        const int v = r - 1;
        // the kernel row's weights (flipped for the transposed convolution)
        const int64_t wrow = flip ? ((int64_t)(g.kt - 1 - u) * g.kh + (g.kh - 1 - v)) * KW
                                  : ((int64_t)u * g.kh + v) * KW;
        float2 w[KW];
#pragma unroll
        for (int j = 0; j < KW; j++) w[j] = wget(wrow + (flip ? KW - 1 - j : j));
        // input column x0 - rw + j feeds output x0 + i through tap j - i
#pragma unroll
        for (int j = 0; j < NJ; j++) {
#pragma unroll
          for (int i = 0; i < kConvStrip; i++) {
            if (j - i >= 0 && j - i < KW) {
              conv_fma2(acc[0][i], w[j - i], pr[j]);
              conv_fma2(acc[1][i], w[j - i], cr[j]);
            }
          }
        }
      }
#pragma unroll
      for (int j = 0; j < NJ; j++) pr[j] = cr[j];
    }
  }
}

// dW and db.  A work item is channel pair c2, kernel plane u, kDwRows kernel rows v0 .. v0 +
// kDwRows - 1 (those below kh), the strip column from x0 and a run of dY frames.  For each frame
// it walks the input rows ys of frame t + u - r_t downward: input row ys meets dY row
// ys - v + r_h for each kernel row v, so a step loads one input row (kConvStrip + KW - 1 values)
// and one new dY strip (kConvStrip values), carries the other kDwRows - 1 dY strips (moved one
// register slot per step), and does kDwRows kConvStrip KW FMAs per channel.
constexpr int kDwRows = 3;

// Work item `it` of the dW kernel: channel pairs fastest, then kernel-row groups, planes, strip
// columns and runs of frames_per_item dY frames [t0, t1).
__host__ __device__ __forceinline__ void dw_decode(int64_t it, const ConvGeo& g, int frames_per_item, int& c2,
                                                   int& u, int& v0, int& x0, int& t0, int& t1) {
  const int pairs = g.C / 2, groups = (g.kh + kDwRows - 1) / kDwRows;
  const int nxs = (g.Wp + kConvStrip - 1) / kConvStrip;
  c2 = (int)(it % pairs);
  int64_t r = it / pairs;
  v0 = (int)(r % groups) * kDwRows;
  r /= groups;
  u = (int)(r % g.kt);
  r /= g.kt;
  x0 = (int)(r % nxs) * kConvStrip;
  t0 = (int)(r / nxs) * frames_per_item;
  t1 = t0 + frames_per_item < g.F ? t0 + frames_per_item : g.F;
}

__host__ __device__ __forceinline__ int64_t dw_items(const ConvGeo& g, int frames_per_item) {
  const int groups = (g.kh + kDwRows - 1) / kDwRows;
  const int nxs = (g.Wp + kConvStrip - 1) / kConvStrip;
  return (int64_t)(g.C / 2) * groups * g.kt * nxs * ((g.F + frames_per_item - 1) / frames_per_item);
}

// dY strip (row y of the frame at dplane, columns x0 .. x0 + kConvStrip - 1) of the pair as fp32;
// zeros for a row outside the frame or columns past its last.
template <typename TD>
__host__ __device__ __forceinline__ void dw_load_dy(const TD* __restrict__ dplane, const ConvGeo& g, int y,
                                                    int x0, float2 (&d)[kConvStrip]) {
  const bool in = y >= 0 && y < g.Hp;
  const TD* row = dplane + ((int64_t)y * g.Wp + x0) * g.C;
#pragma unroll
  for (int i = 0; i < kConvStrip; i++) {
    d[i] = make_float2(0.f, 0.f);
    if (in && x0 + i < g.Wp) d[i] = conv_load2v(row + (int64_t)i * g.C);
  }
}

// *dst = *src (a raw pair), or zeros when !ok.  On the GPU an asynchronous copy into shared
// memory (cp.async; with !ok it copies no bytes, zero-fills, and src is only a valid address),
// complete once dw_wait has covered its group.
template <typename R>
__host__ __device__ __forceinline__ void dw_copy(R* dst, const R* src, bool ok) {
#ifdef __CUDA_ARCH__
  const unsigned d = (unsigned)__cvta_generic_to_shared(dst);
  const int n = ok ? (int)sizeof(R) : 0;
  if constexpr (sizeof(R) == 8)
    asm volatile("cp.async.ca.shared.global [%0], [%1], 8, %2;\n" ::"r"(d), "l"(src), "r"(n) : "memory");
  else
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;\n" ::"r"(d), "l"(src), "r"(n) : "memory");
#else
  *dst = ok ? *src : R{};
#endif
}
__host__ __device__ __forceinline__ void dw_commit() {
#ifdef __CUDA_ARCH__
  asm volatile("cp.async.commit_group;\n" ::: "memory");
#endif
}
// Wait until at most N of this thread's committed copy groups are still in flight.
template <int N>
__host__ __device__ __forceinline__ void dw_wait() {
#ifdef __CUDA_ARCH__
  asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory");
#endif
}

// 16 bytes from src to dst, or zeros when !ok: on the GPU cp.async (through L2 only), otherwise
// as dw_copy.
__host__ __device__ __forceinline__ void dw_copy16(void* dst, const void* src, bool ok) {
#ifdef __CUDA_ARCH__
  const unsigned d = (unsigned)__cvta_generic_to_shared(dst);
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(d), "l"(src), "r"(ok ? 16 : 0) : "memory");
#else
  unsigned char* o = static_cast<unsigned char*>(dst);
  const unsigned char* i = static_cast<const unsigned char*>(src);
  for (int b = 0; b < 16; b++) o[b] = ok ? i[b] : 0;
#endif
}
__host__ __device__ __forceinline__ void dw_syncwarp() {
#ifdef __CUDA_ARCH__
  __syncwarp();
#endif
}

constexpr int kDwStages = 3;  // steps of the dW walk in its staging ring: fetched two steps ahead

// One lane's staging ring of the dW walk: kDwStages steps of an input row (NJ raw pairs) and a
// dY strip (kConvStrip raw pairs).  A warp's lanes are interleaved (entry e of a lane at
// [e * 32]), so the warp's copies and reads of one entry are one contiguous row of shared memory,
// and each lane reads back only what it copied itself.
template <typename T, typename TD, int KW>
struct DwRing {
  static constexpr int NJ = kConvStrip + KW - 1;
  using XR = typename ConvRaw<T>::type;
  using DR = typename ConvRaw<TD>::type;
  XR* x;  // the lane's entry (stage 0, column 0): [stage][NJ], stride 32
  DR* d;  // the lane's entry (stage 0, strip output 0): [stage][kConvStrip], stride 32
  __host__ __device__ static constexpr size_t x_bytes() { return (size_t)kDwStages * NJ * 32 * sizeof(XR); }
  __host__ __device__ static constexpr size_t warp_bytes() {
    return x_bytes() + (size_t)kDwStages * kConvStrip * 32 * sizeof(DR);
  }
  // the ring of lane `lane` in the warp's region at base (8-byte aligned)
  __host__ __device__ static DwRing at(unsigned char* base, int lane) {
    DwRing r;
    r.x = reinterpret_cast<XR*>(base) + lane;
    r.d = reinterpret_cast<DR*>(base + x_bytes()) + lane;
    return r;
  }
};

// Fetch step ys of the walk into ring stage st: input row ys (columns x0 - r_w .. x0 + kConvStrip
// + r_w - 1) of the frame at xplane and dY row ys - v0 + r_h (columns x0 .. x0 + kConvStrip - 1)
// of the frame at dplane; zeros outside the frames.
template <typename T, typename TD, int KW>
__host__ __device__ __forceinline__ void dw_fetch(const DwRing<T, TD, KW>& r, int st, const T* xplane,
                                                  const TD* dplane, const ConvGeo& g, int ys, int v0, int x0) {
  using R = DwRing<T, TD, KW>;
  using XR = typename R::XR;
  using DR = typename R::DR;
  const int rw = (KW - 1) / 2, rh = (g.kh - 1) / 2;
  const T* xrow = xplane + (int64_t)ys * g.Wp * g.C;
#pragma unroll
  for (int j = 0; j < R::NJ; j++) {
    const int xs = x0 - rw + j;
    const bool ok = xs >= 0 && xs < g.Wp;
    dw_copy(r.x + (st * R::NJ + j) * 32, reinterpret_cast<const XR*>(ok ? xrow + (int64_t)xs * g.C : xplane), ok);
  }
  const int y = ys - v0 + rh;
  const bool yin = y >= 0 && y < g.Hp;
  const TD* drow = yin ? dplane + ((int64_t)y * g.Wp + x0) * g.C : dplane;
#pragma unroll
  for (int k = 0; k < kConvStrip; k++) {
    const bool ok = yin && x0 + k < g.Wp;
    dw_copy(r.d + (st * kConvStrip + k) * 32, reinterpret_cast<const DR*>(ok ? drow + (int64_t)k * g.C : dplane), ok);
  }
}

// The 16-byte chunks of one staged run of `tokens` tokens (32 pairs of R each: CPT = 2 sizeof(R)
// chunks per token) that lane `lane` copies: chunk m = lane + 32 i is token m / CPT, chunk m mod
// CPT, so the lane's token advances by 32 / CPT per chunk and its offset in the token is fixed.
// src0: pair 0 of token 0 of the run (tokens C elements apart), ok(j): token j inside the volume;
// dst0: the run's ring entries (token j at dst0 + j 32 sizeof(R) bytes).
template <typename R, int TOKENS, typename TS, typename OK>
__host__ __device__ __forceinline__ void dw_copy_run(unsigned char* dst0, const TS* src0, const TS* fallback,
                                                     int64_t C, int lane, OK ok) {
  constexpr int CPT = 32 * (int)sizeof(R) / 16;
  constexpr int TSTEP = 32 / CPT;  // tokens between a lane's chunks
  const int j0 = lane / CPT, q = lane % CPT;
  const unsigned char* src = reinterpret_cast<const unsigned char*>(src0 + j0 * C) + 16 * q;
  unsigned char* dst = dst0 + (size_t)j0 * 32 * sizeof(R) + 16 * q;
  const int64_t sstep = TSTEP * C * (int64_t)sizeof(TS);
#pragma unroll
  for (int i = 0; i < (TOKENS + TSTEP - 1) / TSTEP; i++) {
    const int j = j0 + i * TSTEP;
    if (j < TOKENS) {
      const bool in = ok(j);
      const unsigned char* from = in ? src + i * sstep : reinterpret_cast<const unsigned char*>(fallback);
      dw_copy16(dst + (size_t)i * TSTEP * 32 * sizeof(R), from, in);
    }
  }
}

// dw_fetch for the whole warp at once, when its 32 lanes are 32 consecutive channel pairs from a
// multiple of 32 (C a multiple of 64) on the same work item: a token's 32 pairs are one
// contiguous run of 128 (bf16) or 256 (fp32) bytes, copied as 16-byte chunks spread over the
// lanes (dw_copy_run), each chunk into the 16 bytes of the ring entry that hold those pairs.
// xplane and dplane point at the lane's own pair; the chunks a lane copies belong to other lanes
// too, so the ring is shared within the warp (dw_syncwarp around its use).  On the host one call
// copies every lane's chunks.
template <typename T, typename TD, int KW>
__host__ __device__ __forceinline__ void dw_fetch_warp(const DwRing<T, TD, KW>& r, int lane, int st,
                                                       const T* xplane, const TD* dplane, const ConvGeo& g,
                                                       int ys, int v0, int x0) {
  using R = DwRing<T, TD, KW>;
  using XR = typename R::XR;
  using DR = typename R::DR;
  const int rw = (KW - 1) / 2, rh = (g.kh - 1) / 2;
  const T* xw = xplane - 2 * lane;  // pair 0 of the warp
  const TD* dw = dplane - 2 * lane;
  unsigned char* rx = reinterpret_cast<unsigned char*>(r.x - lane) + (size_t)st * R::NJ * 32 * sizeof(XR);
  unsigned char* rd = reinterpret_cast<unsigned char*>(r.d - lane) + (size_t)st * kConvStrip * 32 * sizeof(DR);
  const int xs0 = x0 - rw;
  const T* xsrc = xw + ((int64_t)ys * g.Wp + xs0) * g.C;  // token xs0 of row ys (not read unless inside)
  const int y = ys - v0 + rh;
  const bool yin = y >= 0 && y < g.Hp;
  const TD* dsrc = dw + ((int64_t)(yin ? y : 0) * g.Wp + x0) * g.C;
  auto xok = [&](int j) { return xs0 + j >= 0 && xs0 + j < g.Wp; };
  auto dok = [&](int k) { return yin && x0 + k < g.Wp; };
#ifdef __CUDA_ARCH__
  dw_copy_run<XR, R::NJ>(rx, xsrc, xw, g.C, lane, xok);
  dw_copy_run<DR, kConvStrip>(rd, dsrc, dw, g.C, lane, dok);
#else
  for (int l = 0; l < 32; l++) {
    dw_copy_run<XR, R::NJ>(rx, xsrc, xw, g.C, l, xok);
    dw_copy_run<DR, kConvStrip>(rd, dsrc, dw, g.C, l, dok);
  }
#endif
}

// Step of the walk whose data sit in ring stage st: the carried dY strips move one slot down
// (slot i holds the dY row that kernel row v0 + i meets, ys - v0 - i + r_h), slot 0 takes the new
// row ys - v0 + r_h, and the input row ys is multiplied into every kernel row's sums.
template <typename T, int KW, typename TD>
__host__ __device__ __forceinline__ void dw_step(const DwRing<T, TD, KW>& r, int st, const ConvGeo& g, int v0,
                                                 float2 (&d)[kDwRows][kConvStrip],
                                                 float2 (&dwr)[kDwRows][KW]) {
  constexpr int NJ = kConvStrip + KW - 1;
#pragma unroll
  for (int i = kDwRows - 1; i > 0; i--)
#pragma unroll
    for (int k = 0; k < kConvStrip; k++) d[i][k] = d[i - 1][k];
#pragma unroll
  for (int k = 0; k < kConvStrip; k++) d[0][k] = conv_unpack(r.d[(st * kConvStrip + k) * 32]);
  float2 a[NJ];
#pragma unroll
  for (int j = 0; j < NJ; j++) a[j] = conv_unpack(r.x[(st * NJ + j) * 32]);
#pragma unroll
  for (int i = 0; i < kDwRows; i++) {
    if (v0 + i >= g.kh) break;
    // input column x0 - r_w + j meets output x0 + k through tap j - k
#pragma unroll
    for (int j = 0; j < NJ; j++) {
#pragma unroll
      for (int k = 0; k < kConvStrip; k++) {
        if (j - k >= 0 && j - k < KW) conv_fma2(dwr[i][j - k], d[i][k], a[j]);
      }
    }
  }
}

// One work item's sums: dwr[i][w] (.x, .y: channel 2 c2 + e, e = 0, 1) += sum over its frames t,
// rows y and columns x0 + k of dY[(t, y, x0 + k)][2 c2 + e] * X[(t + u - r_t, y + v0 + i - r_h,
// x0 + k + w - r_w)][2 c2 + e]; and, if with_db, db[e] += the sum of its dY strips over every row
// of its frames.  Outputs past the volume's last column are skipped; X and dY are zero outside the
// volume.  TD: the type of dY (the input's, or fp32 for the offset network's backward).  The
// input rows and new dY strips go through the lane's ring, fetched kDwStages - 1 steps ahead.
template <typename T, int KW, typename TD = T, bool Coop = false>
__host__ __device__ __forceinline__ void dw_walk(const T* __restrict__ x, const TD* __restrict__ dy,
                                                 const ConvGeo& g, const DwRing<T, TD, KW>& ring, int c2,
                                                 int u, int v0, int x0, int t0, int t1,
                                                 float2 (&dwr)[kDwRows][KW], bool with_db, float (&db)[2]) {
  constexpr int D = kDwStages - 1;
  const int rt = (g.kt - 1) / 2, rh = (g.kh - 1) / 2;
  const int64_t fstride = (int64_t)g.Hp * g.Wp * g.C;  // one frame
#pragma unroll 1
  for (int t = t0; t < t1; t++) {
    const TD* dplane = dy + t * fstride + 2 * c2;
    if (with_db) {
#pragma unroll 1
      for (int y = 0; y < g.Hp; y++) {
        float2 d[kConvStrip];
        dw_load_dy<TD>(dplane, g, y, x0, d);
#pragma unroll
        for (int k = 0; k < kConvStrip; k++) {
          db[0] += d[k].x;
          db[1] += d[k].y;
        }
      }
    }
    const int ts = t + u - rt;
    if (ts < 0 || ts >= g.F) continue;
    const T* xplane = x + ts * fstride + 2 * c2;
    // the input rows that meet some dY row through kernel rows v0 .. v0 + kDwRows - 1
    const int ys0 = v0 - rh > 0 ? v0 - rh : 0;
    const int ys1 = g.Hp - 1 + v0 + kDwRows - 1 - rh < g.Hp - 1 ? g.Hp - 1 + v0 + kDwRows - 1 - rh : g.Hp - 1;
    const int n = ys1 - ys0 + 1;
    // slot i - 1 holds, before the first step moves it to slot i, kernel row v0 + i's dY row
    float2 d[kDwRows][kConvStrip];
#pragma unroll
    for (int i = 1; i < kDwRows; i++) dw_load_dy<TD>(dplane, g, ys0 - v0 - i + rh, x0, d[i - 1]);
    // copy group s carries step s (empty past the last step): D groups ahead of the step in use
    auto fetch = [&](int st, int ys) {
      if constexpr (Coop)
        dw_fetch_warp(ring, c2 & 31, st, xplane, dplane, g, ys, v0, x0);
      else
        dw_fetch(ring, st, xplane, dplane, g, ys, v0, x0);
    };
    if (Coop) dw_syncwarp();  // the previous frame's last reads are done before the ring refills
#pragma unroll
    for (int s = 0; s < D; s++) {
      if (s < n) fetch(s, ys0 + s);
      dw_commit();
    }
#pragma unroll 1
    for (int s = 0; s < n; s++) {
      if (Coop) dw_syncwarp();  // every lane's reads of step s - 1's stage are done
      if (s + D < n) fetch((s + D) % kDwStages, ys0 + s + D);
      dw_commit();
      dw_wait<D>();  // this lane's groups 0 .. s are complete
      if (Coop) dw_syncwarp();  // and every lane's
      dw_step<T, KW, TD>(ring, s % kDwStages, g, v0, d, dwr);
    }
  }
}

// ---- the forward on strip pairs, input rows through a warp-shared ring ----------------------
// For C a multiple of 32: a block owns kSw2Pairs channel pairs and its warps take units of two
// neighbouring strips on kSw2Rows rows (t, rows y0 .. y0 + kSw2Rows - 1, columns xb .. xb + 2
// kConvStrip - 1); lane 16 h + p computes pair p of strip h.  The two strips' windows share one
// input row of NT tokens, which the warp copies into a ring in shared memory with 16-byte
// cp.async chunks, kSw2Stages - 1 rows ahead of its use.
constexpr int kSw2Pairs = 16;
constexpr int kSw2WStride = 2 * kSw2Pairs + 2;  // floats per staged tap row (2 of padding)
constexpr int kSw2Units = 32;                   // units per block, kSw2Units / kConvSwWarps per warp
constexpr int kSw2Stages = 3;
constexpr int kSw2Rows = 4;                     // output rows per unit

template <typename T, int KW>
struct Sw2Ring {
  using R = typename ConvRaw<T>::type;
  static constexpr int NT = 2 * kConvStrip + KW - 1;                 // tokens of a staged row
  static constexpr int ROW = (NT + (NT + 7) / 8) * kSw2Pairs;        // R entries per staged row
  // entry of token j, pair p: every 8 tokens shift by kSw2Pairs entries, so that the two strips'
  // lanes (tokens j and j + 8) read different banks
  __host__ __device__ static constexpr int at(int j, int p) { return (j + (j >> 3)) * kSw2Pairs + p; }
  __host__ __device__ static constexpr size_t warp_bytes() { return (size_t)kSw2Stages * ROW * sizeof(R); }
};

// Unit `unit` of the strip-pair forward: frames, then groups of kSw2Rows rows (nyr of them), then
// strip pairs (nxp) fastest.
__host__ __device__ __forceinline__ void conv_unit2(int64_t unit, int nxp, int nyr, int& t, int& y0, int& xb) {
  xb = (int)(unit % nxp) * 2 * kConvStrip;
  const int64_t r = unit / nxp;
  y0 = kSw2Rows * (int)(r % nyr);
  t = (int)(r / nyr);
}

template <typename T, int KW>
__host__ __device__ __forceinline__ void sw2_fetch_lane(typename ConvRaw<T>::type* ring, int lane, int st,
                                                        const T* xg, const ConvGeo& g, int ts, int ys, int xb) {
  using S = Sw2Ring<T, KW>;
  using R = typename S::R;
  constexpr int CPT = kSw2Pairs * (int)sizeof(R) / 16;  // 16-byte chunks per token
  constexpr int TSTEP = 32 / CPT;                       // tokens between a lane's chunks
  // the lane's first token j0 < TSTEP, so token j0 + i TSTEP's bank-shift group is (i TSTEP) / 8
  static_assert(TSTEP % 8 == 0 || 8 % TSTEP == 0, "chunk steps aligned with the 8-token bank shift");
  const int rw = (KW - 1) / 2;
  const bool rin = ts >= 0 && ts < g.F && ys >= 0 && ys < g.Hp;
  const int xs0 = xb - rw;
  const T* row = xg + (((int64_t)(rin ? ts : 0) * g.Hp + (rin ? ys : 0)) * g.Wp + xs0) * g.C;  // token xs0
  const int j0 = lane / CPT, q = lane % CPT;
  const unsigned char* src = reinterpret_cast<const unsigned char*>(row + (int64_t)j0 * g.C) + 16 * q;
  unsigned char* dst = reinterpret_cast<unsigned char*>(ring + st * S::ROW + j0 * kSw2Pairs) + 16 * q;
  const int64_t sstep = (int64_t)TSTEP * g.C * (int64_t)sizeof(T);
#pragma unroll
  for (int i = 0; i < (S::NT + TSTEP - 1) / TSTEP; i++) {
    const int j = j0 + i * TSTEP;
    if (j < S::NT) {
      const bool ok = rin && xs0 + j >= 0 && xs0 + j < g.Wp;
      const size_t doff = (size_t)(i * TSTEP + ((i * TSTEP) >> 3)) * kSw2Pairs * sizeof(R);  // S::at(j) - S::at(j0)
      dw_copy16(dst + doff, ok ? src + i * sstep : reinterpret_cast<const unsigned char*>(xg), ok);
    }
  }
}

// Copy input row ys of frame ts (tokens xb - r_w .. xb - r_w + NT - 1 of the group's pairs; xg:
// x at the group's first channel) into ring stage st, zeros outside the volume: chunk m = lane +
// 32 i of the row's 16-byte chunks (token m / CPT, chunk m mod CPT) is lane `lane`'s.  On the
// host one call copies every lane's chunks.
template <typename T, int KW>
__host__ __device__ __forceinline__ void sw2_fetch(typename ConvRaw<T>::type* ring, int lane, int st,
                                                   const T* xg, const ConvGeo& g, int ts, int ys, int xb) {
#ifdef __CUDA_ARCH__
  sw2_fetch_lane<T, KW>(ring, lane, st, xg, g, ts, ys, xb);
#else
  for (int l = 0; l < 32; l++) sw2_fetch_lane<T, KW>(ring, l, st, xg, g, ts, ys, xb);
  (void)lane;
#endif
}

// The convolution sums of lane 16 h + p of a strip-pair unit (strip x0 = xb + h kConvStrip, pair
// p of the group) for output rows y0 + o, o < kSw2Rows, added into acc[o]; Flip as in
// conv_strip2, the weights read from the staged group at wsp (its tap rows kSw2WStride floats
// apart, the lane's pair at 2 p).  The input rows y0 - r_h + r, r < kh + kSw2Rows - 1, of each
// kernel plane run as one sequence, read from the warp's ring (ring: the warp's kSw2Stages
// rows); input row r feeds output row y0 + o through kernel row r - o, whose weights are read
// for it.
template <typename T, int KW, bool Flip>
__host__ __device__ __forceinline__ void conv_strips_ring(typename ConvRaw<T>::type* ring, int lane,
                                                          const T* xg, const float* wsp, const ConvGeo& g,
                                                          int t, int y0, int xb,
                                                          float2 (&acc)[kSw2Rows][kConvStrip]) {
  using S = Sw2Ring<T, KW>;
  using R = typename S::R;
  constexpr int NJ = kConvStrip + KW - 1;
  constexpr int D = kSw2Stages - 1;
  const int h = lane >> 4, p = lane & (kSw2Pairs - 1);
  const int rt = (g.kt - 1) / 2, rh = (g.kh - 1) / 2;
  const int rows = g.kh + kSw2Rows - 1, Q = g.kt * rows;
  int fu = 0, fr = 0;  // plane and row of the next fetch
  auto fetch_next = [&](int q) {
    sw2_fetch<T, KW>(ring, lane, q % kSw2Stages, xg, g, t + fu - rt, y0 - rh + fr, xb);
    if (++fr == rows) {
      fr = 0;
      fu++;
    }
  };
  dw_syncwarp();  // the previous unit's last reads of the ring are done
#pragma unroll
  for (int q = 0; q < D; q++) {
    if (q < Q) fetch_next(q);
    dw_commit();
  }
  int u = 0, r = 0;
  for (int q = 0; q < Q; q++) {
    dw_syncwarp();  // every lane's reads of row q - 1's stage are done
    if (q + D < Q) fetch_next(q + D);
    dw_commit();
    dw_wait<D>();
    dw_syncwarp();  // every lane's copies of row q have landed
    // the lane's tokens h kConvStrip + j: entry (h (kConvStrip + 1) + j + j / 8) kSw2Pairs + p
    const R* row = ring + (q % kSw2Stages) * S::ROW + h * (kConvStrip + 1) * kSw2Pairs + p;
    static_assert(kConvStrip == 8, "the ring's bank shift is per 8 tokens");
    float2 cr[NJ];
#pragma unroll
    for (int j = 0; j < NJ; j++) cr[j] = conv_unpack(row[(j + (j >> 3)) * kSw2Pairs]);
#pragma unroll
    for (int o = 0; o < kSw2Rows; o++) {
      const int v = r - o;
      if (v < 0 || v >= g.kh) continue;
      // kernel row (u, v)'s weights, tap j at wr[j kSw2WStride] (flipped for the transposed
      // convolution: W[c][kt-1-u][kh-1-v][kw-1-j])
      const int wrow = Flip ? ((g.kt - 1 - u) * g.kh + (g.kh - 1 - v)) * KW : (u * g.kh + v) * KW;
      const float* wr = wsp + wrow * kSw2WStride;
      float2 w[KW];
#pragma unroll
      for (int j = 0; j < KW; j++)
        w[j] = *reinterpret_cast<const float2*>(wr + (Flip ? KW - 1 - j : j) * kSw2WStride);
      // input column x0 - r_w + j feeds output x0 + i through tap j - i
#pragma unroll
      for (int j = 0; j < NJ; j++) {
#pragma unroll
        for (int i = 0; i < kConvStrip; i++) {
          if (j - i >= 0 && j - i < KW) conv_fma2(acc[o][i], w[j - i], cr[j]);
        }
      }
    }
    if (++r == rows) {
      r = 0;
      u++;
    }
  }
}

#ifdef __CUDACC__
// Writes the two strips acc (rows y0, y0 + 1 from column x0; channel pair c2), each element plus
// add's (nullable; may equal y); rows and columns past the volume are not written.
template <typename OutT, int NR>
__device__ __forceinline__ void conv_store_strips(const float2 (&acc)[NR][kConvStrip], const OutT* add,
                                                  OutT* y, const ConvGeo& g, int t, int y0, int x0,
                                                  int c2) {
#pragma unroll
  for (int r = 0; r < NR; r++) {
    if (y0 + r >= g.Hp) break;
    const int64_t base = (((int64_t)t * g.Hp + y0 + r) * g.Wp + x0) * g.C + 2 * c2;
#pragma unroll
    for (int i = 0; i < kConvStrip; i++) {
      if (x0 + i >= g.Wp) break;
      const int64_t o = base + (int64_t)i * g.C;
      float a = acc[r][i].x, b = acc[r][i].y;
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

template <int NR>
__device__ __forceinline__ void conv_acc_init(float2 (&acc)[NR][kConvStrip], float b0, float b1) {
#pragma unroll
  for (int r = 0; r < NR; r++)
#pragma unroll
    for (int i = 0; i < kConvStrip; i++) acc[r][i] = make_float2(b0, b1);
}

// Y = conv(X) (+ bias) (+ add), the weights read from global memory (kernels of more than
// kConvSwMaxTaps taps): one thread per (unit, channel pair), channel pairs fastest.  add
// (nullable) is added element by element (the attention output of Eq. 1; may equal y).  OutT: the
// output type (the input's, or fp32 for the offset network's first layer).
template <typename T, int KW, typename OutT = T>
__global__ void __launch_bounds__(kConvFwdThreads)
    dsa3d_dwconv3d_kernel(const T* __restrict__ x, const float* __restrict__ w,
                          const float* __restrict__ bias, const OutT* add, OutT* y,
                          const ConvGeo g, const int flip) {
  const int pairs = g.C / 2;
  const int nxs = (g.Wp + kConvStrip - 1) / kConvStrip;
  const int nyp = (g.Hp + 1) / 2;  // row pairs
  const int64_t items = (int64_t)g.F * nyp * nxs * pairs;
  const int64_t K = (int64_t)g.kt * g.kh * KW;
  for (int64_t it = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; it < items;
       it += (int64_t)gridDim.x * blockDim.x) {
    const int c2 = (int)(it % pairs);
    int t, y0, x0;
    conv_unit(it / pairs, nxs, nyp, t, y0, x0);
    float2 acc[2][kConvStrip];
    conv_acc_init(acc, bias ? __ldg(bias + 2 * c2) : 0.f, bias ? __ldg(bias + 2 * c2 + 1) : 0.f);
    conv_strip2<T, KW>(x, ConvWGlobal{w + 2 * c2 * K, K}, g, t, y0, x0, c2, flip != 0, acc);
    conv_store_strips(acc, add, y, g, t, y0, x0, c2);
  }
}

__device__ __forceinline__ void conv_cp_async4(float* dst, const float* src) {
  const unsigned d = (unsigned)__cvta_generic_to_shared(dst);
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;\n" ::"r"(d), "l"(src) : "memory");
}

// The same with the kernel staged in shared memory (at most kConvSwMaxTaps taps): a block owns
// one group of kConvGroupPairs channel pairs (one per lane) and kConvSwUnits units of one slot
// (conv_sw_unit), kConvSwUnits / kConvSwWarps per warp.  The group's weights are copied in once,
// tap-major (conv_sw_index), before any unit runs; dynamic shared memory: conv_sw_bytes(kt kh
// kw).  Blocks: group fastest, then slot.
template <typename T, int KW, typename OutT = T>
__global__ void __launch_bounds__(kConvSwWarps * 32)
    dsa3d_dwconv3d_sw_kernel(const T* __restrict__ x, const float* __restrict__ w,
                             const float* __restrict__ bias, const OutT* add, OutT* y,
                             const ConvGeo g, const int flip) {
  extern __shared__ __align__(16) float conv_sw[];
  const int pairs = g.C / 2;
  const unsigned groups = (unsigned)((pairs + kConvGroupPairs - 1) / kConvGroupPairs);
  const int grp = (int)(blockIdx.x % groups);
  const int64_t slot = blockIdx.x / groups;
  const int K = g.kt * g.kh * KW;
  const int c0 = 2 * kConvGroupPairs * grp;
  const int nch = min(2 * kConvGroupPairs, g.C - c0);
  const float* wg = w + (int64_t)c0 * K;  // the group's channels: nch x K contiguous floats
  for (int cc = 0; cc < nch; cc++)
    for (int k = threadIdx.x; k < K; k += blockDim.x)
      conv_cp_async4(conv_sw + conv_sw_index(k, cc), wg + (int64_t)cc * K + k);
  asm volatile("cp.async.wait_all;\n" ::: "memory");
  __syncthreads();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int c2 = kConvGroupPairs * grp + lane;
  if (c2 >= pairs) return;
  const int nxs = (g.Wp + kConvStrip - 1) / kConvStrip;
  const int nyp = (g.Hp + 1) / 2;
  const int64_t units = (int64_t)g.F * nyp * nxs;
  const int64_t slots = (units + kConvSwUnits - 1) / kConvSwUnits;
  const ConvWShared ws{conv_sw + 2 * lane};
  const float b0 = bias ? __ldg(bias + 2 * c2) : 0.f, b1 = bias ? __ldg(bias + 2 * c2 + 1) : 0.f;
  for (int i = 0; i < kConvSwUnits / kConvSwWarps; i++) {
    const int64_t unit = conv_sw_unit(slot, slots, warp, i);
    if (unit >= units) break;  // later steps' units are larger still
    int t, y0, x0;
    conv_unit(unit, nxs, nyp, t, y0, x0);
    float2 acc[2][kConvStrip];
    conv_acc_init(acc, b0, b1);
    conv_strip2<T, KW>(x, ws, g, t, y0, x0, c2, flip != 0, acc);
    conv_store_strips(acc, add, y, g, t, y0, x0, c2);
  }
}

// Bytes of the strip-pair forward's staged weights (16-byte aligned; the warps' rings follow).
__host__ __device__ __forceinline__ size_t conv_sw2_weight_bytes(int K) {
  return ((size_t)K * kSw2WStride * sizeof(float) + 15) & ~size_t(15);
}

// The forward on strip pairs (C a multiple of 32, at most kConvSwMaxTaps taps): a block owns one
// group of kSw2Pairs channel pairs and kSw2Units strip-pair units (kSw2Rows rows each) of one slot
// (conv_sw_unit over the strip-pair units), which its warps take in turn.  The group's weights are copied in once,
// tap-major with stride kSw2WStride; each warp then has kSw2Stages rows of ring.  Dynamic shared
// memory: conv_sw2_weight_bytes(K) + kConvSwWarps Sw2Ring<T, KW>::warp_bytes().  Registers capped
// for four blocks per SM up to k_w = 9 (126 at bf16 and k_w = 9, no spills; capped for three
// blocks the kernel takes 150 ms per launch at 1080p instead of 139) and three above.
template <typename T, int KW, typename OutT = T>
__global__ void __launch_bounds__(kConvSwWarps * 32, KW <= 9 ? 4 : 3)
    dsa3d_dwconv3d_sw2_kernel(const T* __restrict__ x, const float* __restrict__ w,
                              const float* __restrict__ bias, const OutT* add, OutT* y,
                              const ConvGeo g, const int flip) {
  using S = Sw2Ring<T, KW>;
  using R = typename S::R;
  extern __shared__ __align__(16) unsigned char conv_sw2[];
  float* ws_all = reinterpret_cast<float*>(conv_sw2);
  const int K = g.kt * g.kh * KW;
  const unsigned groups = (unsigned)(g.C / (2 * kSw2Pairs));
  const int grp = (int)(blockIdx.x % groups);
  const int64_t slot = blockIdx.x / groups;
  const int c0 = 2 * kSw2Pairs * grp;
  const float* wg = w + (int64_t)c0 * K;  // the group's 2 kSw2Pairs channels: contiguous floats
  for (int cc = 0; cc < 2 * kSw2Pairs; cc++)
    for (int k = threadIdx.x; k < K; k += blockDim.x)
      conv_cp_async4(ws_all + k * kSw2WStride + cc, wg + (int64_t)cc * K + k);
  asm volatile("cp.async.wait_all;\n" ::: "memory");
  __syncthreads();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  R* ring = reinterpret_cast<R*>(conv_sw2 + conv_sw2_weight_bytes(K)) + (size_t)warp * kSw2Stages * S::ROW;
  const int h = lane >> 4, p = lane & (kSw2Pairs - 1);
  const int c2 = kSw2Pairs * grp + p;
  const int nxp = (g.Wp + 2 * kConvStrip - 1) / (2 * kConvStrip);
  const int nyr = (g.Hp + kSw2Rows - 1) / kSw2Rows;
  const int64_t units = (int64_t)g.F * nyr * nxp;
  const int64_t slots = (units + kSw2Units - 1) / kSw2Units;
  const float* wsp = ws_all + 2 * p;
  const float b0 = bias ? __ldg(bias + 2 * c2) : 0.f, b1 = bias ? __ldg(bias + 2 * c2 + 1) : 0.f;
  const T* xg = x + c0;
  static_assert(kSw2Units % kConvSwWarps == 0, "whole steps of the warps");
  for (int i = 0; i < kSw2Units / kConvSwWarps; i++) {
    const int64_t unit = conv_sw_unit(slot, slots, warp, i);
    if (unit >= units) break;  // warp-uniform; later steps' units are larger still
    int t, y0, xb;
    conv_unit2(unit, nxp, nyr, t, y0, xb);
    float2 acc[kSw2Rows][kConvStrip];
    conv_acc_init(acc, b0, b1);
    if (flip)
      conv_strips_ring<T, KW, true>(ring, lane, xg, wsp, g, t, y0, xb, acc);
    else
      conv_strips_ring<T, KW, false>(ring, lane, xg, wsp, g, t, y0, xb, acc);
    conv_store_strips(acc, add, y, g, t, y0, xb + h * kConvStrip, c2);
  }
}

// dW (and db): one thread per work item (dw_decode, dw_walk); fp32 partial sums added with
// atomics into dweight [C][kt][kh][kw] and dbias [C] (both zeroed before).  The bias gradient is
// summed by the items of plane 0 and the first kernel-row group.  Dynamic shared memory: a
// DwRing<T, TD, KW>::warp_bytes() region per warp.  Coop (C a multiple of 64, so that every warp
// is 32 aligned pairs of one work item through the whole grid-stride loop): dw_fetch_warp, and a
// register cap for three blocks per SM (168 registers, a 20-byte spill at bf16 and k_w = 9: 222
// -> 183 ms per launch at 1080p); the per-lane copies spill over 100 bytes under that cap.
template <typename T, int KW, typename TD = T, bool Coop = false>
__global__ void __launch_bounds__(kConvDwThreads, Coop ? 3 : 1)
    dsa3d_dwconv3d_dw_kernel(const T* __restrict__ x, const TD* __restrict__ dy, float* dweight,
                             float* dbias, const ConvGeo g, const int frames_per_item) {
  extern __shared__ __align__(16) unsigned char dw_rings[];  // a DwRing region per warp
  using R = DwRing<T, TD, KW>;
  const R ring = R::at(dw_rings + (threadIdx.x >> 5) * R::warp_bytes(), threadIdx.x & 31);
  const int64_t items = dw_items(g, frames_per_item);
  const int64_t K = (int64_t)g.kt * g.kh * KW;
  for (int64_t it = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; it < items;
       it += (int64_t)gridDim.x * blockDim.x) {
    int c2, u, v0, x0, t0, t1;
    dw_decode(it, g, frames_per_item, c2, u, v0, x0, t0, t1);
    float2 dwr[kDwRows][KW];
#pragma unroll
    for (int i = 0; i < kDwRows; i++)
#pragma unroll
      for (int j = 0; j < KW; j++) dwr[i][j] = make_float2(0.f, 0.f);
    float db[2] = {0.f, 0.f};
    const bool with_db = u == 0 && v0 == 0;
    dw_walk<T, KW, TD, Coop>(x, dy, g, ring, c2, u, v0, x0, t0, t1, dwr, with_db, db);
#pragma unroll
    for (int i = 0; i < kDwRows; i++) {
      if (v0 + i >= g.kh) break;
      float* d0 = dweight + (int64_t)(2 * c2) * K + ((int64_t)u * g.kh + v0 + i) * KW;
#pragma unroll
      for (int j = 0; j < KW; j++) {
        atomicAdd(d0 + j, dwr[i][j].x);
        atomicAdd(d0 + K + j, dwr[i][j].y);
      }
    }
    if (with_db) {
      atomicAdd(dbias + 2 * c2, db[0]);
      atomicAdd(dbias + 2 * c2 + 1, db[1]);
    }
  }
}
#endif  // __CUDACC__

}  // namespace dsa3d
