// conv_host_harness.cu -- runs the depthwise-convolution kernels' per-thread routines
// (conv_strip2, dw_walk from the library's dsa3d_conv.cuh) on the CPU, over every work item the
// GPU kernels would process, so that their indexing and arithmetic can be compared with the
// oracle without a GPU.  Test infrastructure: built by tests/test_conv_host.py with nvcc as
// host code; nothing here launches a kernel.
#include <stdint.h>

#include <algorithm>
#include <cmath>
#include <vector>

#include "dsa3d_conv.cuh"
#include "dsa3d_pointwise.cuh"

using namespace dsa3d;

namespace {

template <typename T, int KW, int NR = 2>
void store_strips(const float2 (&acc)[NR][kConvStrip], const ConvGeo& g, int t, int y0, int x0, int c2,
                  float* y) {
  for (int r = 0; r < NR && y0 + r < g.Hp; r++)
    for (int i = 0; i < kConvStrip && x0 + i < g.Wp; i++) {
      const int64_t o = (((int64_t)t * g.Hp + y0 + r) * g.Wp + x0 + i) * g.C + 2 * c2;
      y[o] = acc[r][i].x;
      y[o + 1] = acc[r][i].y;
    }
}

template <int NR>
void init_acc(float2 (&acc)[NR][kConvStrip], const float* b, int c2) {
  for (int r = 0; r < NR; r++)
    for (int i = 0; i < kConvStrip; i++)
      acc[r][i] = b ? make_float2(b[2 * c2], b[2 * c2 + 1]) : make_float2(0.f, 0.f);
}

// The forward as the library launches it: with at most kConvSwMaxTaps taps, the strip-pair
// kernel's blocks for C a multiple of 32 and the staged kernel's blocks otherwise (channel group,
// slot of units; each stages its group's weights and its warps take the units in turn); else the
// global kernel's items (unit, channel pair).
template <typename T, int KW>
void forward_all(const T* x, const float* w, const float* b, const ConvGeo& g, int flip, float* y) {
  const int pairs = g.C / 2, nxs = (g.Wp + kConvStrip - 1) / kConvStrip, nyp = (g.Hp + 1) / 2;
  const int64_t units = (int64_t)g.F * nyp * nxs;
  const int K = g.kt * g.kh * KW;
  float2 acc[2][kConvStrip];
  int t, y0, x0;
  if (K > kConvSwMaxTaps) {
    for (int64_t it = 0; it < units * pairs; it++) {
      const int c2 = (int)(it % pairs);
      conv_unit(it / pairs, nxs, nyp, t, y0, x0);
      init_acc(acc, b, c2);
      conv_strip2<T, KW>(x, ConvWGlobal{w + 2 * c2 * (int64_t)K, K}, g, t, y0, x0, c2, flip != 0, acc);
      store_strips<T, KW>(acc, g, t, y0, x0, c2, y);
    }
    return;
  }
  if (g.C % (2 * kSw2Pairs) == 0) {
    // the strip-pair kernel: each lane runs with its own copy of the warp's ring (the host fetch
    // copies every chunk of a row, so a lane alone sees what the whole warp would)
    using S = Sw2Ring<T, KW>;
    const int nxp = (g.Wp + 2 * kConvStrip - 1) / (2 * kConvStrip);
    const int nyr = (g.Hp + kSw2Rows - 1) / kSw2Rows;
    const int64_t units2 = (int64_t)g.F * nyr * nxp;
    const int64_t slots = (units2 + kSw2Units - 1) / kSw2Units;
    const int groups2 = g.C / (2 * kSw2Pairs);
    std::vector<float> ws((size_t)K * kSw2WStride);
    std::vector<typename S::R> ring((size_t)kSw2Stages * S::ROW);
    for (int64_t blk = 0; blk < slots * groups2; blk++) {
      const int grp = (int)(blk % groups2);
      const int64_t slot = blk / groups2;
      const int c0 = 2 * kSw2Pairs * grp;
      std::fill(ws.begin(), ws.end(), std::nanf(""));  // padding stays poisoned
      for (int cc = 0; cc < 2 * kSw2Pairs; cc++)
        for (int k = 0; k < K; k++) ws[(size_t)k * kSw2WStride + cc] = w[(int64_t)(c0 + cc) * K + k];
      for (int warp = 0; warp < kConvSwWarps; warp++)
        for (int lane = 0; lane < 32; lane++) {
          const int h = lane >> 4, p = lane & (kSw2Pairs - 1);
          const int c2 = kSw2Pairs * grp + p;
          for (int i = 0; i < kSw2Units / kConvSwWarps; i++) {
            const int64_t unit = conv_sw_unit(slot, slots, warp, i);
            if (unit >= units2) break;
            int xb;
            conv_unit2(unit, nxp, nyr, t, y0, xb);
            float2 acc4[kSw2Rows][kConvStrip];
            init_acc(acc4, b, c2);
            if (flip)
              conv_strips_ring<T, KW, true>(ring.data(), lane, x + c0, ws.data() + 2 * p, g, t, y0, xb, acc4);
            else
              conv_strips_ring<T, KW, false>(ring.data(), lane, x + c0, ws.data() + 2 * p, g, t, y0, xb, acc4);
            store_strips<T, KW, kSw2Rows>(acc4, g, t, y0, xb + h * kConvStrip, c2, y);
          }
        }
    }
    return;
  }
  const int groups = (pairs + kConvGroupPairs - 1) / kConvGroupPairs;
  const int64_t blocks = (units + kConvSwUnits - 1) / kConvSwUnits * groups;
  std::vector<float> sw(conv_sw_bytes(K) / sizeof(float));
  for (int64_t blk = 0; blk < blocks; blk++) {
    const int grp = (int)(blk % groups);
    const int64_t slot = blk / groups, slots = (units + kConvSwUnits - 1) / kConvSwUnits;
    const int c0 = 2 * kConvGroupPairs * grp;
    const int nch = std::min(2 * kConvGroupPairs, g.C - c0);
    std::fill(sw.begin(), sw.end(), std::nanf(""));  // unstaged slots poison the result
    for (int cc = 0; cc < nch; cc++)
      for (int k = 0; k < K; k++) sw[conv_sw_index(k, cc)] = w[(int64_t)(c0 + cc) * K + k];
    for (int warp = 0; warp < kConvSwWarps; warp++)
      for (int lane = 0; lane < 32; lane++) {
        const int c2 = kConvGroupPairs * grp + lane;
        if (c2 >= pairs) continue;
        for (int i = 0; i < kConvSwUnits / kConvSwWarps; i++) {
          const int64_t unit = conv_sw_unit(slot, slots, warp, i);
          if (unit >= units) break;
          conv_unit(unit, nxs, nyp, t, y0, x0);
          init_acc(acc, b, c2);
          conv_strip2<T, KW>(x, ConvWShared{sw.data() + 2 * lane}, g, t, y0, x0, c2, flip != 0, acc);
          store_strips<T, KW>(acc, g, t, y0, x0, c2, y);
        }
      }
  }
}

template <typename T, int KW, typename TD = T>
void dw_all(const T* x, const TD* dy, const ConvGeo& g, int frames_per_item, float* dw, float* db) {
  const int64_t K = (int64_t)g.kt * g.kh * KW;
  // one warp's staging region; each item runs as its pair's lane (c2 mod 32) of it, one lane at a
  // time; with C a multiple of 64 the library's warp-cooperative copies (each call copies the
  // whole warp's chunks here)
  using R = DwRing<T, TD, KW>;
  std::vector<double> region((R::warp_bytes() + sizeof(double) - 1) / sizeof(double));
  const bool coop = g.C % 64 == 0;
  for (int64_t it = 0; it < dw_items(g, frames_per_item); it++) {
    int c2, u, v0, x0, t0, t1;
    dw_decode(it, g, frames_per_item, c2, u, v0, x0, t0, t1);
    float2 dwr[kDwRows][KW] = {};
    float dbl[2] = {0.f, 0.f};
    const bool with_db = u == 0 && v0 == 0;
    const R ring = R::at(reinterpret_cast<unsigned char*>(region.data()), c2 & 31);
    if (coop)
      dw_walk<T, KW, TD, true>(x, dy, g, ring, c2, u, v0, x0, t0, t1, dwr, with_db, dbl);
    else
      dw_walk<T, KW, TD, false>(x, dy, g, ring, c2, u, v0, x0, t0, t1, dwr, with_db, dbl);
    for (int i = 0; i < kDwRows && v0 + i < g.kh; i++)
      for (int j = 0; j < KW; j++) {
        const int64_t o = (int64_t)(2 * c2) * K + ((int64_t)u * g.kh + v0 + i) * KW + j;
        dw[o] += dwr[i][j].x;
        dw[o + K] += dwr[i][j].y;
      }
    if (with_db) {
      db[2 * c2] += dbl[0];
      db[2 * c2 + 1] += dbl[1];
    }
  }
}

template <template <typename, int> class Fn, typename T, typename... A>
int by_kw(int kw, A... a) {
  switch (kw) {
    case 1: Fn<T, 1>::run(a...); return 0;
    case 3: Fn<T, 3>::run(a...); return 0;
    case 5: Fn<T, 5>::run(a...); return 0;
    case 7: Fn<T, 7>::run(a...); return 0;
    case 9: Fn<T, 9>::run(a...); return 0;
    case 11: Fn<T, 11>::run(a...); return 0;
    case 13: Fn<T, 13>::run(a...); return 0;
    case 15: Fn<T, 15>::run(a...); return 0;
    default: return -1;
  }
}
template <typename T, int KW>
struct Fwd {
  static void run(const void* x, const float* w, const float* b, ConvGeo g, int flip, float* y) {
    forward_all<T, KW>(static_cast<const T*>(x), w, b, g, flip, y);
  }
};
template <typename T, int KW>
struct DwMixed {  // dY in fp32 (the offset network's backward)
  static void run(const void* x, const void* dy, ConvGeo g, int fpi, float* dw, float* db) {
    dw_all<T, KW, float>(static_cast<const T*>(x), static_cast<const float*>(dy), g, fpi, dw, db);
  }
};
template <typename T, int KW>
struct Dw {
  static void run(const void* x, const void* dy, ConvGeo g, int fpi, float* dw, float* db) {
    dw_all<T, KW>(static_cast<const T*>(x), static_cast<const T*>(dy), g, fpi, dw, db);
  }
};

ConvGeo geo(int F, int Hp, int Wp, int C, int kt, int kh, int kw) {
  ConvGeo g;
  g.F = F; g.Hp = Hp; g.Wp = Wp; g.C = C; g.kt = kt; g.kh = kh; g.kw = kw;
  g.N = (int64_t)F * Hp * Wp;
  return g;
}

}  // namespace

extern "C" {

// io: 0 = fp32, 1 = bf16.  y [N][C] fp32 (every element written).
int conv_host_forward(int io, const void* x, const float* w, const float* b, int F, int Hp, int Wp,
                      int C, int kt, int kh, int kw, int flip, float* y) {
  if (C % 2) return -1;
  const ConvGeo g = geo(F, Hp, Wp, C, kt, kh, kw);
  return io ? by_kw<Fwd, __nv_bfloat16>(kw, x, w, b, g, flip, y)
            : by_kw<Fwd, float>(kw, x, w, b, g, flip, y);
}

// dw [C][kt][kh][kw], db [C]: fp32, accumulated into (zero them first).
int conv_host_dw(int io, const void* x, const void* dy, int F, int Hp, int Wp, int C, int kt, int kh,
                 int kw, int frames_per_item, float* dw, float* db) {
  if (C % 2 || frames_per_item < 1) return -1;
  const ConvGeo g = geo(F, Hp, Wp, C, kt, kh, kw);
  return io ? by_kw<Dw, __nv_bfloat16>(kw, x, dy, g, frames_per_item, dw, db)
            : by_kw<Dw, float>(kw, x, dy, g, frames_per_item, dw, db);
}

// dW with x in the I/O type (io) and dY in fp32.
int conv_host_dw_mixed(int io, const void* x, const float* dy, int F, int Hp, int Wp, int C, int kt,
                       int kh, int kw, int frames_per_item, float* dw, float* db) {
  if (C % 2 || frames_per_item < 1) return -1;
  const ConvGeo g = geo(F, Hp, Wp, C, kt, kh, kw);
  return io ? by_kw<DwMixed, __nv_bfloat16>(kw, x, (const void*)dy, g, frames_per_item, dw, db)
            : by_kw<DwMixed, float>(kw, x, (const void*)dy, g, frames_per_item, dw, db);
}

// The pointwise layer's backward over every work item of its two kernels: dz [N][C] written;
// dwp [C][width] and dbp [width] accumulated into (zero them first).
int pw_host_backward(const float* z, const float* doff, const float* wp, int C, int width, int taps3,
                     long long N, long long tokens_per_item, float* dz, float* dwp, float* dbp) {
  if (C % kPwChannels || width % taps3 || tokens_per_item < 1) return -1;
  const int64_t tiles = (N + kPwTokens - 1) / kPwTokens;
  for (int64_t tile = 0; tile < tiles; tile++)
    for (int c = 0; c < C; c++) {
      float acc[kPwTokens];
      pw_dz_tile(doff, wp, width, taps3, N, tile * kPwTokens, c, acc);
      for (int t = 0; t < kPwTokens && tile * kPwTokens + t < N; t++) dz[(tile * kPwTokens + t) * C + c] = acc[t];
    }
  const int64_t chunks = (N + tokens_per_item - 1) / tokens_per_item;
  for (int64_t chunk = 0; chunk < chunks; chunk++)
    for (int grp = 0; grp < C / kPwChannels; grp++)
      for (int o = 0; o < width; o++) {
        float acc[kPwChannels] = {};
        float db = 0.f;
        const int64_t nbeg = chunk * tokens_per_item;
        const int64_t nend = nbeg + tokens_per_item < N ? nbeg + tokens_per_item : N;
        pw_dw_tile(z, doff, C, taps3, N, nbeg, nend, o, grp * kPwChannels, acc, grp == 0 ? &db : nullptr);
        for (int i = 0; i < kPwChannels; i++) dwp[(int64_t)(grp * kPwChannels + i) * width + o] += acc[i];
        if (grp == 0) dbp[o] += db;
      }
  return 0;
}

// The offset network's pointwise layer over every (token tile, output channel) item:
// z [N][C] fp32, wp [C][width], bp [width]; offsets [heads][N][taps3 / 3][3] (written).
int pw_host_offsets(const float* z, const float* wp, const float* bp, int C, int width, int taps3,
                    long long N, float* offsets) {
  if (C % 4 || width % taps3) return -1;
  const int64_t tiles = (N + kPwTokens - 1) / kPwTokens;
  for (int64_t tile = 0; tile < tiles; tile++)
    for (int o = 0; o < width; o++) {
      float acc[kPwTokens];
      pw_tile(z, wp, bp, C, width, N, tile * kPwTokens, o, acc);
      for (int t = 0; t < kPwTokens && tile * kPwTokens + t < N; t++)
        offsets[pw_out_index(N, taps3, tile * kPwTokens + t, o)] = acc[t];
    }
  return 0;
}

}  // extern "C"
