// dsa3d_pointwise.cuh -- the offset network's pointwise layer (MegaSlide-DiT, arXiv 2607.22696,
// the 3D-DSA definition: offsets are predicted by a depthwise 3-D convolution followed by a
// linear layer), written straight into the attention's offset layout:
//
//   O[n][o] = b[o] + sum_c Z[n][c] * Wp[c][o],   o = (h * K + tau) * 3 + a   (K = 1: per token)
//   offsets[h][n][tau][a] = O[n][o]
//
// Z [N][C] is the depthwise convolution's fp32 output (the offsets feed a floor, so they are
// formed in fp32 throughout).  A lane owns one output channel o (consecutive lanes read
// consecutive weights: coalesced) and a register tile of kPwTokens tokens; Z is read as float4
// broadcasts (all lanes of the warp read the same 16 bytes), 4 channels at a time: 64 FMAs per
// 20 loads.  The per-lane routine (pw_tile) is __host__ __device__ so that a host harness can run
// it on the CPU.
#pragma once

#include <stdint.h>

namespace dsa3d {

constexpr int kPwTokens = 16;  // tokens per lane tile

__host__ __device__ __forceinline__ float4 pw_ld4(const float* p) {
#ifdef __CUDA_ARCH__
  return __ldg(reinterpret_cast<const float4*>(p));
#else
  return *reinterpret_cast<const float4*>(p);
#endif
}
__host__ __device__ __forceinline__ float pw_ld(const float* p) {
#ifdef __CUDA_ARCH__
  return __ldg(p);
#else
  return *p;
#endif
}

// acc[t] = b[o] + sum_c Z[n0 + t][c] Wp[c][o] for t < kPwTokens with n0 + t < N (C % 4 == 0).
__host__ __device__ __forceinline__ void pw_tile(const float* __restrict__ z,
                                                 const float* __restrict__ wp,
                                                 const float* __restrict__ bp, int C, int width,
                                                 int64_t N, int64_t n0, int o,
                                                 float (&acc)[kPwTokens]) {
  const float b = pw_ld(bp + o);
#pragma unroll
  for (int t = 0; t < kPwTokens; t++) acc[t] = b;
  const int nt = (N - n0 < kPwTokens) ? (int)(N - n0) : kPwTokens;
  for (int c = 0; c < C; c += 4) {
    const float w0 = pw_ld(wp + (int64_t)c * width + o);
    const float w1 = pw_ld(wp + (int64_t)(c + 1) * width + o);
    const float w2 = pw_ld(wp + (int64_t)(c + 2) * width + o);
    const float w3 = pw_ld(wp + (int64_t)(c + 3) * width + o);
#pragma unroll
    for (int t = 0; t < kPwTokens; t++) {
      if (t < nt) {
        const float4 v = pw_ld4(z + (n0 + t) * C + c);
        acc[t] = fmaf(v.x, w0, fmaf(v.y, w1, fmaf(v.z, w2, fmaf(v.w, w3, acc[t]))));
      }
    }
  }
}

// Index of O[n][o] in the offset layout [heads][N][K][3] (K = 1: [heads][N][3]).
__host__ __device__ __forceinline__ int64_t pw_out_index(int64_t N, int taps3, int64_t n, int o) {
  const int h = o / taps3, rem = o % taps3;
  return ((int64_t)h * N + n) * taps3 + rem;
}

// Backward.  dO is the offsets' gradient in the offset layout, read through pw_out_index.
// dZ[n][c] = sum_o dO[n][o] Wp[c][o] for the tokens of one tile and one channel c.
__host__ __device__ __forceinline__ void pw_dz_tile(const float* __restrict__ doff,
                                                    const float* __restrict__ wp, int width,
                                                    int taps3, int64_t N, int64_t n0, int c,
                                                    float (&acc)[kPwTokens]) {
#pragma unroll
  for (int t = 0; t < kPwTokens; t++) acc[t] = 0.f;
  const int nt = (N - n0 < kPwTokens) ? (int)(N - n0) : kPwTokens;
  const float* wr = wp + (int64_t)c * width;
  for (int o = 0; o < width; o++) {
    const float w = pw_ld(wr + o);
#pragma unroll
    for (int t = 0; t < kPwTokens; t++)
      if (t < nt) acc[t] = fmaf(pw_ld(doff + pw_out_index(N, taps3, n0 + t, o)), w, acc[t]);
  }
}

constexpr int kPwChannels = 16;  // channels per thread in the weight gradient

// dWp[c0 + i][o] partial sums over tokens [nbeg, nend): acc[i] += Z[n][c0 + i] dO[n][o]
// (C % 16 == 0), and db += dO[n][o] when db != nullptr.
__host__ __device__ __forceinline__ void pw_dw_tile(const float* __restrict__ z,
                                                    const float* __restrict__ doff, int C,
                                                    int taps3, int64_t N, int64_t nbeg,
                                                    int64_t nend, int o, int c0,
                                                    float (&acc)[kPwChannels], float* db) {
  for (int64_t n = nbeg; n < nend; n++) {
    const float d = pw_ld(doff + pw_out_index(N, taps3, n, o));
    if (db) *db += d;
#pragma unroll
    for (int i = 0; i < kPwChannels; i += 4) {
      const float4 v = pw_ld4(z + n * C + c0 + i);
      acc[i] = fmaf(v.x, d, acc[i]);
      acc[i + 1] = fmaf(v.y, d, acc[i + 1]);
      acc[i + 2] = fmaf(v.z, d, acc[i + 2]);
      acc[i + 3] = fmaf(v.w, d, acc[i + 3]);
    }
  }
}

#ifdef __CUDACC__
// One thread per (token tile, output channel); width = heads * K * 3 outputs.
__global__ void __launch_bounds__(256)
    dsa3d_pointwise_offsets_kernel(const float* __restrict__ z, const float* __restrict__ wp,
                                   const float* __restrict__ bp, float* __restrict__ offsets,
                                   const int C, const int width, const int taps3, const int64_t N) {
  const int64_t tiles = (N + kPwTokens - 1) / kPwTokens;
  const int64_t items = tiles * width;
  for (int64_t it = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; it < items;
       it += (int64_t)gridDim.x * blockDim.x) {
    const int o = (int)(it % width);
    const int64_t n0 = (it / width) * kPwTokens;
    float acc[kPwTokens];
    pw_tile(z, wp, bp, C, width, N, n0, o, acc);
#pragma unroll
    for (int t = 0; t < kPwTokens; t++)
      if (n0 + t < N) offsets[pw_out_index(N, taps3, n0 + t, o)] = acc[t];
  }
}
// dZ: one thread per (token tile, channel), channels fastest.
__global__ void __launch_bounds__(256)
    dsa3d_pointwise_dz_kernel(const float* __restrict__ doff, const float* __restrict__ wp,
                              float* __restrict__ dz, const int C, const int width, const int taps3,
                              const int64_t N) {
  const int64_t tiles = (N + kPwTokens - 1) / kPwTokens;
  const int64_t items = tiles * C;
  for (int64_t it = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; it < items;
       it += (int64_t)gridDim.x * blockDim.x) {
    const int c = (int)(it % C);
    const int64_t n0 = (it / C) * kPwTokens;
    float acc[kPwTokens];
    pw_dz_tile(doff, wp, width, taps3, N, n0, c, acc);
#pragma unroll
    for (int t = 0; t < kPwTokens; t++)
      if (n0 + t < N) dz[(n0 + t) * C + c] = acc[t];
  }
}

// dWp, dbp: one thread per (token chunk, 16-channel group, output channel), outputs fastest;
// fp32 atomics into dwp [C][width] and dbp [width] (zeroed before).
__global__ void __launch_bounds__(256)
    dsa3d_pointwise_dw_kernel(const float* __restrict__ z, const float* __restrict__ doff,
                              float* dwp, float* dbp, const int C, const int width,
                              const int taps3, const int64_t N, const int64_t tokens_per_item) {
  const int groups = C / kPwChannels;
  const int64_t chunks = (N + tokens_per_item - 1) / tokens_per_item;
  const int64_t items = chunks * groups * width;
  for (int64_t it = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; it < items;
       it += (int64_t)gridDim.x * blockDim.x) {
    const int o = (int)(it % width);
    const int grp = (int)((it / width) % groups);
    const int64_t chunk = it / ((int64_t)width * groups);
    const int64_t nbeg = chunk * tokens_per_item;
    const int64_t nend = nbeg + tokens_per_item < N ? nbeg + tokens_per_item : N;
    float acc[kPwChannels];
#pragma unroll
    for (int i = 0; i < kPwChannels; i++) acc[i] = 0.f;
    float db = 0.f;
    pw_dw_tile(z, doff, C, taps3, N, nbeg, nend, o, grp * kPwChannels, acc, grp == 0 ? &db : nullptr);
#pragma unroll
    for (int i = 0; i < kPwChannels; i++)
      atomicAdd(dwp + (int64_t)(grp * kPwChannels + i) * width + o, acc[i]);
    if (grp == 0) atomicAdd(dbp + o, db);
  }
}
#endif  // __CUDACC__

}  // namespace dsa3d
