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
#endif  // __CUDACC__

}  // namespace dsa3d
