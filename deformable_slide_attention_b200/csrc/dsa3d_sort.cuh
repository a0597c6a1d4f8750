// dsa3d_sort.cuh -- counting sort of queries by box origin, per head.
//
// The box of a query with origin o = p + i - r spans o .. o + k on each axis; it meets the volume
// iff o + k lies in [0, dim + k).  Buckets are the extended origins e = o + k over the grid
// Et x Ey x Ex = (F + kt) x (Hp + kh) x (Wp + kw), x fastest, one bucket array per head with one
// extra end entry ([E + 1] per head).  After the sort, the queries of one "bucket row" (fixed
// e_t, e_y) are contiguous and ordered by e_x, so consecutive ones share box rows and their keys
// fall in a narrow x-range of the same key rows.
//
// Steps: count (per query: bucket and rank by atomicAdd), exclusive scan over all heads' bucket
// counts (block sums, a single-block scan of those, block-local scans), fill (scatter token
// index and e_x to the sorted position).  The order within one bucket follows the atomics.
#pragma once

#include "dsa3d_common.cuh"

namespace dsa3d {

struct SortGeo {
  int Et, Ey, Ex;
  int64_t E1;  // buckets per head + 1
};

// Per query of heads [h0, h0 + hg): bucket and rank; queries without a valid tap get key -1.
// Such queries' rows of `out` (the forward's out, or the backward's dq) are zeroed here when out
// is given, their lse set to -inf when lse is given and their offset gradient zeroed when doff is.
template <typename T, int DH>
__global__ void dsa3d_sort_count_kernel(const float* __restrict__ off, const Geo g, const SortGeo sg,
                                        const int h0, const int hg, int* __restrict__ cnt,
                                        int* __restrict__ qkey, int* __restrict__ qrank,
                                        T* __restrict__ out, float* __restrict__ lse,
                                        float* __restrict__ doff) {
  const int64_t items = (int64_t)hg * g.N;
  for (int64_t it = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; it < items;
       it += (int64_t)gridDim.x * blockDim.x) {
    const int hh = (int)(it / g.N);
    const int64_t n = it - (int64_t)hh * g.N;
    const int h = h0 + hh;
    const Query Q = decode_query(g, off, h, n);
    if (!Q.ok) {
      qkey[it] = -1;
      if (out) {
        T* row = out + (n * g.heads + h) * DH;
        float z[Elems<T>::kPerLoad];
#pragma unroll
        for (int e = 0; e < Elems<T>::kPerLoad; e++) z[e] = 0.f;
#pragma unroll
        for (int c = 0; c < DH / Elems<T>::kPerLoad; c++) store16(row + c * Elems<T>::kPerLoad, z);
      }
      if (lse) lse[(int64_t)h * g.N + n] = -INFINITY;
      if (doff) {
        float* od = doff + ((int64_t)h * g.N + n) * 3;
        od[0] = od[1] = od[2] = 0.f;
      }
      continue;
    }
    const int et = Q.o[0] + g.kt, ey = Q.o[1] + g.kh, ex = Q.o[2] + g.kw;
    DSA3D_DEVICE_CHECK(et >= 0 && et < sg.Et && ey >= 0 && ey < sg.Ey && ex >= 0 && ex < sg.Ex);
    const int64_t b = (int64_t)hh * sg.E1 + ((int64_t)et * sg.Ey + ey) * sg.Ex + ex;
    qkey[it] = (int)(b - (int64_t)hh * sg.E1);
    qrank[it] = atomicAdd(cnt + b, 1);
  }
}

constexpr int kScanThreads = 256;
constexpr int kScanPerThread = 8;
constexpr int kScanTile = kScanThreads * kScanPerThread;  // 2048 entries per block

__device__ __forceinline__ int block_exclusive_scan(int x, int* sh, int& total) {
  // sh: kScanThreads/32 ints.  Returns the exclusive prefix of x over the block.
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int incl = x;
#pragma unroll
  for (int d = 1; d < 32; d <<= 1) {
    const int y = __shfl_up_sync(kFull, incl, d);
    if (lane >= d) incl += y;
  }
  if (lane == 31) sh[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    int w = (lane < kScanThreads / 32) ? sh[lane] : 0;
    int wi = w;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
      const int y = __shfl_up_sync(kFull, wi, d);
      if (lane >= d) wi += y;
    }
    if (lane < kScanThreads / 32) sh[lane] = wi - w;
    if (lane == kScanThreads / 32 - 1) sh[kScanThreads / 32] = wi;
  }
  __syncthreads();
  const int res = sh[warp] + incl - x;
  total = sh[kScanThreads / 32];
  __syncthreads();
  return res;
}

// Block sums of a[0..n).
__global__ void __launch_bounds__(kScanThreads)
    dsa3d_scan_blocks_kernel(const int* __restrict__ a, const int64_t n, int* __restrict__ bsum) {
  __shared__ int sh[kScanThreads / 32 + 1];
  const int64_t base = (int64_t)blockIdx.x * kScanTile + (int64_t)threadIdx.x * kScanPerThread;
  int s = 0;
#pragma unroll
  for (int i = 0; i < kScanPerThread; i++)
    if (base + i < n) s += a[base + i];
  int total;
  block_exclusive_scan(s, sh, total);
  if (threadIdx.x == 0) bsum[blockIdx.x] = total;
}

// Exclusive scan of bsum[0..nb) in place, one block.
__global__ void __launch_bounds__(kScanThreads)
    dsa3d_scan_sums_kernel(int* __restrict__ bsum, const int nb) {
  __shared__ int sh[kScanThreads / 32 + 1];
  int carry = 0;
  for (int base = 0; base < nb; base += kScanThreads) {
    const int i = base + threadIdx.x;
    const int x = (i < nb) ? bsum[i] : 0;
    int total;
    const int ex = block_exclusive_scan(x, sh, total);
    if (i < nb) bsum[i] = carry + ex;
    carry += total;
  }
}

// In-place exclusive scan of a[0..n) given the scanned block sums.
__global__ void __launch_bounds__(kScanThreads)
    dsa3d_scan_apply_kernel(int* __restrict__ a, const int64_t n, const int* __restrict__ bsum) {
  __shared__ int sh[kScanThreads / 32 + 1];
  const int64_t base = (int64_t)blockIdx.x * kScanTile + (int64_t)threadIdx.x * kScanPerThread;
  int v[kScanPerThread];
  int s = 0;
#pragma unroll
  for (int i = 0; i < kScanPerThread; i++) {
    v[i] = (base + i < n) ? a[base + i] : 0;
    s += v[i];
  }
  int total;
  int run = block_exclusive_scan(s, sh, total) + bsum[blockIdx.x];
#pragma unroll
  for (int i = 0; i < kScanPerThread; i++) {
    if (base + i < n) a[base + i] = run;
    run += v[i];
  }
}

// Scatter each bucketed query to its sorted position: token index and extended x origin.
__global__ void dsa3d_sort_fill_kernel(const int* __restrict__ start, const int* __restrict__ qkey,
                                       const int* __restrict__ qrank, const Geo g, const SortGeo sg,
                                       const int hg, int* __restrict__ sorted_n,
                                       int* __restrict__ sorted_ex) {
  const int64_t items = (int64_t)hg * g.N;
  for (int64_t it = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; it < items;
       it += (int64_t)gridDim.x * blockDim.x) {
    const int key = qkey[it];
    if (key < 0) continue;
    const int hh = (int)(it / g.N);
    const int64_t n = it - (int64_t)hh * g.N;
    const int64_t pos = (int64_t)start[(int64_t)hh * sg.E1 + key] + qrank[it];
    DSA3D_DEVICE_CHECK(pos >= 0 && pos < items);
    sorted_n[pos] = (int)n;
    sorted_ex[pos] = key % sg.Ex;
  }
}

}  // namespace dsa3d
