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
// index and e_x to the sorted position), order (sort each bucket's queries by token index).  The
// fill's order within one bucket follows the atomics; the order step makes the sorted arrays,
// and with them every kernel that reads them, the same from run to run.
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

// ---- deterministic order within a bucket ---------------------------------------------------
// dsa3d_sort_order_kernel sorts each bucket's run of sorted_n by token index: one thread per
// bucket of at most kSmallBucket queries (insertion sort in place); larger buckets are listed in
// big[] (count in *nbig, zero on entry) for dsa3d_sort_order_big_kernel, one CTA per listed
// bucket: bitonic sorts of kBigChunk-query chunks in shared memory, then bottom-up merges of the
// sorted runs between the run and a scratch array of the same positions.  sorted_ex is the same
// for every query of a bucket, so it needs no reordering.  nb = buckets of the head group
// (hg * E1 - 1: bucket b's run is [start[b], start[b+1])).
constexpr int kSmallBucket = 32;
constexpr int kBigThreads = 512;
constexpr int kBigChunk = 4096;  // ints per shared-memory chunk (a power of two)

__global__ void dsa3d_sort_order_kernel(const int* __restrict__ start, const int64_t nb,
                                        int* __restrict__ sorted_n, int* __restrict__ big,
                                        int* __restrict__ nbig) {
  for (int64_t b = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; b < nb;
       b += (int64_t)gridDim.x * blockDim.x) {
    const int lo = start[b], S = start[b + 1] - lo;
    if (S < 2) continue;
    if (S > kSmallBucket) {
      big[atomicAdd(nbig, 1)] = (int)b;
      continue;
    }
    int* a = sorted_n + lo;
    for (int i = 1; i < S; i++) {
      const int x = a[i];
      int j = i - 1;
      while (j >= 0 && a[j] > x) {
        a[j + 1] = a[j];
        j--;
      }
      a[j + 1] = x;
    }
  }
}

__global__ void __launch_bounds__(kBigThreads)
    dsa3d_sort_order_big_kernel(const int* __restrict__ start, const int* __restrict__ big,
                                const int* __restrict__ nbig, int* __restrict__ sorted_n,
                                int* __restrict__ scratch) {
  __shared__ int sh[kBigChunk];
  const int count = *nbig;
  for (int e = blockIdx.x; e < count; e += gridDim.x) {
    const int b = big[e];
    const int lo = start[b], S = start[b + 1] - lo;
    int* a = sorted_n + lo;
    // 1. sort each chunk (padded to a power of two with INT_MAX, larger than any token index)
    for (int c0 = 0; c0 < S; c0 += kBigChunk) {
      const int n = min(kBigChunk, S - c0);
      int P = 1;
      while (P < n) P <<= 1;
      for (int i = threadIdx.x; i < P; i += blockDim.x) sh[i] = i < n ? a[c0 + i] : 0x7fffffff;
      __syncthreads();
      for (int k = 2; k <= P; k <<= 1)
        for (int j = k >> 1; j > 0; j >>= 1) {
          for (int i = threadIdx.x; i < P; i += blockDim.x) {
            const int l = i ^ j;
            if (l > i) {
              const bool up = (i & k) == 0;
              const int x = sh[i], y = sh[l];
              if ((x > y) == up) {
                sh[i] = y;
                sh[l] = x;
              }
            }
          }
          __syncthreads();
        }
      for (int i = threadIdx.x; i < n; i += blockDim.x) a[c0 + i] = sh[i];
      __syncthreads();
    }
    // 2. merge pairs of sorted runs of width w (token indices are distinct: no ties); output
    //    element o of a pair takes the co-rank i (elements of the first run before it) by binary
    //    search along the merge path
    int* src = a;
    int* dst = scratch + lo;
    for (int w = kBigChunk; w < S; w <<= 1) {
      for (int o = threadIdx.x; o < S; o += blockDim.x) {
        const int p0 = (o / (2 * w)) * (2 * w);
        const int n1 = min(w, S - p0), n2 = max(0, min(w, S - p0 - w));
        const int* A = src + p0;
        const int* B = A + n1;
        const int k = o - p0;
        int ilo = max(0, k - n2), ihi = min(k, n1);
        while (ilo < ihi) {
          const int i = (ilo + ihi) >> 1;
          if (A[i] < B[k - i - 1]) ilo = i + 1;
          else ihi = i;
        }
        const int i = ilo, j = k - ilo;
        dst[o] = (i < n1 && (j >= n2 || A[i] < B[j])) ? A[i] : B[j];
      }
      __syncthreads();
      int* tmp = src;
      src = dst;
      dst = tmp;
    }
    if (src != a) {
      for (int i = threadIdx.x; i < S; i += blockDim.x) a[i] = src[i];
    }
    __syncthreads();
  }
}

}  // namespace dsa3d
