// dsa3d_fwd.cuh -- 3D-DSA forward on CUDA cores (MegaSlide-DiT, arXiv 2607.22696, Eq. 1 and
// the softmax over the window that follows it).
//
// One warp computes one (head, query) at a time, persistent over a head-major item order (so
// neighbouring warps work on neighbouring tokens of one head and share K/V rows through L1/L2):
//   1. decode the offset; list the box tokens that carry a nonzero corner weight of a valid tap
//      (compacted in shared memory, with their box coordinates);
//   2. raw scores  s[j] = scale * log2(e) * q . K[j]  for every listed box token j: each lane
//      group of L = dh/E lanes reads one 16-byte chunk per lane of a key row (E elements), so a
//      row is one coalesced access; partial dots are reduced by a group transpose-sum;
//   3. tap scores  s_tau = sum_c w_c s[tau + c]  (8 trilinear weights), softmax over the valid
//      taps (base-2 exponent), lse;
//   4. value weights beta[j] = sum_c w_c p[j - c] / l  (the transpose of step 3);
//   5. out = sum_j beta[j] V[j]  with lanes over dh, reduced across the lane groups.
#pragma once

#include "dsa3d_common.cuh"

namespace dsa3d {

// Per-warp shared memory of the forward (bytes), for box size B and tap count K.
__host__ __device__ inline int fwd_warp_smem(int B, int K) {
  const int bytes = B * 4 /*tok*/ + B * 4 /*sraw*/ + B * 4 /*beta*/ + K * 4 /*ptap*/ + B * 2 /*bidx*/;
  return (bytes + 15) & ~15;
}
__host__ __device__ inline int table_smem(int B, int K) { return ((B + K) * 4 + 15) & ~15; }

// Fill the CTA-wide coordinate tables: box index -> (jt,jy,jx), tap index -> (u,v,w).
__device__ __forceinline__ void fill_tables(const Geo& g, int* relB, int* relT) {
  for (int e = threadIdx.x; e < g.B; e += blockDim.x) {
    const int jx = e % g.Bw, jy = (e / g.Bw) % g.Bh, jt = e / (g.Bw * g.Bh);
    relB[e] = pack3(jt, jy, jx);
  }
  for (int e = threadIdx.x; e < g.K; e += blockDim.x) {
    const int w = e % g.kw, v = (e / g.kw) % g.kh, u = e / (g.kw * g.kh);
    relT[e] = pack3(u, v, w);
  }
}

// Compact the box tokens with a nonzero corner weight of some valid tap.  Writes tok[] (token
// index) and bidx[] (box index) for count entries and zeroes zr[0..B) if zr != nullptr.
// Returns count (same value in every lane).
__device__ __forceinline__ int compact_box(const Geo& g, const Query& Q, const int* relB, int* tok,
                                           short* bidx, float* zr0, float* zr1, int lane) {
  int count = 0;
  for (int e0 = 0; e0 < g.B; e0 += 32) {
    const int e = e0 + lane;
    bool need = false;
    int t = 0;
    if (e < g.B) {
      int jt, jy, jx;
      unpack3(relB[e], jt, jy, jx);
      need = jt >= Q.lo[0] && jt <= Q.nhi[0] && jy >= Q.lo[1] && jy <= Q.nhi[1] &&
             jx >= Q.lo[2] && jx <= Q.nhi[2];
      if (need) t = (Q.o[0] + jt) * g.HW + (Q.o[1] + jy) * g.Wp + (Q.o[2] + jx);
      if (zr0) zr0[e] = 0.f;
      if (zr1) zr1[e] = 0.f;
    }
    const unsigned bal = __ballot_sync(kFull, need);
    if (need) {
      const int pos = count + __popc(bal & ((1u << lane) - 1u));
      DSA3D_DEVICE_CHECK(t >= 0 && (int64_t)t < g.N);
      tok[pos] = t;
      bidx[pos] = (short)e;
    }
    count += __popc(bal);
  }
  return count;
}

template <typename T, int DH, int WARPS>
__global__ void __launch_bounds__(WARPS * 32)
    dsa3d_fwd_kernel(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
                     const float* __restrict__ off, T* __restrict__ out, float* __restrict__ lse,
                     const Geo g, const int64_t n_items) {
  constexpr int E = Elems<T>::kPerLoad;  // elements per 16-byte chunk
  constexpr int L = DH / E;              // lanes per key row
  constexpr int G = 32 / L;              // key rows per warp step
  extern __shared__ __align__(16) unsigned char smem[];
  int* relB = reinterpret_cast<int*>(smem);
  int* relT = relB + g.B;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  unsigned char* wb = smem + table_smem(g.B, g.K) + warp * fwd_warp_smem(g.B, g.K);
  int* tok = reinterpret_cast<int*>(wb);
  float* sraw = reinterpret_cast<float*>(tok + g.B);
  float* beta = sraw + g.B;
  float* ptap = beta + g.B;
  short* bidx = reinterpret_cast<short*>(ptap + g.K);

  fill_tables(g, relB, relT);
  __syncthreads();

  const int grp = lane / L, sub = lane % L;
  const int64_t rs = (int64_t)g.heads * DH;  // token stride in elements
  const int cs[8] = {0, 1, g.Bw, g.Bw + 1, g.Bh * g.Bw, g.Bh * g.Bw + 1, g.Bh * g.Bw + g.Bw,
                     g.Bh * g.Bw + g.Bw + 1};
  const float sc = g.scale * kLog2e;

  for (int64_t item = (int64_t)blockIdx.x * WARPS + warp; item < n_items;
       item += (int64_t)gridDim.x * WARPS) {
    const int h = (int)(item / g.N);
    const int64_t n = item - (int64_t)h * g.N;
    const Query Q = decode_query(g, off, h, n);
    T* orow = out + (n * g.heads + h) * DH;
    if (!Q.ok) {
      if (grp == 0) {
        float z[E];
#pragma unroll
        for (int e = 0; e < E; e++) z[e] = 0.f;
        store16(orow + sub * E, z);
      }
      if (lane == 0 && lse) lse[(int64_t)h * g.N + n] = -INFINITY;
      continue;
    }
    float qv[E];
    load16(q + (n * g.heads + h) * DH + sub * E, qv);

    const int count = compact_box(g, Q, relB, tok, bidx, sraw, nullptr, lane);
    __syncwarp();

    // 2. raw scores over the compacted box tokens, 32 per round
    const T* kb = k + (int64_t)h * DH + sub * E;
    for (int c0 = 0; c0 < count; c0 += 32) {
      float part[L];
#pragma unroll
      for (int it = 0; it < L; it++) {
        const int c = c0 + it * G + grp;
        float kv[E];
        load16(kb + (int64_t)tok[min(c, count - 1)] * rs, kv);
        float acc = 0.f;
#pragma unroll
        for (int e = 0; e < E; e++) acc = fmaf(qv[e], kv[e], acc);
        part[it] = (c < count) ? acc : 0.f;
      }
      const float s = group_transpose_sum<L>(part, lane);
      const int c = c0 + sub * G + grp;
      if (c < count) sraw[bidx[c]] = s * sc;
    }
    __syncwarp();

    // 3. tap scores and softmax (base 2)
    float w8[8];
    corner_weights(Q.f, w8);
    float mx = -INFINITY;
    for (int tau = lane; tau < g.K; tau += 32) {
      int u, vv, w;
      unpack3(relT[tau], u, vv, w);
      float s = -INFINITY;
      if (u >= Q.lo[0] && u <= Q.hi[0] && vv >= Q.lo[1] && vv <= Q.hi[1] && w >= Q.lo[2] &&
          w <= Q.hi[2]) {
        const int e = (u * g.Bh + vv) * g.Bw + w;
        s = 0.f;
#pragma unroll
        for (int c = 0; c < 8; c++) s = fmaf(w8[c], sraw[e + cs[c]], s);
      }
      ptap[tau] = s;
      mx = fmaxf(mx, s);
    }
    mx = warp_max(mx);
    float lsum = 0.f;
    for (int tau = lane; tau < g.K; tau += 32) {
      const float s = ptap[tau];
      const float p = (s == -INFINITY) ? 0.f : exp2f(s - mx);
      ptap[tau] = p;
      lsum += p;
    }
    lsum = warp_sum(lsum);
    __syncwarp();

    // 4. value weights per compacted box token
    const float inv_l = 1.f / lsum;
    for (int c = lane; c < count; c += 32) {
      int jt, jy, jx;
      unpack3(relB[bidx[c]], jt, jy, jx);
      float b = 0.f;
#pragma unroll
      for (int cc = 0; cc < 8; cc++) {
        const int u = jt - ((cc >> 2) & 1), vv = jy - ((cc >> 1) & 1), w = jx - (cc & 1);
        if (u >= 0 && u < g.kt && vv >= 0 && vv < g.kh && w >= 0 && w < g.kw)
          b = fmaf(w8[cc], ptap[(u * g.kh + vv) * g.kw + w], b);
      }
      beta[c] = b * inv_l;
    }
    __syncwarp();

    // 5. out = sum_j beta[j] V[j]
    const T* vb = v + (int64_t)h * DH + sub * E;
    float acc[E];
#pragma unroll
    for (int e = 0; e < E; e++) acc[e] = 0.f;
    int c = grp;
    for (; c + G < count; c += 2 * G) {  // two rows in flight per lane
      const float b0 = beta[c], b1 = beta[c + G];
      float v0[E], v1[E];
      load16(vb + (int64_t)tok[c] * rs, v0);
      load16(vb + (int64_t)tok[c + G] * rs, v1);
#pragma unroll
      for (int e = 0; e < E; e++) acc[e] = fmaf(b1, v1[e], fmaf(b0, v0[e], acc[e]));
    }
    if (c < count) {
      const float b0 = beta[c];
      float v0[E];
      load16(vb + (int64_t)tok[c] * rs, v0);
#pragma unroll
      for (int e = 0; e < E; e++) acc[e] = fmaf(b0, v0[e], acc[e]);
    }
#pragma unroll
    for (int w = L; w < 32; w <<= 1)
#pragma unroll
      for (int e = 0; e < E; e++) acc[e] += __shfl_xor_sync(kFull, acc[e], w);
    if (grp == 0) store16(orow + sub * E, acc);
    if (lane == 0 && lse) lse[(int64_t)h * g.N + n] = (mx + log2f(lsum)) * kLn2;
    __syncwarp();
  }
}

}  // namespace dsa3d
