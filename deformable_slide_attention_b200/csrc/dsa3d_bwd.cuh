// dsa3d_bwd.cuh -- 3D-DSA backward on CUDA cores.
//
// The paper trains through the operator (full-parameter adaptation, MegaSlide-DiT arXiv
// 2607.22696) but gives no backward; this is the exact derivative of the forward with the tap
// mask and the integer offset parts held fixed.  Per (head, query), with P = exp(s - lse),
// dP_tau = dO . v~_tau, D = sum_tau P_tau dP_tau (= dO . out for the exact out, so the stored,
// rounded out is not needed) and dS_tau = P_tau (dP_tau - D):
//   dq        = scale * sum_tau dS_tau k~_tau        = scale * sum_j gamma[j] K[j]
//   dK[j]    += scale * gamma[j] * q,   gamma[j] = sum_c w_c dS[j - c]
//   dV[j]    += beta[j] * dO,           beta[j]  = sum_c w_c P[j - c]
//   doff_a    = sum_tau scale dS_tau q . dk~_tau/df_a + P_tau dO . dv~_tau/df_a
// One warp per (head, query) recomputes the raw box dots q.K[j] and dO.V[j], forms the tap
// quantities, writes dq and doff, and scatters dK/dV with 16-byte vector reductions into an fp32
// accumulator ([N][heads in pass][dh]); a finalize pass converts it to the I/O type.
#pragma once

#include "dsa3d_fwd.cuh"

namespace dsa3d {

__host__ __device__ inline int bwd_warp_smem(int B, int K) {
  const int bytes = B * 4 /*tok*/ + 4 * B * 4 /*sraw, praw, gamma, beta*/ + 2 * K * 4 /*P, dS*/ +
                    B * 2 /*bidx*/;
  return (bytes + 15) & ~15;
}

__device__ __forceinline__ void red_add16(float* p, const float* x) {
  atomicAdd(reinterpret_cast<float4*>(p), make_float4(x[0], x[1], x[2], x[3]));
}

// acc_k/acc_v: fp32 accumulators, row (token, head h) at (tok * acc_heads + (h - acc_h0)) * DH.
template <typename T, int DH, int WARPS>
__global__ void __launch_bounds__(WARPS * 32)
    dsa3d_bwd_kernel(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
                     const float* __restrict__ off, const float* __restrict__ lse,
                     const T* __restrict__ dout, T* __restrict__ dq,
                     float* __restrict__ doff, float* __restrict__ acc_k, float* __restrict__ acc_v,
                     const int acc_heads, const int h0, const Geo g, const int64_t n_items) {
  constexpr int E = Elems<T>::kPerLoad;
  constexpr int L = DH / E;
  constexpr int G = 32 / L;
  extern __shared__ __align__(16) unsigned char smem[];
  int* relB = reinterpret_cast<int*>(smem);
  int* relT = relB + g.B;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  unsigned char* wb = smem + table_smem(g.B, g.K) + warp * bwd_warp_smem(g.B, g.K);
  int* tok = reinterpret_cast<int*>(wb);
  float* sraw = reinterpret_cast<float*>(tok + g.B);
  float* praw = sraw + g.B;
  float* gam = praw + g.B;
  float* bet = gam + g.B;
  float* ptap = bet + g.B;
  float* dstap = ptap + g.K;
  short* bidx = reinterpret_cast<short*>(dstap + g.K);

  fill_tables(g, relB, relT);
  __syncthreads();

  const int grp = lane / L, sub = lane % L;
  const int64_t rs = (int64_t)g.heads * DH;
  const int cs[8] = {0, 1, g.Bw, g.Bw + 1, g.Bh * g.Bw, g.Bh * g.Bw + 1, g.Bh * g.Bw + g.Bw,
                     g.Bh * g.Bw + g.Bw + 1};
  const float sc = g.scale * kLog2e;

  for (int64_t item = (int64_t)blockIdx.x * WARPS + warp; item < n_items;
       item += (int64_t)gridDim.x * WARPS) {
    const int h = h0 + (int)(item / g.N);
    const int64_t n = item - (int64_t)(h - h0) * g.N;
    const int64_t row = (n * g.heads + h) * DH + sub * E;
    const Query Q0 = decode_query(g, off, h, n, /*for_grad=*/true);
    const float lse_n = __ldg(lse + (int64_t)h * g.N + n);
    const bool ok = Q0.ok && lse_n != -INFINITY;
    if (!ok) {
      if (grp == 0) {
        float z[E];
#pragma unroll
        for (int e = 0; e < E; e++) z[e] = 0.f;
        store16(dq + row, z);
      }
      if (lane < 3) doff[((int64_t)h * g.N + n) * 3 + lane] = 0.f;
      continue;
    }
    const Query& Q = Q0;
    float qv[E], gv[E];
    load16(q + row, qv);
    load16(dout + row, gv);

    const int count = compact_box(g, Q, relB, tok, bidx, sraw, praw, lane);
    __syncwarp();

    // raw box dots: sraw = scale*log2e * q.K[j], praw = dO.V[j]
    const T* kb = k + (int64_t)h * DH + sub * E;
    const T* vb = v + (int64_t)h * DH + sub * E;
    for (int c0 = 0; c0 < count; c0 += 32) {
      float ps[L], pp[L];
#pragma unroll
      for (int it = 0; it < L; it++) {
        const int c = c0 + it * G + grp;
        const int64_t tr = (int64_t)tok[min(c, count - 1)] * rs;
        float kv[E], vv[E];
        load16(kb + tr, kv);
        load16(vb + tr, vv);
        float a = 0.f, b = 0.f;
#pragma unroll
        for (int e = 0; e < E; e++) {
          a = fmaf(qv[e], kv[e], a);
          b = fmaf(gv[e], vv[e], b);
        }
        ps[it] = (c < count) ? a : 0.f;
        pp[it] = (c < count) ? b : 0.f;
      }
      const float s = group_transpose_sum<L>(ps, lane);
      const float p = group_transpose_sum<L>(pp, lane);
      const int c = c0 + sub * G + grp;
      if (c < count) {
        sraw[bidx[c]] = s * sc;
        praw[bidx[c]] = p;
      }
    }
    __syncwarp();

    // taps: P, dP and the sums that give D and the offset gradient.  With ds_a, dp_a the
    // derivatives of the tap's score (log2 units) and dP along f_a:
    //   doff_a = sum P (dP - D) ds_a ln2 + P dp_a = ln2 (A_a - D B_a) + C_a,
    //   A_a = sum P dP ds_a,  B_a = sum P ds_a,  C_a = sum P dp_a,  D = sum P dP.
    float w8[8], dw[3][8];
    corner_weights(Q.f, w8);
    corner_dweights(Q.f, dw);
    const float lse2 = lse_n * kLog2e;
    float Dp = 0.f, A[3] = {0.f, 0.f, 0.f}, Bs[3] = {0.f, 0.f, 0.f}, C[3] = {0.f, 0.f, 0.f};
    for (int tau = lane; tau < g.K; tau += 32) {
      int u, vv, w;
      unpack3(relT[tau], u, vv, w);
      float P = 0.f, PdP = 0.f;
      if (u >= Q.lo[0] && u <= Q.hi[0] && vv >= Q.lo[1] && vv <= Q.hi[1] && w >= Q.lo[2] &&
          w <= Q.hi[2]) {
        const int e = (u * g.Bh + vv) * g.Bw + w;
        float s = 0.f, dP = 0.f, ds[3] = {0.f, 0.f, 0.f}, dp[3] = {0.f, 0.f, 0.f};
#pragma unroll
        for (int c = 0; c < 8; c++) {
          const float a = sraw[e + cs[c]], b = praw[e + cs[c]];
          s = fmaf(w8[c], a, s);
          dP = fmaf(w8[c], b, dP);
#pragma unroll
          for (int ax = 0; ax < 3; ax++) {
            ds[ax] = fmaf(dw[ax][c], a, ds[ax]);
            dp[ax] = fmaf(dw[ax][c], b, dp[ax]);
          }
        }
        P = exp2f(s - lse2);
        PdP = P * dP;
        Dp += PdP;
#pragma unroll
        for (int ax = 0; ax < 3; ax++) {
          A[ax] = fmaf(PdP, ds[ax], A[ax]);
          Bs[ax] = fmaf(P, ds[ax], Bs[ax]);
          C[ax] = fmaf(P, dp[ax], C[ax]);
        }
      }
      ptap[tau] = P;
      dstap[tau] = PdP;
    }
    const float D = warp_sum(Dp);
#pragma unroll
    for (int ax = 0; ax < 3; ax++) {
      A[ax] = warp_sum(A[ax]);
      Bs[ax] = warp_sum(Bs[ax]);
      C[ax] = warp_sum(C[ax]);
    }
    if (lane == 0) {
      float* od = doff + ((int64_t)h * g.N + n) * 3;
#pragma unroll
      for (int ax = 0; ax < 3; ax++) od[ax] = fmaf(kLn2, fmaf(-D, Bs[ax], A[ax]), C[ax]);
    }
    __syncwarp();

    // splat to box tokens
    for (int c = lane; c < count; c += 32) {
      int jt, jy, jx;
      unpack3(relB[bidx[c]], jt, jy, jx);
      float gp = 0.f, be = 0.f;  // splats of P dP and of P; gamma = splat(P (dP - D))
#pragma unroll
      for (int cc = 0; cc < 8; cc++) {
        const int u = jt - ((cc >> 2) & 1), vv = jy - ((cc >> 1) & 1), w = jx - (cc & 1);
        if (u >= 0 && u < g.kt && vv >= 0 && vv < g.kh && w >= 0 && w < g.kw) {
          const int t = (u * g.kh + vv) * g.kw + w;
          gp = fmaf(w8[cc], dstap[t], gp);
          be = fmaf(w8[cc], ptap[t], be);
        }
      }
      gam[c] = fmaf(-D, be, gp);
      bet[c] = be;
    }
    __syncwarp();

    // dq (gather) and dK/dV (scatter)
    float dqa[E];
#pragma unroll
    for (int e = 0; e < E; e++) dqa[e] = 0.f;
    const int64_t acc_h = (int64_t)(h - h0) * DH + sub * E;
    for (int c = grp; c < count; c += G) {
      const float ga = gam[c], be = bet[c];
      const int t = tok[c];
      float kv[E];
      load16(kb + (int64_t)t * rs, kv);
#pragma unroll
      for (int e = 0; e < E; e++) dqa[e] = fmaf(ga, kv[e], dqa[e]);
      float xk[E], xv[E];
      const float gs = ga * g.scale;
#pragma unroll
      for (int e = 0; e < E; e++) {
        xk[e] = gs * qv[e];
        xv[e] = be * gv[e];
      }
      const int64_t ar = (int64_t)t * acc_heads * DH + acc_h;
#pragma unroll
      for (int e = 0; e < E; e += 4) {
        red_add16(acc_k + ar + e, xk + e);
        red_add16(acc_v + ar + e, xv + e);
      }
    }
#pragma unroll
    for (int w = L; w < 32; w <<= 1)
#pragma unroll
      for (int e = 0; e < E; e++) dqa[e] += __shfl_xor_sync(kFull, dqa[e], w);
    if (grp == 0) {
#pragma unroll
      for (int e = 0; e < E; e++) dqa[e] *= g.scale;
      store16(dq + row, dqa);
    }
    __syncwarp();
  }
}

__global__ void dsa3d_zero_kernel(uint4* __restrict__ p, const int64_t n16) {
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n16;
       i += (int64_t)gridDim.x * blockDim.x)
    p[i] = make_uint4(0u, 0u, 0u, 0u);
}

// fp32 accumulators [N][hc][DH] -> I/O-type dk/dv [N][heads][DH] for heads [h0, h0 + hc).
template <typename T, int DH>
__global__ void dsa3d_bwd_finalize_kernel(const float* __restrict__ acc_k,
                                          const float* __restrict__ acc_v, T* __restrict__ dk,
                                          T* __restrict__ dv, const int heads, const int h0,
                                          const int hc, const int64_t N) {
  constexpr int E = Elems<T>::kPerLoad;
  const int64_t chunks = N * hc * (DH / E);
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < chunks;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t src = i * E;
    const int64_t row = src / DH, col = src % DH;
    const int64_t n = row / hc;
    const int hh = (int)(row % hc);
    const int64_t dst = (n * heads + h0 + hh) * DH + col;
    float xk[E], xv[E];
#pragma unroll
    for (int e = 0; e < E; e += 4) {
      const float4 a = *reinterpret_cast<const float4*>(acc_k + src + e);
      const float4 b = *reinterpret_cast<const float4*>(acc_v + src + e);
      xk[e] = a.x; xk[e + 1] = a.y; xk[e + 2] = a.z; xk[e + 3] = a.w;
      xv[e] = b.x; xv[e + 1] = b.y; xv[e + 2] = b.z; xv[e + 3] = b.w;
    }
    store16(dk + dst, xk);
    store16(dv + dst, xv);
  }
}

}  // namespace dsa3d
