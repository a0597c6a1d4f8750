// dsa3d_taps.cuh -- 3D-DSA with per-tap offsets on CUDA cores (MegaSlide-DiT, arXiv 2607.22696,
// the 3D-DSA definition, Eq. 1: the offset tensor carries one 3-vector per window tap).
//
// Tap tau of query p samples K and V at p + tau + delta_tau, each tap with its own integer and
// fractional part.  The taps of a query therefore do not share one integer box (the factorised
// form of the per-token kernels does not apply): every tap reads its own 8 trilinear corners.
//
// Offsets and their gradient are [heads][N][K][3] fp32, taps in (u, v, w) order with u (time)
// outermost.  Each tap's components are decoded like a per-token offset (decode_delta); an
// invalid component masks that tap only.  A tap is valid iff its sample position lies in the
// closed box [0, dim - 1] on every axis.
//
// One warp computes one (head, query) at a time, persistent over a head-major item order.  Taps
// are taken 32 at a time (a "block"): lane i decodes tap i of the block into shared memory, then
// each lane group of L = dh/E lanes (E elements per 16-byte chunk) works on whole taps or whole
// (tap, corner) pairs, reading each corner row as one coalesced access; partial dots are reduced
// across the group with a transpose-sum (L items per L - 1 shuffles).
#pragma once

#include "dsa3d_bwd.cuh"

// Consecutive (head, query) items a warp takes at a time (neighbouring queries read overlapping
// corner rows, so a run of them reuses the rows in L1), and warps per CTA of the forward.
#ifndef DSA3D_TAPS_RUN
#define DSA3D_TAPS_RUN 4
#endif
#ifndef DSA3D_TAPS_FWD_WARPS
#define DSA3D_TAPS_FWD_WARPS 4
#endif

namespace dsa3d {

constexpr int kTapsRun = DSA3D_TAPS_RUN;
constexpr int kTapsFwdWarps = DSA3D_TAPS_FWD_WARPS;

// The items of a persistent warp: runs of kTapsRun consecutive items, run r = the warp's global
// index + i * (all warps).  next() advances; valid while item < n_items.
struct ItemWalk {
  int64_t item, run_end, stride;
  __device__ ItemWalk(int64_t warp_global, int64_t warps_total, int64_t n_items) {
    item = warp_global * kTapsRun;
    run_end = item + kTapsRun;
    stride = warps_total * kTapsRun;
    (void)n_items;
  }
  __device__ void next() {
    if (++item == run_end) {
      item += stride - kTapsRun;
      run_end = item + kTapsRun;
    }
  }
};

// One decoded tap: base token of its trilinear cell (-1 if the tap is masked or beyond the
// block's end) and the fractional parts, as an int4 {tok, f_t, f_y, f_x}; and two corner masks
// (corner c = (ct << 2) | (cy << 1) | cx): corners with a nonzero weight (bits 0-7) and corners
// inside the volume (bits 8-15), both empty for a masked tap.  For a valid tap every corner of
// nonzero weight lies inside the volume (the tap's cell is inside it on every axis whose fraction
// is nonzero), so base + corner_off(c) is a valid token for every set bit.
struct TapCell {
  int4 m;
  int masks;
};

__device__ __forceinline__ TapCell decode_tap(const Geo& g, const float* __restrict__ o, const int p[3],
                                              int tau) {
  const int uvw[3] = {tau / (g.kw * g.kh), (tau / g.kw) % g.kh, tau % g.kw};
  bool ok = true;
  int wm = 0xff, vm = 0xff;
  int b[3];
  float f[3];
#pragma unroll
  for (int a = 0; a < 3; a++) {
    int ii;
    if (!decode_delta(__ldg(o + a), ii, f[a])) ok = false;
    const int k = win_of(g, a), D = dim_of(g, a);
    const long long ba = (long long)p[a] + uvw[a] - (k - 1) / 2 + ii;
    if (ba < 0 || ba > D - 1 || (ba == D - 1 && f[a] != 0.f)) ok = false;
    b[a] = (int)ba;
    const int lower = (a == 0) ? 0x0f : (a == 1 ? 0x33 : 0x55);  // corners with c_a = 0
    if (f[a] == 0.f) wm &= lower;
    if (ba >= D - 1) vm &= lower;
  }
  TapCell c;
  c.m = make_int4(ok ? (b[0] * g.HW + b[1] * g.Wp + b[2]) : -1, __float_as_int(f[0]),
                  __float_as_int(f[1]), __float_as_int(f[2]));
  c.masks = ok ? (wm | (vm << 8)) : 0;  // a masked tap reads no corner (kernels rely on this)
  return c;
}

// Token offset of corner c from its cell's base token.
__device__ __forceinline__ int corner_off(const Geo& g, int c) {
  return ((c >> 2) & 1) * g.HW + ((c >> 1) & 1) * g.Wp + (c & 1);
}

__device__ __forceinline__ void tap_fracs(const int4& m, float f[3]) {
  f[0] = __int_as_float(m.y);
  f[1] = __int_as_float(m.z);
  f[2] = __int_as_float(m.w);
}

// acc[e] += w * x[e] for e < E, as packed pairs (fma.rn.f32x2: half the FMA issue slots of the
// forward, which is bound by instruction issue).
template <int E>
__device__ __forceinline__ void axpy_pairs(float w, const float* x, float* acc) {
  const float2 w2 = make_float2(w, w);
#pragma unroll
  for (int e = 0; e < E; e += 2) {
    const float2 r = __ffma2_rn(w2, make_float2(x[e], x[e + 1]), make_float2(acc[e], acc[e + 1]));
    acc[e] = r.x;
    acc[e + 1] = r.y;
  }
}

// Decode taps [c0, c0 + 32) of query (h, n) at p into the warp's block arrays.
__device__ __forceinline__ void decode_block(const Geo& g, const float* __restrict__ offq,
                                             const int p[3], int c0, int lane, int4* meta,
                                             int* masks) {
  __syncwarp();
  const int tau = c0 + lane;
  TapCell c;
  c.m = make_int4(-1, 0, 0, 0);
  c.masks = 0;
  if (tau < g.K) c = decode_tap(g, offq + (int64_t)tau * 3, p, tau);
  meta[lane] = c.m;
  masks[lane] = c.masks;
  __syncwarp();
}

// --- forward ------------------------------------------------------------------------------------
//   per block: 1. decode; 2. scores: lane group grp forms, for taps j = it*G + grp (it < L), the
//   chunk of k~_j = sum_c w_c K[base_j + c] over the nonzero-weight corners and its dot with the
//   q chunk; after the transpose-sum lane grp*L + sub holds the score of tap sub*G + grp;
//   3. online softmax update (running max m and sum l in base 2, accumulator rescaled);
//   4. values: the same lane groups add p_j * v~_j for their taps (p_j fetched by shuffle).
template <typename T, int DH, int WARPS>
__global__ void __launch_bounds__(WARPS * 32)
    dsa3d_fwd_taps_kernel(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
                          const float* __restrict__ off, T* __restrict__ out, float* __restrict__ lse,
                          const Geo g, const int64_t n_items) {
  constexpr int E = Elems<T>::kPerLoad;
  constexpr int L = DH / E;
  constexpr int G = 32 / L;
  __shared__ int4 meta_s[WARPS][32];
  __shared__ int masks_s[WARPS][32];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int4* meta = meta_s[warp];
  int* masks = masks_s[warp];
  const int grp = lane / L, sub = lane % L;
  const int64_t rs = (int64_t)g.heads * DH;
  const float sc = g.scale * kLog2e;

  for (ItemWalk wk((int64_t)blockIdx.x * WARPS + warp, (int64_t)gridDim.x * WARPS, n_items);
       wk.item < n_items; wk.next()) {
    const int64_t item = wk.item;
    const int h = (int)(item / g.N);
    const int64_t n = item - (int64_t)h * g.N;
    const int p[3] = {(int)(n / g.HW), (int)((n / g.Wp) % g.Hp), (int)(n % g.Wp)};
    const float* offq = off + ((int64_t)h * g.N + n) * g.K * 3;
    const T* kb = k + (int64_t)h * DH + sub * E;
    const T* vb = v + (int64_t)h * DH + sub * E;
    float qv[E], acc[E];
    load16(q + (n * g.heads + h) * DH + sub * E, qv);
#pragma unroll
    for (int e = 0; e < E; e++) acc[e] = 0.f;
    float m = -INFINITY, l = 0.f;

    for (int c0 = 0; c0 < g.K; c0 += 32) {
      decode_block(g, offq, p, c0, lane, meta, masks);
      float s_raw = 0.f;
#pragma unroll 2
      for (int it = 0; it < L; it++) {
        // branch-free, so that the loads of two taps are in flight together: a masked tap reads
        // the query's own row (its score is replaced by -inf below), a corner of zero weight
        // reads the cell's base row (adding 0 times a finite value)
        const int j = it * G + grp;
        const int4 md = meta[j];
        const int wm = masks[j];
        const int base = md.x >= 0 ? md.x : (int)n;
        float f[3], w8[8], kt[E];
        tap_fracs(md, f);
        corner_weights(f, w8);
#pragma unroll
        for (int e = 0; e < E; e++) kt[e] = 0.f;
#pragma unroll
        for (int c = 0; c < 8; c++) {
          float kv[E];
          load16(kb + (int64_t)(base + ((wm >> c) & 1 ? corner_off(g, c) : 0)) * rs, kv);
          axpy_pairs<E>(w8[c], kv, kt);
        }
        float a = 0.f;
#pragma unroll
        for (int e = 0; e < E; e++) a = fmaf(qv[e], kt[e], a);
#pragma unroll
        for (int w = 1; w < L; w <<= 1) a += __shfl_xor_sync(kFull, a, w);  // over the group
        if (sub == it) s_raw = a;
      }
      const bool valid = meta[sub * G + grp].x >= 0;
      const float s = valid ? s_raw * sc : -INFINITY;
      const float mn = fmaxf(m, warp_max(s));
      if (mn == -INFINITY) continue;  // no valid tap yet (warp-uniform)
      const float alpha = exp2f(m - mn);
      const float pr = valid ? exp2f(s - mn) : 0.f;
      l = fmaf(l, alpha, warp_sum(pr));
      m = mn;
#pragma unroll
      for (int e = 0; e < E; e++) acc[e] *= alpha;
#pragma unroll 2
      for (int it = 0; it < L; it++) {
        // branch-free as above: a masked tap has p = 0 and reads the query's own row
        const int j = it * G + grp;
        const float pj = __shfl_sync(kFull, pr, grp * L + it);
        const int4 md = meta[j];
        const int wm = masks[j];
        const int base = md.x >= 0 ? md.x : (int)n;
        float f[3], w8[8];
        tap_fracs(md, f);
        corner_weights(f, w8);
#pragma unroll
        for (int c = 0; c < 8; c++) {
          float vv[E];
          load16(vb + (int64_t)(base + ((wm >> c) & 1 ? corner_off(g, c) : 0)) * rs, vv);
          axpy_pairs<E>(pj * w8[c], vv, acc);
        }
      }
    }
#pragma unroll
    for (int w = L; w < 32; w <<= 1)
#pragma unroll
      for (int e = 0; e < E; e++) acc[e] += __shfl_xor_sync(kFull, acc[e], w);
    const float inv_l = (l > 0.f) ? 1.f / l : 0.f;
    if (grp == 0) {
#pragma unroll
      for (int e = 0; e < E; e++) acc[e] *= inv_l;
      store16(out + (n * g.heads + h) * DH + sub * E, acc);
    }
    if (lane == 0 && lse) lse[(int64_t)h * g.N + n] = (l > 0.f) ? (m + log2f(l)) * kLn2 : -INFINITY;
  }
}

// --- backward -----------------------------------------------------------------------------------
// Exact derivative of the forward above with the masks and integer parts held fixed.  Per
// (head, query), with P = exp(s - lse), dP_tau = dO . v~_tau, D = sum_tau P dP and
// dS = P (dP - D):
//   dq               = scale * sum_tau dS_tau k~_tau
//   dK[base + c]    += scale * dS_tau * w_c * q,    dV[base + c] += P_tau * w_c * dO
//   doff_tau,a       = scale dS_tau q . dk~_tau/df_a + P_tau dO . dv~_tau/df_a
// Pass 1 reads every tap's 8 K and 8 V corner rows once (corners inside the volume: a
// zero-weight corner still carries a weight derivative).  A lane group takes one tap at a time,
// forms the lane's partials of the 8 tap quantities s, dP, q . dk~/df_a, dO . dv~/df_a, reduces
// them over the group and accumulates what is linear in the not yet known D:
//   dq = scale (U - D W),  U = sum P dP k~,  W = sum P k~    (dh-vectors in registers)
//   doff = X - D Y,        X = scale P dP (q . dk~/df_a) + P (dO . dv~/df_a),  Y = scale P (q . dk~/df_a)
// X goes to doffsets; P, dP and Y stay in shared memory (20 bytes per tap per warp).  Pass 2, once
// D is known, decodes the taps again, finishes doff and scatters the dK/dV contributions (16-byte
// vector reductions into fp32 accumulators [N][heads in pass][dh], as in the per-token CUDA-core
// backward); it reads no K or V row.

// Element ownership of the backward.  fp32: lane sub of a row's lane group owns the 4
// contiguous elements [4 sub, 4 sub + 4), so one 16-byte reduction per lane covers a contiguous
// span.  bf16 (8 elements per lane): the lane owns [4 sub, 4 sub + 4) and [DH/2 + 4 sub, ...),
// read and written as two 8-byte halves, so that each of its two 16-byte fp32 reductions also
// covers, across the group, one contiguous 256-byte span (whole 32-byte sectors) instead of
// every other 16 bytes.
template <typename T, int DH>
struct ScatterRow;
template <int DH>
struct ScatterRow<float, DH> {
  __device__ static void load(const float* row, int sub, float* x) { load16(row + sub * 4, x); }
  __device__ static void store(float* row, int sub, const float* x) { store16(row + sub * 4, x); }
  __device__ static void red(float* row, int sub, const float* x) { red_add16(row + sub * 4, x); }
};
template <int DH>
struct ScatterRow<__nv_bfloat16, DH> {
  __device__ static void half(const __nv_bfloat16* p, float* x) {
    const uint2 v = __ldg(reinterpret_cast<const uint2*>(p));
    x[0] = __uint_as_float(v.x << 16);
    x[1] = __uint_as_float(v.x & 0xffff0000u);
    x[2] = __uint_as_float(v.y << 16);
    x[3] = __uint_as_float(v.y & 0xffff0000u);
  }
  __device__ static void load(const __nv_bfloat16* row, int sub, float* x) {
    half(row + sub * 4, x);
    half(row + DH / 2 + sub * 4, x + 4);
  }
  __device__ static void store(__nv_bfloat16* row, int sub, const float* x) {
#pragma unroll
    for (int hlf = 0; hlf < 2; hlf++) {
      const __nv_bfloat162 a = __floats2bfloat162_rn(x[4 * hlf], x[4 * hlf + 1]);
      const __nv_bfloat162 b = __floats2bfloat162_rn(x[4 * hlf + 2], x[4 * hlf + 3]);
      uint2 v;
      v.x = *reinterpret_cast<const unsigned*>(&a);
      v.y = *reinterpret_cast<const unsigned*>(&b);
      *reinterpret_cast<uint2*>(row + hlf * (DH / 2) + sub * 4) = v;
    }
  }
  __device__ static void red(float* row, int sub, const float* x) {
    red_add16(row + sub * 4, x);
    red_add16(row + DH / 2 + sub * 4, x + 4);
  }
};

// Sum the 8 tap partials v[] over the L lanes of each lane group.  L >= 8: butterfly down to 8
// lanes, then a transpose-sum, after which v[0] of lane sub holds quantity (sub & 7).  L = 4: a
// plain butterfly, after which every lane holds all 8 in v[].
template <int L>
__device__ __forceinline__ void reduce_tap8(float (&v)[8], int lane) {
  if constexpr (L >= 8) {
#pragma unroll
    for (int w = L / 2; w >= 8; w >>= 1)
#pragma unroll
      for (int i = 0; i < 8; i++) v[i] += __shfl_xor_sync(kFull, v[i], w);
    group_transpose_sum<8>(v, lane);
  } else {
#pragma unroll
    for (int w = L / 2; w >= 1; w >>= 1)
#pragma unroll
      for (int i = 0; i < 8; i++) v[i] += __shfl_xor_sync(kFull, v[i], w);
  }
}

__host__ __device__ inline int bwd_taps_warp_bytes(int K) { return (5 * K * 4 + 15) & ~15; }

template <typename T, int DH, int WARPS>
__global__ void __launch_bounds__(WARPS * 32)
    dsa3d_bwd_taps_kernel(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
                          const float* __restrict__ off, const float* __restrict__ lse,
                          const T* __restrict__ dout, T* __restrict__ dq, float* __restrict__ doff,
                          float* __restrict__ acc_k, float* __restrict__ acc_v, const int acc_heads,
                          const int h0, const Geo g, const int64_t n_items) {
  constexpr int E = Elems<T>::kPerLoad;
  constexpr int L = DH / E;
  constexpr int G = 32 / L;
  using SR = ScatterRow<T, DH>;
  __shared__ int4 meta_s[WARPS][32];
  __shared__ int masks_s[WARPS][32];
  extern __shared__ __align__(16) unsigned char smem[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int4* meta = meta_s[warp];
  int* masks = masks_s[warp];
  float* tP = reinterpret_cast<float*>(smem + warp * bwd_taps_warp_bytes(g.K));
  float* tdP = tP + g.K;
  float* tY = tdP + g.K;  // [3][K]
  const int grp = lane / L, sub = lane % L;
  // the group lane that holds tap quantity 2 + a (L >= 8) or all of them (L = 4) handles axis a
  const int ax = (L >= 8) ? sub - 2 : sub;
  const bool ax_lane = ax >= 0 && ax < 3;
  const int64_t rs = (int64_t)g.heads * DH;
  const float sc = g.scale * kLog2e;

  for (ItemWalk wk((int64_t)blockIdx.x * WARPS + warp, (int64_t)gridDim.x * WARPS, n_items);
       wk.item < n_items; wk.next()) {
    const int64_t item = wk.item;
    const int h = h0 + (int)(item / g.N);
    const int64_t n = item - (int64_t)(h - h0) * g.N;
    const int64_t row = (n * g.heads + h) * DH;  // start of the (token, head) row
    const int p[3] = {(int)(n / g.HW), (int)((n / g.Wp) % g.Hp), (int)(n % g.Wp)};
    const int64_t qo = ((int64_t)h * g.N + n) * g.K * 3;
    const float* offq = off + qo;
    float* doffq = doff + qo;
    const float lse_n = __ldg(lse + (int64_t)h * g.N + n);
    if (lse_n == -INFINITY) {  // no valid tap: zero gradients
      if (grp == 0) {
        float z[E];
#pragma unroll
        for (int e = 0; e < E; e++) z[e] = 0.f;
        SR::store(dq + row, sub, z);
      }
      for (int i = lane; i < 3 * g.K; i += 32) doffq[i] = 0.f;
      continue;
    }
    const float lse2 = lse_n * kLog2e;
    const T* kr = k + (int64_t)h * DH;
    const T* vr = v + (int64_t)h * DH;
    float qv[E], gv[E], U[E], W[E];
    SR::load(q + row, sub, qv);
    SR::load(dout + row, sub, gv);
#pragma unroll
    for (int e = 0; e < E; e++) U[e] = W[e] = 0.f;
    float Dg = 0.f;  // sum of P dP over this lane group's taps

    // pass 1
    for (int c0 = 0; c0 < g.K; c0 += 32) {
      decode_block(g, offq, p, c0, lane, meta, masks);
#pragma unroll 1
      for (int it = 0; it < L; it++) {
        // branch-free up to the stores (the reductions are warp-wide): a masked tap reads the
        // query's own row and counts zero; an out-of-volume corner reads the cell's base row
        const int j = it * G + grp;
        const int4 md = meta[j];
        const int mk = masks[j];
        const bool valid = md.x >= 0;
        const int base = valid ? md.x : (int)n;
        float f[3], w8[8], dw[3][8];
        tap_fracs(md, f);
        corner_weights(f, w8);
        corner_dweights(f, dw);
        float part[8], kt[E];
#pragma unroll
        for (int i = 0; i < 8; i++) part[i] = 0.f;
#pragma unroll
        for (int e = 0; e < E; e++) kt[e] = 0.f;
#pragma unroll
        for (int c = 0; c < 8; c++) {
          const bool in = (mk >> (8 + c)) & 1;
          const int64_t tr = (int64_t)(base + (in ? corner_off(g, c) : 0)) * rs;
          float kv[E], vv[E];
          SR::load(kr + tr, sub, kv);
          SR::load(vr + tr, sub, vv);
          float a = 0.f, b = 0.f;
#pragma unroll
          for (int e = 0; e < E; e++) {
            a = fmaf(qv[e], kv[e], a);
            b = fmaf(gv[e], vv[e], b);
            kt[e] = fmaf(w8[c], kv[e], kt[e]);  // zero weight outside the volume
          }
          a = in ? a : 0.f;
          b = in ? b : 0.f;
          part[0] = fmaf(w8[c], a, part[0]);
          part[1] = fmaf(w8[c], b, part[1]);
#pragma unroll
          for (int x = 0; x < 3; x++) {
            part[2 + x] = fmaf(dw[x][c], a, part[2 + x]);
            part[5 + x] = fmaf(dw[x][c], b, part[5 + x]);
          }
        }
        reduce_tap8<L>(part, lane);
        float s_raw, dPt, mine, other;
        if constexpr (L >= 8) {
          s_raw = __shfl_sync(kFull, part[0], grp * L);
          dPt = __shfl_sync(kFull, part[0], grp * L + 1);
          mine = part[0];
          other = __shfl_sync(kFull, part[0], (lane + 3) & 31);
        } else {
          s_raw = part[0];
          dPt = part[1];
          mine = (sub == 0) ? part[2] : (sub == 1 ? part[3] : part[4]);
          other = (sub == 0) ? part[5] : (sub == 1 ? part[6] : part[7]);
        }
        const float P = valid ? exp2f(fmaf(s_raw, sc, -lse2)) : 0.f;
        const float PdP = P * dPt;
        Dg += PdP;
#pragma unroll
        for (int e = 0; e < E; e++) {
          U[e] = fmaf(PdP, kt[e], U[e]);
          W[e] = fmaf(P, kt[e], W[e]);
        }
        const int tau = c0 + j;
        if (tau < g.K) {
          if (sub == 0) {
            tP[tau] = P;
            tdP[tau] = dPt;
          }
          if (ax_lane) {
            const float y = g.scale * P * mine;
            tY[ax * g.K + tau] = y;
            doffq[tau * 3 + ax] = fmaf(y, dPt, P * other);
          }
        }
      }
    }
    float D = Dg;
#pragma unroll
    for (int w = L; w < 32; w <<= 1) D += __shfl_xor_sync(kFull, D, w);  // over the groups
    __syncwarp();

    // dq = scale (U - D W), summed over the groups
#pragma unroll
    for (int e = 0; e < E; e++) {
      float x = fmaf(-D, W[e], U[e]);
#pragma unroll
      for (int w = L; w < 32; w <<= 1) x += __shfl_xor_sync(kFull, x, w);
      U[e] = x * g.scale;
    }
    if (grp == 0) SR::store(dq + row, sub, U);

    // pass 2: doff -= D Y (each lane rereads what it wrote), dK/dV scatter
    const int64_t acc_h = (int64_t)(h - h0) * DH;
    for (int c0 = 0; c0 < g.K; c0 += 32) {
      decode_block(g, offq, p, c0, lane, meta, masks);
#pragma unroll 1
      for (int it = 0; it < L; it++) {
        const int j = it * G + grp;
        const int tau = c0 + j;
        const int4 md = meta[j];
        if (md.x < 0) continue;  // masked, or beyond the last tap
        if (ax_lane) doffq[tau * 3 + ax] = fmaf(-D, tY[ax * g.K + tau], doffq[tau * 3 + ax]);
        const float P = tP[tau];
        if (P == 0.f) continue;
        const float dS = P * (tdP[tau] - D);
        float f[3], w8[8];
        tap_fracs(md, f);
        corner_weights(f, w8);
        const int wm = masks[j] & 0xff;
#pragma unroll
        for (int c = 0; c < 8; c++) {
          if ((wm >> c) & 1) {
            const float gs = g.scale * dS * w8[c], gb = P * w8[c];
            float xk[E], xv[E];
#pragma unroll
            for (int e = 0; e < E; e++) {
              xk[e] = gs * qv[e];
              xv[e] = gb * gv[e];
            }
            const int64_t ar = (int64_t)(md.x + corner_off(g, c)) * acc_heads * DH + acc_h;
            SR::red(acc_k + ar, sub, xk);
            SR::red(acc_v + ar, sub, xv);
          }
        }
      }
    }
    __syncwarp();
  }
}

}  // namespace dsa3d
