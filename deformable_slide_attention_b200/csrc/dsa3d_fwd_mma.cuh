// dsa3d_fwd_mma.cuh -- 3D-DSA forward on tensor cores (bf16 I/O, dh 64 or 128, k_w <= 15).
//
// Input: queries sorted by box origin (dsa3d_sort.cuh).  One warp takes one bucket row (all
// queries sharing the origin's t and y) and cuts it into chunks of at most 16 queries whose
// x-origins span at most 16.  For a chunk, box row (bt, by) of every query lies in key row
// (o_t + bt, o_y + by) inside the 32-key segment [X0, X0 + 32), X0 = the chunk's smallest
// x-origin.  Per tap plane u and box row by:
//   S_t  = (1-f_t) * Q.K[u, by]^T + f_t * Q.K[u+1, by]^T        (m16n8k16 MMAs, fp32 blend)
//   taps of row ty = by-1:  s = x-lerp(y-lerp(S_t[by-1], S_t[by]))  masked per query
//   online softmax (base 2) over the taps, P = exp2(s - m)
//   value weights of box row ty: beta = y-mix of the x-transposed P of tap rows ty and ty-1
//   O += [(1-f_t) beta | f_t beta] . [V[u, ty]; V[u+1, ty]]     (MMAs, beta as bf16 A operand)
// The MMA accumulator layout of S is the A-operand layout of P.V (lanes hold rows g and g+8,
// column pairs), so the whole per-query epilogue stays in registers; x-neighbours come from the
// neighbouring lane of the quad.  Only rows of valid queries exist here (the sort drops the rest).
//
// Operand layouts.  S = Q.K^T contracts dh: in k-step s, lane quad position q supplies the dims
// of its slice [q*DH/4, (q+1)*DH/4) at words 2s and 2s+1, for the Q rows (A) and the key rows
// (B) alike, so every lane reads contiguous 16-byte chunks.  O = P.V maps output column n of
// n-tile j to dim n*NT + j, so lane g reads the contiguous dims [g*NT, (g+1)*NT) of each value
// row and lane (g, q) ends up owning the contiguous output dims [2q*NT, 2q*NT + 2*NT).
#pragma once

#include "dsa3d_common.cuh"
#include "dsa3d_sort.cuh"

namespace dsa3d {

__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], unsigned a0, unsigned a1, unsigned a2,
                                               unsigned a3, unsigned b0, unsigned b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ unsigned pack_bf16(float lo, float hi) {
  const __nv_bfloat162 b = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const unsigned*>(&b);
}

__device__ __forceinline__ uint4 ldg16(const void* p) { return __ldg(reinterpret_cast<const uint4*>(p)); }

// Per-row state of a chunk (rows g and g+8 of the lane).
struct MmaRow {
  bool live;        // row holds a query
  int n;            // token
  int ox;           // x-origin minus X0, in [0, 16)
  float f[3];
  int lo[3], hi[3];
};

template <int DH>
struct MmaShape {
  static constexpr int KS = DH / 16;   // k-steps of Q.K^T
  static constexpr int QW = DH / 8;    // 32-bit words in a lane's dim slice of a Q/K row
  static constexpr int NT = DH / 8;    // n-tiles of O
  static constexpr int VW = NT / 2;    // 32-bit words in a lane's dim slice of a V row
};

// x-neighbour helpers over the 4 n-tiles of one row-half (values v[jt][e], e = 0 even, 1 odd col).
// next[c] = v[c + 1]; prev[c] = v[c - 1] (0 outside the segment).
__device__ __forceinline__ void col_next(const float (&ev)[4], const float (&od)[4], int q, int lane,
                                         float (&nx_ev)[4], float (&nx_od)[4]) {
  const int src = (lane & ~3) | ((q + 1) & 3);
#pragma unroll
  for (int jt = 0; jt < 4; jt++) {
    const float send = (q == 0) ? ((jt + 1 < 4) ? ev[jt + 1] : 0.f) : ev[jt];
    const float r = __shfl_sync(kFull, send, src);
    nx_ev[jt] = od[jt];  // col 2q -> 2q+1 in the same lane
    nx_od[jt] = r;       // col 2q+1 -> 2q+2 (lane q+1, or next n-tile's q = 0)
  }
}
__device__ __forceinline__ void col_prev(const float (&ev)[4], const float (&od)[4], int q, int lane,
                                         float (&pv_ev)[4], float (&pv_od)[4]) {
  const int src = (lane & ~3) | ((q + 3) & 3);
#pragma unroll
  for (int jt = 0; jt < 4; jt++) {
    // receiver q = 0 wants lane 3's odd value of n-tile jt-1; receivers q > 0 want lane q-1's of jt
    const float send = (q == 3) ? ((jt > 0) ? od[jt - 1] : 0.f) : od[jt];
    pv_ev[jt] = __shfl_sync(kFull, send, src);
    pv_od[jt] = ev[jt];  // col 2q+1 -> 2q in the same lane
  }
}

// O += [(1-f_t) beta | f_t beta] . [V[t0, y, seg]; V[t0+1, y, seg]] for the 32-key segment at X0.
// beta is in accumulator layout (n-tile jt: row g cols 8jt+2q, 8jt+2q+1 in [0],[1]; row g+8 in
// [2],[3]), which is the A-operand layout of k-step kk = n-tiles 2kk, 2kk+1.
template <int DH>
__device__ __forceinline__ void dsa3d_pv_rows(float (&o)[MmaShape<DH>::NT][4], const float (&beta)[4][4],
                                              const float (&ft)[2], int t0, int y, int X0, int segw,
                                              const __nv_bfloat16* vh, int64_t rs, const Geo& g,
                                              int gq, int qq) {
  using S = MmaShape<DH>;
  if (y < 0 || y >= g.Hp) return;
#pragma unroll
  for (int pl = 0; pl < 2; pl++) {
    const int t = t0 + pl;
    if (t < 0 || t >= g.F) continue;
    const float w0 = pl ? ft[0] : 1.f - ft[0], w1 = pl ? ft[1] : 1.f - ft[1];
#pragma unroll
    for (int kk = 0; kk < 2; kk++) {
      const unsigned a0 = pack_bf16(w0 * beta[2 * kk][0], w0 * beta[2 * kk][1]);
      const unsigned a1 = pack_bf16(w1 * beta[2 * kk][2], w1 * beta[2 * kk][3]);
      const unsigned a2 = pack_bf16(w0 * beta[2 * kk + 1][0], w0 * beta[2 * kk + 1][1]);
      const unsigned a3 = pack_bf16(w1 * beta[2 * kk + 1][2], w1 * beta[2 * kk + 1][3]);
      unsigned vw[4][S::VW];
#pragma unroll
      for (int i = 0; i < 4; i++) {
        const int key = 16 * kk + 2 * qq + (i & 1) + 8 * (i >> 1);
        const int x = X0 + key;
        const bool ok = key < segw && x >= 0 && x < g.Wp;
        const __nv_bfloat16* vr = vh + ((int64_t)(t * g.Hp + y) * g.Wp + max(x, 0)) * rs + gq * S::NT;
#pragma unroll
        for (int c = 0; c < S::VW / 4; c++) {
          const uint4 a = ok ? ldg16(vr + c * 8) : make_uint4(0, 0, 0, 0);
          vw[i][4 * c] = a.x; vw[i][4 * c + 1] = a.y; vw[i][4 * c + 2] = a.z; vw[i][4 * c + 3] = a.w;
        }
      }
#pragma unroll
      for (int j = 0; j < S::NT; j++) {
        const unsigned sel = (j & 1) ? 0x7632u : 0x5410u;
        const unsigned b0 = __byte_perm(vw[0][j >> 1], vw[1][j >> 1], sel);
        const unsigned b1 = __byte_perm(vw[2][j >> 1], vw[3][j >> 1], sel);
        mma_bf16_16816(o[j], a0, a1, a2, a3, b0, b1);
      }
    }
  }
}

template <int DH>
__global__ void __launch_bounds__(128, DSA3D_MMA_MINB)
    dsa3d_fwd_mma_kernel(const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k,
                         const __nv_bfloat16* __restrict__ v, const float* __restrict__ off,
                         __nv_bfloat16* __restrict__ out, float* __restrict__ lse,
                         const int* __restrict__ start, const int* __restrict__ sorted_n,
                         const int* __restrict__ sorted_ex, const Geo g, const SortGeo sg,
                         const int h0, const int hg) {
  using S = MmaShape<DH>;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int gq = lane >> 2, qq = lane & 3;  // fragment row group / quad position
  const int64_t rs = (int64_t)g.heads * DH;
  const float sc = g.scale * kLog2e;
  const int segw = 16 + g.kw;  // keys of the segment that can carry weight
  const int64_t rows = (int64_t)hg * sg.Et * sg.Ey;

  for (int64_t row = (int64_t)blockIdx.x * 4 + warp; row < rows; row += (int64_t)gridDim.x * 4) {
    const int hh = (int)(row / ((int64_t)sg.Et * sg.Ey));
    const int rem = (int)(row - (int64_t)hh * sg.Et * sg.Ey);
    const int et = rem / sg.Ey, ey = rem % sg.Ey;
    const int h = h0 + hh;
    const int64_t b0 = (int64_t)hh * sg.E1 + ((int64_t)et * sg.Ey + ey) * sg.Ex;
    const int qbeg = start[b0], qend = start[b0 + sg.Ex];
    const int ot = et - g.kt, oy = ey - g.kh;
    const __nv_bfloat16* kh_ = k + (int64_t)h * DH;
    const __nv_bfloat16* vh_ = v + (int64_t)h * DH;

    for (int pos = qbeg; pos < qend;) {
      // ---- chunk: <= 16 consecutive queries whose x-origins span <= 16
      const int ex_l = (lane < 16 && pos + lane < qend) ? sorted_ex[pos + lane] : 0x7fffffff;
      const int ex0 = __shfl_sync(kFull, ex_l, 0);
      const unsigned bal = __ballot_sync(kFull, lane < 16 && pos + lane < qend && ex_l - ex0 < 16);
      const int cnt = __popc(bal);
      const int X0 = ex0 - g.kw;

      MmaRow R[2];
#pragma unroll
      for (int hf = 0; hf < 2; hf++) {
        const int r = gq + 8 * hf;
        R[hf].live = r < cnt;
        R[hf].n = R[hf].live ? sorted_n[pos + r] : 0;
        const Query Qd = decode_query(g, off, h, R[hf].n);
        R[hf].ox = Qd.o[2] - X0;
#pragma unroll
        for (int a = 0; a < 3; a++) {
          R[hf].f[a] = Qd.f[a];
          R[hf].lo[a] = Qd.lo[a];
          R[hf].hi[a] = R[hf].live ? Qd.hi[a] : -1;  // dead rows: no valid tap
        }
        DSA3D_DEVICE_CHECK(!R[hf].live || (Qd.ok && Qd.o[0] == ot && Qd.o[1] == oy && R[hf].ox >= 0 && R[hf].ox < 16));
      }

      // ---- Q fragments
      unsigned qa[S::KS][4];
      {
        unsigned w0[S::QW], w1[S::QW];
#pragma unroll
        for (int c = 0; c < S::QW / 4; c++) {
          uint4 a = make_uint4(0, 0, 0, 0), b = make_uint4(0, 0, 0, 0);
          if (R[0].live) a = ldg16(q + ((int64_t)R[0].n * g.heads + h) * DH + qq * (DH / 4) + c * 8);
          if (R[1].live) b = ldg16(q + ((int64_t)R[1].n * g.heads + h) * DH + qq * (DH / 4) + c * 8);
          w0[4 * c] = a.x; w0[4 * c + 1] = a.y; w0[4 * c + 2] = a.z; w0[4 * c + 3] = a.w;
          w1[4 * c] = b.x; w1[4 * c + 1] = b.y; w1[4 * c + 2] = b.z; w1[4 * c + 3] = b.w;
        }
#pragma unroll
        for (int s = 0; s < S::KS; s++) {
          qa[s][0] = w0[2 * s];
          qa[s][1] = w1[2 * s];
          qa[s][2] = w0[2 * s + 1];
          qa[s][3] = w1[2 * s + 1];
        }
      }

      float o[S::NT][4];
#pragma unroll
      for (int j = 0; j < S::NT; j++) o[j][0] = o[j][1] = o[j][2] = o[j][3] = 0.f;
      float m[2] = {-INFINITY, -INFINITY}, l[2] = {0.f, 0.f};

      for (int u = 0; u < g.kt; u++) {
        const bool plane_live = (R[0].lo[0] <= u && u <= R[0].hi[0]) || (R[1].lo[0] <= u && u <= R[1].hi[0]);
        if (!__any_sync(kFull, plane_live)) continue;
        const float ft[2] = {R[0].f[0], R[1].f[0]};
        float st_prev[4][4];
        float bx_prev[4][4];
#pragma unroll
        for (int jt = 0; jt < 4; jt++)
#pragma unroll
          for (int e = 0; e < 4; e++) st_prev[jt][e] = bx_prev[jt][e] = 0.f;

        for (int by = 0; by <= g.kh; by++) {
          // --- t-blended raw scores of box row by
          float st[4][4];
#pragma unroll
          for (int jt = 0; jt < 4; jt++) st[jt][0] = st[jt][1] = st[jt][2] = st[jt][3] = 0.f;
          const int y = oy + by;
#pragma unroll
          for (int pl = 0; pl < 2; pl++) {
            const int t = ot + u + pl;
            if (t < 0 || t >= g.F || y < 0 || y >= g.Hp) continue;
            float acc[4][4];
#pragma unroll
            for (int jt = 0; jt < 4; jt++) {
              acc[jt][0] = acc[jt][1] = acc[jt][2] = acc[jt][3] = 0.f;
              const int col = 8 * jt + gq;
              const int x = X0 + col;
              unsigned kw_[S::QW];
              const bool ok = col < segw && x >= 0 && x < g.Wp;
              const __nv_bfloat16* kr = kh_ + ((int64_t)(t * g.Hp + y) * g.Wp + max(x, 0)) * rs + qq * (DH / 4);
#pragma unroll
              for (int c = 0; c < S::QW / 4; c++) {
                const uint4 a = ok ? ldg16(kr + c * 8) : make_uint4(0, 0, 0, 0);
                kw_[4 * c] = a.x; kw_[4 * c + 1] = a.y; kw_[4 * c + 2] = a.z; kw_[4 * c + 3] = a.w;
              }
#pragma unroll
              for (int s = 0; s < S::KS; s++)
                mma_bf16_16816(acc[jt], qa[s][0], qa[s][1], qa[s][2], qa[s][3], kw_[2 * s], kw_[2 * s + 1]);
            }
#pragma unroll
            for (int jt = 0; jt < 4; jt++) {
              const float w0 = pl ? ft[0] : 1.f - ft[0], w1 = pl ? ft[1] : 1.f - ft[1];
              st[jt][0] = fmaf(w0, acc[jt][0], st[jt][0]);
              st[jt][1] = fmaf(w0, acc[jt][1], st[jt][1]);
              st[jt][2] = fmaf(w1, acc[jt][2], st[jt][2]);
              st[jt][3] = fmaf(w1, acc[jt][3], st[jt][3]);
            }
          }

          if (by >= 1) {
            const int ty = by - 1;
            // --- tap scores of tap row ty: y-lerp then x-lerp
            float sy_e[2][4], sy_o[2][4];
#pragma unroll
            for (int hf = 0; hf < 2; hf++) {
              const float fy = R[hf].f[1];
#pragma unroll
              for (int jt = 0; jt < 4; jt++) {
                sy_e[hf][jt] = fmaf(fy, st[jt][2 * hf] - st_prev[jt][2 * hf], st_prev[jt][2 * hf]);
                sy_o[hf][jt] = fmaf(fy, st[jt][2 * hf + 1] - st_prev[jt][2 * hf + 1], st_prev[jt][2 * hf + 1]);
              }
            }
            float p_e[2][4], p_o[2][4];
            float alpha[2];
#pragma unroll
            for (int hf = 0; hf < 2; hf++) {
              float nx_e[4], nx_o[4];
              col_next(sy_e[hf], sy_o[hf], qq, lane, nx_e, nx_o);
              const float fx = R[hf].f[2];
              const bool row_ok = R[hf].lo[0] <= u && u <= R[hf].hi[0] && R[hf].lo[1] <= ty && ty <= R[hf].hi[1];
              float mx = -INFINITY;
#pragma unroll
              for (int jt = 0; jt < 4; jt++) {
                const int wx0 = 8 * jt + 2 * qq - R[hf].ox;
                const bool v0 = row_ok && wx0 >= R[hf].lo[2] && wx0 <= R[hf].hi[2];
                const bool v1 = row_ok && wx0 + 1 >= R[hf].lo[2] && wx0 + 1 <= R[hf].hi[2];
                const float s0 = fmaf(fx, nx_e[jt] - sy_e[hf][jt], sy_e[hf][jt]) * sc;
                const float s1 = fmaf(fx, nx_o[jt] - sy_o[hf][jt], sy_o[hf][jt]) * sc;
                p_e[hf][jt] = v0 ? s0 : -INFINITY;
                p_o[hf][jt] = v1 ? s1 : -INFINITY;
                mx = fmaxf(mx, fmaxf(p_e[hf][jt], p_o[hf][jt]));
              }
              mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 1));
              mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 2));
              alpha[hf] = 1.f;
              if (mx != -INFINITY) {
                const float mn = fmaxf(m[hf], mx);
                alpha[hf] = exp2f(m[hf] - mn);  // 0 when m was -inf
                m[hf] = mn;
              }
              float ls = 0.f;
#pragma unroll
              for (int jt = 0; jt < 4; jt++) {
                p_e[hf][jt] = (p_e[hf][jt] == -INFINITY) ? 0.f : exp2f(p_e[hf][jt] - m[hf]);
                p_o[hf][jt] = (p_o[hf][jt] == -INFINITY) ? 0.f : exp2f(p_o[hf][jt] - m[hf]);
                ls += p_e[hf][jt] + p_o[hf][jt];
              }
              l[hf] = fmaf(l[hf], alpha[hf], ls);
            }
            if (__any_sync(kFull, alpha[0] != 1.f || alpha[1] != 1.f)) {
#pragma unroll
              for (int j = 0; j < S::NT; j++) {
                o[j][0] *= alpha[0]; o[j][1] *= alpha[0];
                o[j][2] *= alpha[1]; o[j][3] *= alpha[1];
              }
#pragma unroll
              for (int jt = 0; jt < 4; jt++) {
                bx_prev[jt][0] *= alpha[0]; bx_prev[jt][1] *= alpha[0];
                bx_prev[jt][2] *= alpha[1]; bx_prev[jt][3] *= alpha[1];
              }
            }
            // --- value weights: x-transpose of P (this tap row), y-mix with the previous one
            float beta[4][4];
#pragma unroll
            for (int hf = 0; hf < 2; hf++) {
              float pv_e[4], pv_o[4];
              col_prev(p_e[hf], p_o[hf], qq, lane, pv_e, pv_o);
              const float fx = R[hf].f[2], fy = R[hf].f[1];
#pragma unroll
              for (int jt = 0; jt < 4; jt++) {
                const float bxe = fmaf(fx, pv_e[jt] - p_e[hf][jt], p_e[hf][jt]);
                const float bxo = fmaf(fx, pv_o[jt] - p_o[hf][jt], p_o[hf][jt]);
                beta[jt][2 * hf] = fmaf(fy, bx_prev[jt][2 * hf] - bxe, bxe);
                beta[jt][2 * hf + 1] = fmaf(fy, bx_prev[jt][2 * hf + 1] - bxo, bxo);
                bx_prev[jt][2 * hf] = bxe;
                bx_prev[jt][2 * hf + 1] = bxo;
              }
            }
            // --- O += beta . V over box row ty of planes u, u+1
            dsa3d_pv_rows<DH>(o, beta, ft, ot + u, oy + ty, X0, segw, vh_, rs, g, gq, qq);
          }
#pragma unroll
          for (int jt = 0; jt < 4; jt++)
#pragma unroll
            for (int e = 0; e < 4; e++) st_prev[jt][e] = st[jt][e];
        }
        // box row kh takes only the y-carry of tap row kh-1
        {
          float beta[4][4];
#pragma unroll
          for (int jt = 0; jt < 4; jt++) {
            beta[jt][0] = R[0].f[1] * bx_prev[jt][0];
            beta[jt][1] = R[0].f[1] * bx_prev[jt][1];
            beta[jt][2] = R[1].f[1] * bx_prev[jt][2];
            beta[jt][3] = R[1].f[1] * bx_prev[jt][3];
          }
          dsa3d_pv_rows<DH>(o, beta, ft, ot + u, oy + g.kh, X0, segw, vh_, rs, g, gq, qq);
        }
      }

      // ---- normalise and store
#pragma unroll
      for (int hf = 0; hf < 2; hf++) {
        float lt = l[hf];
        lt += __shfl_xor_sync(kFull, lt, 1);
        lt += __shfl_xor_sync(kFull, lt, 2);
        if (!R[hf].live) continue;
        const float inv = 1.f / lt;
        __nv_bfloat16* orow = out + ((int64_t)R[hf].n * g.heads + h) * DH + qq * (DH / 4);
        float vals[S::NT * 2];
#pragma unroll
        for (int j = 0; j < S::NT; j++) {
          vals[j] = o[j][2 * hf] * inv;
          vals[S::NT + j] = o[j][2 * hf + 1] * inv;
        }
#pragma unroll
        for (int c = 0; c < S::NT * 2 / 8; c++) store16(orow + c * 8, vals + c * 8);
        if (qq == 0 && lse) lse[(int64_t)h * g.N + R[hf].n] = (m[hf] + log2f(lt)) * kLn2;
      }
      pos += cnt;
    }
  }
}

}  // namespace dsa3d
