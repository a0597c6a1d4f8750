// dsa3d_bwd_mma.cuh -- 3D-DSA backward on tensor cores (bf16 I/O, dh 64 or 128, k_w <= 15).
//
// Exact derivative of the forward (MegaSlide-DiT, arXiv 2607.22696, Eq. 1) with the tap mask and
// the integer offset parts held fixed; D = sum_tau P_tau dP_tau (dout . out for the exact out).
// Queries are sorted by window origin and cut into the forward's chunks (<= 16 queries of one
// bucket row whose x-origins differ by <= chunk_span(kw), 32-key segment per box row).  Three
// passes, no global atomics:
//
//  1. query side (dsa3d_bwd_q_kernel, two warps per chunk): per tap plane u and box row, Q.K and
//     dO.V of box planes u and u+1 on tensor cores; per tap: P = exp2(s - lse2), dP, their
//     derivatives along the three fractional coordinates; per query D = sum P dP and
//        doff_a = scale (sum P dP ds_a - D sum P ds_a) + sum P dp_a.
//     It stores, per query and tap plane, the y/x-transposed splats of P (beta) and of P dP
//     (gamma') onto the box rows, in bf16: box[pos][u][by][bx], and D, f_t per query.
//  2. dq (dsa3d_bwd_dq_kernel): dq = scale sum_j gamma[j] K[j], gamma = gamma' - D beta and the
//     t-mix of the two tap planes feeding each box plane, as tensor-core products per box row
//     (K segments staged in shared memory by cp.async, one step ahead).
//  3. key side (dsa3d_bwd_kv_kernel): one warp owns 16 keys x dh/2 dims of one key row (a CTA
//     owns kKvRows rows) and gathers, from the bucket ranges of the queries whose boxes cover
//     those keys, the stored gamma/beta rows, kKvQ queries per step: dK += scale Gamma^T Q,
//     dV += Beta^T dO on tensor cores, written once.
#pragma once

#include "dsa3d_fwd_mma.cuh"

namespace dsa3d {

// Geometry of the stored per-query splats.
struct BoxGeo {
  int rows;      // kt * (kh + 1) box rows per query (tap plane u, box row by)
  int width;     // kw + 1
  int per_q;     // rows * width bf16 values per query and array
};

__device__ __forceinline__ float bf16_val(unsigned short u) { return __uint_as_float((unsigned)u << 16); }

// One 16 x 32 raw-dot block: acc[jt] (n-tile jt, keys X0 + 8jt + [0,8)) = A . src[t, y, seg]^T,
// A = 16 rows given as k-step fragments af (dims as laid out by MmaShape).
template <int DH>
__device__ __forceinline__ void raw_block(float (&acc)[4][4], const unsigned (&af)[MmaShape<DH>::KS][4],
                                          const __nv_bfloat16* src_h, int t, int y, int X0, int segw,
                                          int64_t rs, const Geo& g, int gq, int qq) {
  using S = MmaShape<DH>;
#pragma unroll
  for (int jt = 0; jt < 4; jt++) acc[jt][0] = acc[jt][1] = acc[jt][2] = acc[jt][3] = 0.f;
  if (t < 0 || t >= g.F || y < 0 || y >= g.Hp) return;
#pragma unroll
  for (int jt = 0; jt < 4; jt++) {
    const int col = 8 * jt + gq;
    const int x = X0 + col;
    const bool ok = col < segw && x >= 0 && x < g.Wp;
    const __nv_bfloat16* r = src_h + ((int64_t)(t * g.Hp + y) * g.Wp + max(x, 0)) * rs;
    unsigned w[S::QW];
#pragma unroll
    for (int c = 0; c < S::QW / 4; c++) {
      const uint4 a = ok ? ldg16(r + qk_off(c, qq)) : make_uint4(0, 0, 0, 0);
      w[4 * c] = a.x; w[4 * c + 1] = a.y; w[4 * c + 2] = a.z; w[4 * c + 3] = a.w;
    }
#pragma unroll
    for (int s = 0; s < S::KS; s++)
      mma_bf16_16816(acc[jt], af[s][0], af[s][1], af[s][2], af[s][3], w[2 * s], w[2 * s + 1]);
  }
}

template <int DH>
__device__ __forceinline__ void load_afrags(unsigned (&af)[MmaShape<DH>::KS][4], const __nv_bfloat16* base,
                                            const MmaRow (&R)[2], int h, int heads, int qq) {
  using S = MmaShape<DH>;
  unsigned w0[S::QW], w1[S::QW];
#pragma unroll
  for (int c = 0; c < S::QW / 4; c++) {
    uint4 a = make_uint4(0, 0, 0, 0), b = make_uint4(0, 0, 0, 0);
    if (R[0].live) a = ldg16(base + ((int64_t)R[0].n * heads + h) * DH + qk_off(c, qq));
    if (R[1].live) b = ldg16(base + ((int64_t)R[1].n * heads + h) * DH + qk_off(c, qq));
    w0[4 * c] = a.x; w0[4 * c + 1] = a.y; w0[4 * c + 2] = a.z; w0[4 * c + 3] = a.w;
    w1[4 * c] = b.x; w1[4 * c + 1] = b.y; w1[4 * c + 2] = b.z; w1[4 * c + 3] = b.w;
  }
#pragma unroll
  for (int s = 0; s < S::KS; s++) {
    af[s][0] = w0[2 * s];
    af[s][1] = w1[2 * s];
    af[s][2] = w0[2 * s + 1];
    af[s][3] = w1[2 * s + 1];
  }
}

// Decode the rows of a chunk starting at sorted position pos (cnt rows).
__device__ __forceinline__ void chunk_rows(MmaRow (&R)[2], const Geo& g, const float* off, int h,
                                           const int* sorted_n, int pos, int cnt, int X0, int gq) {
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
      R[hf].hi[a] = R[hf].live ? Qd.hi[a] : -1;
    }
  }
}

// Chunk of the bucket row [pos, qend): count of rows, X0.
__device__ __forceinline__ int chunk_len(const int* sorted_ex, int pos, int qend, int kw, int lane, int& X0) {
  const int ex_l = (lane < 16 && pos + lane < qend) ? sorted_ex[pos + lane] : 0x7fffffff;
  const int ex0 = __shfl_sync(kFull, ex_l, 0);
  const unsigned bal = __ballot_sync(kFull, lane < 16 && pos + lane < qend && ex_l - ex0 <= chunk_span(kw));
  X0 = ex0 - kw;
  return __popc(bal);
}

// ---- pass 1: query side ---------------------------------------------------------------------
// Two warps per chunk.  Per tap plane u and box row by, warp 0 of the pair computes the Q.K MMA
// blocks of box planes u and u+1 and warp 1 the dO.V blocks; each blends its two blocks in
// registers -- (st = S0 + f_t (S1 - S0), bd = S1 - S0), resp. (dpt, dbd) -- and stores them in a
// three-slot ring in shared memory, with one pair barrier per box row (a slot is rewritten two
// box rows after it was read).  Then each warp evaluates eight of the chunk's queries, four lanes
// per query, each lane taking every fourth tap of tap row by-1 (only the query's kw taps, not the
// 32 segment columns): the tap's score, dP, their derivatives along (t, y, x), P and the
// per-query sums.  The taps' P and P dP go to the warp's rows of a two-row tap ring, from which
// box row by-1's splats (x-transpose, then y-mix with the previous tap row) are stored.
constexpr int kRawStride = 40;  // floats per row of a raw block (conflict-free float2 fragment stores)
constexpr int kTapStride = 20;  // floats per row of a tap-row buffer (kw <= 15; 20: four lanes per row
                                // of eight rows fall on distinct banks)
constexpr int kBwdqSlots = 3;

__host__ __device__ constexpr int bwdq_pair_floats() {
  return kBwdqSlots * 4 * 16 * kRawStride + 2 * 2 * 16 * kTapStride;
}

template <int DH>
__global__ void __launch_bounds__(64, DSA3D_BWDQ_MINB)
    dsa3d_bwd_q_kernel(const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k,
                       const __nv_bfloat16* __restrict__ v, const __nv_bfloat16* __restrict__ dout,
                       const float* __restrict__ off, const float* __restrict__ lse,
                       float* __restrict__ doff, const int* __restrict__ start,
                       const int* __restrict__ sorted_n, const int* __restrict__ sorted_ex,
                       unsigned short* __restrict__ gbox, unsigned short* __restrict__ bbox,
                       float2* __restrict__ dft, const Geo g, const SortGeo sg, const BoxGeo bg,
                       const int h0, const int hg) {
  using S = MmaShape<DH>;
  extern __shared__ __align__(16) float dyn_sh[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int pair = warp >> 1, role = warp & 1;  // role 0: Q.K blocks, role 1: dO.V blocks
  const int gq = lane >> 2, qq = lane & 3;
  float* raw = dyn_sh + pair * bwdq_pair_floats();     // [slot 3][block 4][16 rows][stride]
  float* tapb = raw + kBwdqSlots * 4 * 16 * kRawStride;  // [ring 2][P, PdP][16 rows][stride]
  const int er = 8 * role + (lane >> 2), s4 = lane & 3;  // epilogue: query row, tap phase
  const int64_t rs = (int64_t)g.heads * DH;
  const float sc = g.scale * kLog2e;
  const int segw = segment_keys(g.kw);
  const int64_t rows = (int64_t)hg * sg.Et * sg.Ey;
  const unsigned bar_id = 1 + pair;
  const __nv_bfloat16* asrc = role ? dout : q;  // A operand rows of this warp
  int sidx = 0;                                  // box-row steps so far (ring slot = sidx % 3)

  for (int64_t row = (int64_t)blockIdx.x + pair; row < rows; row += (int64_t)gridDim.x) {
    const int hh = (int)(row / ((int64_t)sg.Et * sg.Ey));
    const int rem = (int)(row - (int64_t)hh * sg.Et * sg.Ey);
    const int et = rem / sg.Ey, ey = rem % sg.Ey;
    const int h = h0 + hh;
    const int64_t b0 = (int64_t)hh * sg.E1 + ((int64_t)et * sg.Ey + ey) * sg.Ex;
    const int qbeg = start[b0], qend = start[b0 + sg.Ex];
    const int ot = et - g.kt, oy = ey - g.kh;
    const __nv_bfloat16* bsrc = (role ? v : k) + (int64_t)h * DH;  // B operand rows

    for (int pos = qbeg; pos < qend;) {
      int X0;
      const int cnt = chunk_len(sorted_ex, pos, qend, g.kw, lane, X0);
      MmaRow R[2];  // fragment rows g, g+8 (for the MMA operands and the t-blend)
      chunk_rows(R, g, off, h, sorted_n, pos, cnt, X0, gq);
      unsigned af[S::KS][4];
      load_afrags<DH>(af, asrc, R, h, g.heads, qq);
      // epilogue row er
      const bool elive = er < cnt;
      const int en = elive ? sorted_n[pos + er] : 0;
      const Query EQ = decode_query(g, off, h, en);
      const int eox = EQ.o[2] - X0;
      const float ft = EQ.f[0], fy = EQ.f[1], fx = EQ.f[2];
      const int lo_t = EQ.lo[0], hi_t = elive ? EQ.hi[0] : -1;
      const float lse2 = elive ? __ldg(lse + (int64_t)h * g.N + en) * kLog2e : 0.f;
      float Dp = 0.f, A[3] = {0.f, 0.f, 0.f}, Bs[3] = {0.f, 0.f, 0.f}, C[3] = {0.f, 0.f, 0.f};
      const int64_t qbox = (int64_t)(elive ? pos + er : pos) * bg.per_q;

      for (int u = 0; u < g.kt; u++) {
        const bool eplane = lo_t <= u && u <= hi_t;
        for (int sk = 0; sk < 4; sk++)
          for (int c = s4; c < kTapStride; c += 4) tapb[(sk * 16 + er) * kTapStride + c] = 0.f;
        __syncwarp();
        for (int by = 0; by <= g.kh; by++, sidx++) {
          const int y = oy + by;
          float* rc = raw + (sidx % kBwdqSlots) * 4 * 16 * kRawStride;
          {
            float s0[4][4], s1[4][4];
            raw_block<DH>(s0, af, bsrc, ot + u, y, X0, segw, rs, g, gq, qq);
            raw_block<DH>(s1, af, bsrc, ot + u + 1, y, X0, segw, rs, g, gq, qq);
            float* blk = rc + (2 * role) * 16 * kRawStride;
#pragma unroll
            for (int jt = 0; jt < 4; jt++)
#pragma unroll
              for (int hf = 0; hf < 2; hf++) {
                const int rr = gq + 8 * hf, cc = 8 * jt + 2 * qq;
                const float d0 = s1[jt][2 * hf] - s0[jt][2 * hf], d1 = s1[jt][2 * hf + 1] - s0[jt][2 * hf + 1];
                *reinterpret_cast<float2*>(blk + rr * kRawStride + cc) =
                    make_float2(fmaf(R[hf].f[0], d0, s0[jt][2 * hf]), fmaf(R[hf].f[0], d1, s0[jt][2 * hf + 1]));
                *reinterpret_cast<float2*>(blk + (16 + rr) * kRawStride + cc) = make_float2(d0, d1);
              }
          }
          asm volatile("bar.sync %0, 64;\n" ::"r"(bar_id) : "memory");
          if (by >= 1) {
            const int ty = by - 1;
            const float* rp = raw + ((sidx + kBwdqSlots - 1) % kBwdqSlots) * 4 * 16 * kRawStride;
            float* tp = tapb + (ty & 1) * 2 * 16 * kTapStride;
            const bool erow = eplane && EQ.lo[1] <= ty && ty <= EQ.hi[1];
            // this lane's taps form a run [t0, t1) of tap row ty; tap wx blends columns wx and
            // wx+1, so each column's four blocks are read and y-blended once and kept for the
            // next tap: Y = y-lerps of blocks 0..3, then the y-differences of blocks 0 and 2
            {
              const int run = (g.kw + 3) >> 2;
              const int t0 = s4 * run, t1 = min(t0 + run, g.kw);
              float Yp[6] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
              for (int jj = 0; jj <= 4; jj++) {  // run <= 4 taps (kw <= 15): at most 5 columns
                const int j = t0 + jj;
                if (j > t1 || t0 >= t1) break;
                const int c = er * kRawStride + eox + j;
                float Y[6];
#pragma unroll
                for (int b = 0; b < 4; b++) {
                  const float pv = rp[b * 16 * kRawStride + c], cv = rc[b * 16 * kRawStride + c];
                  Y[b] = fmaf(fy, cv - pv, pv);
                  if (b == 0) Y[4] = cv - pv;
                  if (b == 2) Y[5] = cv - pv;
                }
                if (j > t0) {
                  const int wx = j - 1;
                  float P = 0.f, PdP = 0.f;
                  if (erow && wx >= EQ.lo[2] && wx <= EQ.hi[2]) {
                    const float s = fmaf(fx, Y[0] - Yp[0], Yp[0]);
                    const float dpv = fmaf(fx, Y[2] - Yp[2], Yp[2]);
                    const float ds[3] = {fmaf(fx, Y[1] - Yp[1], Yp[1]), fmaf(fx, Y[4] - Yp[4], Yp[4]),
                                         Y[0] - Yp[0]};
                    const float dp[3] = {fmaf(fx, Y[3] - Yp[3], Yp[3]), fmaf(fx, Y[5] - Yp[5], Yp[5]),
                                         Y[2] - Yp[2]};
                    P = exp2f(fmaf(s, sc, -lse2));
                    PdP = P * dpv;
                    Dp += PdP;
#pragma unroll
                    for (int ax = 0; ax < 3; ax++) {
                      A[ax] = fmaf(PdP, ds[ax], A[ax]);
                      Bs[ax] = fmaf(P, ds[ax], Bs[ax]);
                      C[ax] = fmaf(P, dp[ax], C[ax]);
                    }
                  }
                  tp[(0 * 16 + er) * kTapStride + wx] = P;
                  tp[(1 * 16 + er) * kTapStride + wx] = PdP;
                }
#pragma unroll
                for (int e = 0; e < 6; e++) Yp[e] = Y[e];
              }
            }
            __syncwarp();
            // splat onto box row ty: this lane's run of column pairs [w0, w1); column bx takes
            // taps bx and bx-1 of each tap row, so tap values roll from one column to the next
            const float* tq = tapb + ((ty + 1) & 1) * 2 * 16 * kTapStride;  // tap row ty-1
            {
              const int words = bg.width >> 1, wrun = (words + 3) >> 2;
              const int w0 = s4 * wrun, w1 = min(w0 + wrun, words);
              if (elive && w0 < w1) {
                const int64_t o = qbox + (u * (g.kh + 1) + ty) * bg.width;
                float prv[4];  // taps at bx - 1: tap row ty (P, P dP), tap row ty-1 (P, P dP)
                {
                  const int x = 2 * w0 - 1;
                  const bool in = x >= 0;
                  prv[0] = in ? tp[er * kTapStride + x] : 0.f;
                  prv[1] = in ? tp[(16 + er) * kTapStride + x] : 0.f;
                  prv[2] = in ? tq[er * kTapStride + x] : 0.f;
                  prv[3] = in ? tq[(16 + er) * kTapStride + x] : 0.f;
                }
#pragma unroll
                for (int ww = 0; ww < 2; ww++) {  // wrun <= 2 (kw <= 15)
                  const int w = w0 + ww;
                  if (w >= w1) break;
                  float vb[2], vg[2];
#pragma unroll
                  for (int e = 0; e < 2; e++) {
                    const int bx = 2 * w + e;
                    const bool in = bx < g.kw;
                    const float cur[4] = {in ? tp[er * kTapStride + bx] : 0.f,
                                          in ? tp[(16 + er) * kTapStride + bx] : 0.f,
                                          in ? tq[er * kTapStride + bx] : 0.f,
                                          in ? tq[(16 + er) * kTapStride + bx] : 0.f};
                    const float cb0 = fmaf(fx, prv[0] - cur[0], cur[0]), cg0 = fmaf(fx, prv[1] - cur[1], cur[1]);
                    const float cb1 = fmaf(fx, prv[2] - cur[2], cur[2]), cg1 = fmaf(fx, prv[3] - cur[3], cur[3]);
                    vb[e] = fmaf(fy, cb1 - cb0, cb0);
                    vg[e] = fmaf(fy, cg1 - cg0, cg0);
#pragma unroll
                    for (int i = 0; i < 4; i++) prv[i] = cur[i];
                  }
                  *reinterpret_cast<unsigned*>(bbox + o + 2 * w) = bf16x2_bits(vb[0], vb[1]);
                  *reinterpret_cast<unsigned*>(gbox + o + 2 * w) = bf16x2_bits(vg[0], vg[1]);
                }
              }
            }
            __syncwarp();
          }
        }
        // box row kh takes only the y-carry of tap row kh-1
        {
          const float* tq = tapb + ((g.kh - 1) & 1) * 2 * 16 * kTapStride;
          const int words = bg.width >> 1, wrun = (words + 3) >> 2;
          const int w0 = s4 * wrun, w1 = min(w0 + wrun, words);
          if (elive && w0 < w1) {
            const int64_t o = qbox + (u * (g.kh + 1) + g.kh) * bg.width;
            const int x = 2 * w0 - 1;
            float prv[2] = {x >= 0 ? tq[er * kTapStride + x] : 0.f, x >= 0 ? tq[(16 + er) * kTapStride + x] : 0.f};
#pragma unroll
            for (int ww = 0; ww < 2; ww++) {
              const int w = w0 + ww;
              if (w >= w1) break;
              float vb[2], vg[2];
#pragma unroll
              for (int e = 0; e < 2; e++) {
                const int bx = 2 * w + e;
                const bool in = bx < g.kw;
                const float c0 = in ? tq[er * kTapStride + bx] : 0.f, c1 = in ? tq[(16 + er) * kTapStride + bx] : 0.f;
                vb[e] = fy * fmaf(fx, prv[0] - c0, c0);
                vg[e] = fy * fmaf(fx, prv[1] - c1, c1);
                prv[0] = c0;
                prv[1] = c1;
              }
              *reinterpret_cast<unsigned*>(bbox + o + 2 * w) = bf16x2_bits(vb[0], vb[1]);
              *reinterpret_cast<unsigned*>(gbox + o + 2 * w) = bf16x2_bits(vg[0], vg[1]);
            }
          }
        }
        __syncwarp();
      }

      // per-query totals: combine the row's four lanes, then D, doff, (D, f_t)
#pragma unroll
      for (int d = 1; d <= 2; d <<= 1) {
        Dp += __shfl_xor_sync(kFull, Dp, d);
#pragma unroll
        for (int ax = 0; ax < 3; ax++) {
          A[ax] += __shfl_xor_sync(kFull, A[ax], d);
          Bs[ax] += __shfl_xor_sync(kFull, Bs[ax], d);
          C[ax] += __shfl_xor_sync(kFull, C[ax], d);
        }
      }
      if (elive && s4 == 0) {
        float* od = doff + ((int64_t)h * g.N + en) * 3;
#pragma unroll
        for (int ax = 0; ax < 3; ax++) od[ax] = fmaf(g.scale, fmaf(-Dp, Bs[ax], A[ax]), C[ax]);
        dft[pos + er] = make_float2(Dp, ft);
      }
      pos += cnt;
    }
  }
}

// ---- shared helpers of passes 2 and 3 ----------------------------------------------------------
// gamma and beta of one query at box plane bt, box row by, columns 2w and 2w+1 (one 32-bit word
// of each stored row; rows hold an even number of bf16 values, so words are 4-byte aligned).
__device__ __forceinline__ void box_word(const unsigned short* gbox, const unsigned short* bbox,
                                         int64_t pos, const BoxGeo& bg, int kt, int kh, int bt,
                                         int by, int w, float D, float ft, float (&gam)[2],
                                         float (&bet)[2]) {
  gam[0] = gam[1] = bet[0] = bet[1] = 0.f;
  if (bt < kt) {
    const int64_t o = (pos * bg.rows + bt * (kh + 1) + by) * bg.width + 2 * w;
    const unsigned bw = *reinterpret_cast<const unsigned*>(bbox + o);
    const unsigned gw = *reinterpret_cast<const unsigned*>(gbox + o);
#pragma unroll
    for (int e = 0; e < 2; e++) {
      const float b = bf16_val((unsigned short)(bw >> (16 * e))), gp = bf16_val((unsigned short)(gw >> (16 * e)));
      bet[e] = (1.f - ft) * b;
      gam[e] = (1.f - ft) * fmaf(-D, b, gp);
    }
  }
  if (bt >= 1) {
    const int64_t o = (pos * bg.rows + (bt - 1) * (kh + 1) + by) * bg.width + 2 * w;
    const unsigned bw = *reinterpret_cast<const unsigned*>(bbox + o);
    const unsigned gw = *reinterpret_cast<const unsigned*>(gbox + o);
#pragma unroll
    for (int e = 0; e < 2; e++) {
      const float b = bf16_val((unsigned short)(bw >> (16 * e))), gp = bf16_val((unsigned short)(gw >> (16 * e)));
      bet[e] = fmaf(ft, b, bet[e]);
      gam[e] = fmaf(ft, fmaf(-D, b, gp), gam[e]);
    }
  }
}

// ---- pass 2: dq = scale * sum_j gamma[j] K[j] ----------------------------------------------------
// Per warp and chunk, per box plane bt and box row by (the box's in-volume rectangle, in order):
// the chunk's gamma tile (16 queries x 32 segment keys, bf16) and the K segment of key row
// (o_t + bt, o_y + by) in shared memory, then acc += gamma . K_seg on tensor cores (A by ldmatrix,
// B by ldmatrix.trans of the staged key rows).  Software pipeline: the next step's K segment is
// copied by cp.async into the other of two buffers and its stored splat words are loaded into
// registers while the current step's MMAs run.
constexpr int kDqTile = 40;  // gamma tile row stride (bf16): conflict-free ldmatrix
template <int DH>
__host__ __device__ constexpr int dq_warp_bytes() {
  return (2 * 32 * (DH + 8) + 16 * kDqTile) * 2;
}

template <int DH>
__global__ void __launch_bounds__(128, DSA3D_DQ_MINB)
    dsa3d_bwd_dq_kernel(const __nv_bfloat16* __restrict__ k, __nv_bfloat16* __restrict__ dq,
                        const int* __restrict__ start, const int* __restrict__ sorted_n,
                        const int* __restrict__ sorted_ex, const unsigned short* __restrict__ gbox,
                        const unsigned short* __restrict__ bbox, const float2* __restrict__ dft,
                        const Geo g, const SortGeo sg, const BoxGeo bg, const int h0, const int hg) {
  constexpr int NT = DH / 8;       // n-tiles of dq
  constexpr int KR = DH + 8;       // staged key row stride (bf16): conflict-free ldmatrix.trans
  constexpr int CH = DH / 8;       // 16-byte chunks per key row
  extern __shared__ __align__(16) unsigned char dq_sh[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int gq = lane >> 2, qq = lane & 3;
  unsigned short* kbuf = reinterpret_cast<unsigned short*>(dq_sh + warp * dq_warp_bytes<DH>());
  unsigned short* tile = kbuf + 2 * 32 * KR;
  const int64_t rs = (int64_t)g.heads * DH;
  const int segw = segment_keys(g.kw);
  const int64_t rows = (int64_t)hg * sg.Et * sg.Ey;
  const int r = lane >> 1;  // gather: query row of this lane, stored words (lane & 1) + 2i

  for (int64_t row = (int64_t)blockIdx.x * 4 + warp; row < rows; row += (int64_t)gridDim.x * 4) {
    const int hh = (int)(row / ((int64_t)sg.Et * sg.Ey));
    const int rem = (int)(row - (int64_t)hh * sg.Et * sg.Ey);
    const int et = rem / sg.Ey, ey = rem % sg.Ey;
    const int h = h0 + hh;
    const int64_t b0 = (int64_t)hh * sg.E1 + ((int64_t)et * sg.Ey + ey) * sg.Ex;
    const int qbeg = start[b0], qend = start[b0 + sg.Ex];
    const int ot = et - g.kt, oy = ey - g.kh;
    const __nv_bfloat16* kh_ = k + (int64_t)h * DH;
    // the box's planes and rows inside the volume
    const int bt0 = max(0, -ot), bt1 = min(g.kt, g.F - 1 - ot);
    const int by0 = max(0, -oy), by1 = min(g.kh, g.Hp - 1 - oy);
    const int nby = by1 - by0 + 1;
    const int nsteps = (bt1 >= bt0 && by1 >= by0) ? (bt1 - bt0 + 1) * nby : 0;

    for (int pos = qbeg; pos < qend;) {
      int X0;
      const int cnt = chunk_len(sorted_ex, pos, qend, g.kw, lane, X0);
      const bool rlive = r < cnt;
      const float2 d = rlive ? dft[pos + r] : make_float2(0.f, 0.f);
      const int col0 = rlive ? sorted_ex[pos + r] - g.kw - X0 : 0;
      float acc[NT][4];
#pragma unroll
      for (int j = 0; j < NT; j++) acc[j][0] = acc[j][1] = acc[j][2] = acc[j][3] = 0.f;

      // This lane's part of a K segment copy: keys lane / CH + KPI * i (i < CH), 16-byte chunk
      // lane % CH.  The segment's x-range is fixed for the chunk, so the per-key source offsets
      // and the in-row mask are set once here; a step only adds its key row's base.
      constexpr int KPI = 32 / CH;
      const int key_l = lane / CH, ch_l = lane % CH;
      const int64_t src0 = (int64_t)(X0 + key_l) * rs + ch_l * 8;
      unsigned vmask = 0;
#pragma unroll
      for (int i = 0; i < CH; i++) {
        const int key = key_l + KPI * i, x = X0 + key;
        vmask |= (key < segw && x >= 0 && x < g.Wp) ? (1u << i) : 0u;
      }
      // K segment of step i -> buffer b (zero-filled outside the row and the segment)
      auto issue_k = [&](int i, int b) {
        const int bt = bt0 + i / nby, by = by0 + i % nby;
        const __nv_bfloat16* krow = kh_ + (int64_t)((ot + bt) * g.Hp + oy + by) * g.Wp * rs;
        const __nv_bfloat16* src = krow + src0;
        unsigned short* dst = kbuf + b * 32 * KR + key_l * KR + ch_l * 8;
#pragma unroll
        for (int c = 0; c < CH; c++) {
          const bool ok = (vmask >> c) & 1u;
          cp_async16_zfill(dst + c * KPI * KR, ok ? src + (int64_t)c * KPI * rs : krow, ok);
        }
        cp_async_commit();
      };
      // stored gamma'/beta words of step i for this lane's row: [word][plane bt, bt-1][gamma', beta]
      const int64_t gofs = (int64_t)(rlive ? pos + r : pos) * bg.per_q + 2 * (lane & 1);
      const unsigned short* grow = gbox + gofs;
      const unsigned short* brow = bbox + gofs;
      unsigned wd[4][4];
      auto gather_load = [&](int i) {
        const int bt = bt0 + i / nby, by = by0 + i % nby;
        const int o0 = (bt * (g.kh + 1) + by) * bg.width, o1 = o0 - (g.kh + 1) * bg.width;
#pragma unroll
        for (int ii = 0; ii < 4; ii++) {
          const int w = (lane & 1) + 2 * ii;
          wd[ii][0] = wd[ii][1] = wd[ii][2] = wd[ii][3] = 0u;
          if (!rlive || 2 * w >= bg.width) continue;
          if (bt < g.kt) {
            wd[ii][0] = *reinterpret_cast<const unsigned*>(grow + o0 + 4 * ii);
            wd[ii][1] = *reinterpret_cast<const unsigned*>(brow + o0 + 4 * ii);
          }
          if (bt >= 1) {
            wd[ii][2] = *reinterpret_cast<const unsigned*>(grow + o1 + 4 * ii);
            wd[ii][3] = *reinterpret_cast<const unsigned*>(brow + o1 + 4 * ii);
          }
        }
      };

      if (nsteps > 0) {
        issue_k(0, 0);
        gather_load(0);
      }
      for (int s = 0; s < nsteps; s++) {
        // gamma tile of step s: t-mix of (gamma' - D beta) of the tap planes bt and bt-1
        for (int i = lane; i < 16 * kDqTile / 8; i += 32) reinterpret_cast<uint4*>(tile)[i] = make_uint4(0, 0, 0, 0);
        __syncwarp();
        if (rlive) {
#pragma unroll
          for (int ii = 0; ii < 4; ii++) {
            const int w = (lane & 1) + 2 * ii;
            if (2 * w >= bg.width) continue;
#pragma unroll
            for (int e = 0; e < 2; e++) {
              const float g0 = bf16_val((unsigned short)(wd[ii][0] >> (16 * e)));
              const float b0_ = bf16_val((unsigned short)(wd[ii][1] >> (16 * e)));
              const float g1 = bf16_val((unsigned short)(wd[ii][2] >> (16 * e)));
              const float b1_ = bf16_val((unsigned short)(wd[ii][3] >> (16 * e)));
              const float c0 = fmaf(-d.x, b0_, g0), c1 = fmaf(-d.x, b1_, g1);
              tile[r * kDqTile + col0 + 2 * w + e] = bf16_bits(fmaf(d.y, c1 - c0, c0));
            }
          }
        }
        const bool more = s + 1 < nsteps;
        if (more) {
          issue_k(s + 1, (s + 1) & 1);
          gather_load(s + 1);
          cp_async_wait_group1();
        } else {
          cp_async_wait_all();
        }
        __syncwarp();
        const unsigned short* kb_ = kbuf + (s & 1) * 32 * KR;
        const int rr = (lane & 7) + 8 * ((lane >> 3) & 1);
#pragma unroll
        for (int kk = 0; kk < 2; kk++) {
          unsigned a[4];
          ldsm_x4(a, tile + rr * kDqTile + 8 * (lane >> 4) + 16 * kk);
#pragma unroll
          for (int j2 = 0; j2 < NT / 2; j2++) {
            unsigned bq[4];
            ldsm_x4_trans(bq, kb_ + (16 * kk + rr) * KR + 16 * j2 + 8 * (lane >> 4));
            mma_bf16_16816(acc[2 * j2], a[0], a[1], a[2], a[3], bq[0], bq[1]);
            mma_bf16_16816(acc[2 * j2 + 1], a[0], a[1], a[2], a[3], bq[2], bq[3]);
          }
        }
        __syncwarp();
      }
      // n-tile j, columns 2q, 2q+1 -> dims 8j + 2q, 8j + 2q + 1
#pragma unroll
      for (int hf = 0; hf < 2; hf++) {
        const int rq = gq + 8 * hf;
        if (rq >= cnt) continue;
        const int n = sorted_n[pos + rq];
        __nv_bfloat16* drow = dq + ((int64_t)n * g.heads + h) * DH;
#pragma unroll
        for (int j = 0; j < NT; j++)
          *reinterpret_cast<__nv_bfloat162*>(drow + 8 * j + 2 * qq) =
              __floats2bfloat162_rn(acc[j][2 * hf] * g.scale, acc[j][2 * hf + 1] * g.scale);
      }
      pos += cnt;
    }
  }
}

// ---- pass 3: key side ------------------------------------------------------------------------
// One CTA owns a key tile of kKvRows consecutive key rows x 16 keys
// (x in [16b, 16b+16)) of one frame tk and head; warp w takes key row w/2 and half w%2 of the
// head dims, with dK and dV in registers.  The queries whose windows cover the tile have origins
// o_t = tk - bt, o_y in [yk0 - kh, yk0 + kKvRows - 1], o_x in [16b - kw, 16b + 15], i.e. bucket
// rows e_t = tk - bt + kt, e_y in [yk0, yk0 + kKvRows - 1 + kh] and the e_x range
// [16b, 16b + 16 + kw).  Per step (kKvQ such queries, in sorted order across those bucket rows)
// the CTA stages their q and dO rows and its key rows' Gamma^T / Beta^T tiles (key x query,
// gathered from the stored splats) in shared memory; each warp then adds Gamma^T q and Beta^T dO
// for its key row with m16n8k16 MMAs (B fragments by ldmatrix.trans of the staged rows).  A query
// row is loaded once per tile, not once per key row.
#ifndef DSA3D_KV_ROWS
#define DSA3D_KV_ROWS 4
#endif
constexpr int kKvRows = DSA3D_KV_ROWS;  // key rows per CTA (2 warps each)
constexpr int kKvThreads = 64 * kKvRows;
constexpr int kKvRanges = 64;  // bucket-row ranges per batch (two per lane of warp 0)
#ifndef DSA3D_KV_QPS
#define DSA3D_KV_QPS 32
#endif
constexpr int kKvQ = DSA3D_KV_QPS;  // queries per step (the MMAs' k dimension: 16 per k-step)
static_assert(kKvQ % 16 == 0 && kKvQ <= 32, "whole k-steps; one warp locates a step's slots");

// One query slot of a key-side step.
struct KvSlot {
  int64_t row;   // element offset of the query's q / dO row
  int64_t box;   // element offset of the query's stored splats
  int tok;     // token, -1 for an empty slot
  int bt;      // box plane of the tile's frame in the query's box
  int by0;     // box row of the tile's first key row (may lie outside [0, kh])
  int ox;      // x-origin minus the tile's first key x
  float2 d;    // (D, f_t)
};

template <int DH>
__host__ __device__ constexpr int kv_dyn_bytes() {
  return (6 * kKvRows * 16 * (kKvQ + 8) + 4 * kKvQ * (DH + 8)) * 2;
}

template <int DH>
__global__ void __launch_bounds__(kKvThreads, DSA3D_KV_MINB)
    dsa3d_bwd_kv_kernel(const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ dout,
                        __nv_bfloat16* __restrict__ dk, __nv_bfloat16* __restrict__ dv,
                        const int* __restrict__ start, const int* __restrict__ sorted_n,
                        const int* __restrict__ sorted_ex, const unsigned short* __restrict__ gbox,
                        const unsigned short* __restrict__ bbox, const float2* __restrict__ dft,
                        const Geo g, const SortGeo sg, const BoxGeo bg, const int h0, const int hg) {
  constexpr int HALF = DH / 2;  // dims per warp
  constexpr int NTH = HALF / 8; // n-tiles per warp
  constexpr int TS = kKvQ + 8;  // Gamma/Beta tile row stride (bf16): conflict-free ldmatrix
  constexpr int RS = DH + 8;    // staged q/dO row stride (bf16): conflict-free ldmatrix.trans
  constexpr int TILE = kKvRows * 16 * TS;  // one stage of Gamma^T (or Beta^T) tiles
  constexpr int WT = kKvThreads / kKvQ;    // gather threads per query slot
  constexpr int NW = (8 + WT - 1) / WT;    // stored words per gather thread (a row has <= 8)
  // dynamic shared memory: Gamma^T and Beta^T tiles [3 stages][TILE], q and dO rows [2][kKvQ][RS]
  extern __shared__ __align__(16) unsigned short kv_sh[];
  unsigned short (*tg)[TILE] = reinterpret_cast<unsigned short (*)[TILE]>(kv_sh);
  unsigned short (*tb)[TILE] = reinterpret_cast<unsigned short (*)[TILE]>(kv_sh + 3 * TILE);
  unsigned short (*qs)[kKvQ * RS] = reinterpret_cast<unsigned short (*)[kKvQ * RS]>(kv_sh + 6 * TILE);
  unsigned short (*os)[kKvQ * RS] = reinterpret_cast<unsigned short (*)[kKvQ * RS]>(kv_sh + 6 * TILE + 2 * kKvQ * RS);
  __shared__ KvSlot meta[2][kKvQ];
  __shared__ int r_beg[kKvRanges], r_pre[kKvRanges + 1];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int gq = lane >> 2, qq = lane & 3;
  const int wr = warp >> 1, half = warp & 1;
  const int gm = tid / WT, gw = tid % WT;  // gather: query slot, stored word
  const int NB = (g.Wp + 15) / 16;
  const int NY = (g.Hp + kKvRows - 1) / kKvRows;
  const int64_t tiles = (int64_t)hg * g.F * NY * NB;

  for (int64_t tile = blockIdx.x; tile < tiles; tile += gridDim.x) {
    int64_t r = tile;
    const int b = (int)(r % NB);
    r /= NB;
    const int yb = (int)(r % NY);
    r /= NY;
    const int tk = (int)(r % g.F);
    const int hh = (int)(r / g.F);
    const int h = h0 + hh;
    const int x_lo = 16 * b, yk0 = kKvRows * yb;
    const int myk = yk0 + wr;  // this warp's key row

    float ak[NTH][4], av[NTH][4];
#pragma unroll
    for (int j = 0; j < NTH; j++)
#pragma unroll
      for (int e = 0; e < 4; e++) ak[j][e] = av[j][e] = 0.f;

    // The queries covering the tile lie in (kt + 1) x ney bucket-row ranges of the sorted order
    // (range r: bt = r / ney, ey = yk0 + r % ney).  They are taken in batches of up to kKvRanges
    // ranges, concatenated, and consumed kKvQ at a time, so a step mixes queries of several bucket
    // rows and only the last step of a batch is partly empty.
    const int ney = min(yk0 + kKvRows - 1 + g.kh, sg.Ey - 1) - yk0 + 1;
    const int nranges = (g.kt + 1) * ney;
    for (int rb = 0; rb < nranges; rb += kKvRanges) {
      const int nr = min(kKvRanges, nranges - rb);
      __syncthreads();  // the previous batch's ranges and buffers are consumed
      if (warp == 0) {
        int len[2];
#pragma unroll
        for (int e = 0; e < 2; e++) {
          const int rr = 2 * lane + e;
          len[e] = 0;
          if (rr < nr) {
            const int bt = (rb + rr) / ney, ey = yk0 + (rb + rr) - bt * ney;
            const int64_t b0 = (int64_t)hh * sg.E1 + ((int64_t)(tk - bt + g.kt) * sg.Ey + ey) * sg.Ex;
            const int qb = start[b0 + x_lo];
            r_beg[rr] = qb;
            len[e] = start[b0 + min(x_lo + 16 + g.kw, sg.Ex)] - qb;
          }
        }
        const int pair = len[0] + len[1];
        int incl = pair;
#pragma unroll
        for (int d = 1; d < 32; d <<= 1) {
          const int y = __shfl_up_sync(kFull, incl, d);
          if (lane >= d) incl += y;
        }
        r_pre[2 * lane] = incl - pair;
        r_pre[2 * lane + 1] = incl - pair + len[0];
        if (lane == 31) r_pre[kKvRanges] = incl;
      }
      __syncthreads();
      const int total = r_pre[kKvRanges];
      const int nsteps = (total + kKvQ - 1) / kKvQ;
      if (nsteps == 0) continue;

      // slot tid (< kKvQ) of step s: the query's sorted position, box plane, box row of key row
      // yk0, token, x-origin relative to the tile and (D, f_t); tok = -1 for an empty slot
      auto load_slot = [&](int s) {
        KvSlot m;
        m.tok = -1;
        const int i = kKvQ * s + tid;
        if (i < total) {
          int lo = 0, hi = kKvRanges;  // largest r with r_pre[r] <= i (a non-empty range)
          while (hi - lo > 1) {
            const int mid = (lo + hi) >> 1;
            if (r_pre[mid] <= i) lo = mid; else hi = mid;
          }
          const int pos = r_beg[lo] + (i - r_pre[lo]);
          const int bt = (rb + lo) / ney;
          m.bt = bt;
          m.box = (int64_t)pos * bg.per_q;
          m.by0 = g.kh - ((rb + lo) - bt * ney);  // yk0 - ey + kh
          m.tok = sorted_n[pos];
          m.row = ((int64_t)m.tok * g.heads + h) * DH;
          m.ox = sorted_ex[pos] - g.kw - x_lo;
          m.d = dft[pos];
        }
        return m;
      };
      // q and dO rows of step s into buffer s & 1 (zero-filled for empty slots)
      auto stage_rows = [&](int s) {
        const KvSlot* ms = meta[s & 1];
        constexpr int CH = DH / 8;  // 16-byte chunks per row
        static_assert((2 * kKvQ * CH) % kKvThreads == 0, "whole copy rounds");
#pragma unroll
        for (int k = 0; k < 2 * kKvQ * CH / kKvThreads; k++) {
          const int i = tid + k * kKvThreads;
          const int which = i / (kKvQ * CH);
          const int m = (i / CH) % kKvQ, c = i % CH;
          const bool ok = ms[m].tok >= 0;
          const __nv_bfloat16* src = (which ? dout : q) + (ok ? ms[m].row + c * 8 : 0);
          cp_async16_zfill((which ? os[s & 1] : qs[s & 1]) + m * RS + c * 8, src, ok);
        }
        cp_async_commit();
      };
      // the stored words of step s this thread gathers (words gw + WT iw of the query's rows):
      // per key row, planes bt and bt-1
      struct Words { unsigned g0[NW][kKvRows], b0[NW][kKvRows], g1[NW][kKvRows], b1[NW][kKvRows]; };
      auto gather_load = [&](int s, Words& wd, KvSlot& m) {
        m = meta[s & 1][gm];
#pragma unroll
        for (int iw = 0; iw < NW; iw++)
#pragma unroll
          for (int kr = 0; kr < kKvRows; kr++) wd.g0[iw][kr] = wd.b0[iw][kr] = wd.g1[iw][kr] = wd.b1[iw][kr] = 0u;
        if (m.tok < 0) return;
        const int o0 = (m.bt * (g.kh + 1) + m.by0) * bg.width, o1 = o0 - (g.kh + 1) * bg.width;
#pragma unroll
        for (int iw = 0; iw < NW; iw++) {
          const int w = gw + WT * iw;
          const int key0 = m.ox + 2 * w;
          if (2 * w >= bg.width || key0 + 1 < 0 || key0 >= 16) continue;
          const unsigned short* grow = gbox + m.box + 2 * w;
          const unsigned short* brow = bbox + m.box + 2 * w;
#pragma unroll
          for (int kr = 0; kr < kKvRows; kr++) {
            const int by = m.by0 + kr;
            if (by < 0 || by > g.kh || yk0 + kr >= g.Hp) continue;
            if (m.bt < g.kt) {
              wd.g0[iw][kr] = *reinterpret_cast<const unsigned*>(grow + o0 + kr * bg.width);
              wd.b0[iw][kr] = *reinterpret_cast<const unsigned*>(brow + o0 + kr * bg.width);
            }
            if (m.bt >= 1) {
              wd.g1[iw][kr] = *reinterpret_cast<const unsigned*>(grow + o1 + kr * bg.width);
              wd.b1[iw][kr] = *reinterpret_cast<const unsigned*>(brow + o1 + kr * bg.width);
            }
          }
        }
      };
      // gamma = t-mix of (gamma' - D beta), beta = t-mix of beta, into the stage's tiles
      auto gather_store = [&](int stage, const Words& wd, const KvSlot& m) {
        if (m.tok < 0) return;
        const float D = m.d.x, ft = m.d.y;
#pragma unroll
        for (int iw = 0; iw < NW; iw++) {
          const int w = gw + WT * iw;
          const int key0 = m.ox + 2 * w;
          if (2 * w >= bg.width || key0 + 1 < 0 || key0 >= 16) continue;
#pragma unroll
          for (int kr = 0; kr < kKvRows; kr++) {
#pragma unroll
            for (int e = 0; e < 2; e++) {
              const int key = key0 + e;
              if (key < 0 || key >= 16) continue;
              const float bb0 = bf16_val((unsigned short)(wd.b0[iw][kr] >> (16 * e)));
              const float gg0 = bf16_val((unsigned short)(wd.g0[iw][kr] >> (16 * e)));
              const float bb1 = bf16_val((unsigned short)(wd.b1[iw][kr] >> (16 * e)));
              const float gg1 = bf16_val((unsigned short)(wd.g1[iw][kr] >> (16 * e)));
              const float be = fmaf(ft, bb1 - bb0, bb0);
              const float c0 = fmaf(-D, bb0, gg0), c1 = fmaf(-D, bb1, gg1);
              const float ga = fmaf(ft, c1 - c0, c0);
              tg[stage][kr * 16 * TS + key * TS + gm] = bf16_bits(ga);
              tb[stage][kr * 16 * TS + key * TS + gm] = bf16_bits(be);
            }
          }
        }
      };
      auto zero_stage = [&](int stage) {
        for (int i = tid; i < TILE / 8; i += kKvThreads) {
          reinterpret_cast<uint4*>(tg[stage])[i] = make_uint4(0, 0, 0, 0);
          reinterpret_cast<uint4*>(tb[stage])[i] = make_uint4(0, 0, 0, 0);
        }
      };

      // prologue: slots of steps 0 and 1, step 0's rows and tiles
      if (tid < kKvQ) {
        meta[0][tid] = load_slot(0);
        meta[1][tid] = load_slot(1);
      }
      zero_stage(0);
      zero_stage(1);
      __syncthreads();
      {
        stage_rows(0);
        Words wd;
        KvSlot m;
        gather_load(0, wd, m);
        gather_store(0, wd, m);
        cp_async_wait_all();
      }
      __syncthreads();

      // step s: prefetch step s+1 (rows by cp.async, stored words into registers) and the slots
      // of step s+2, run step s's MMAs, then complete step s+1's tiles; one barrier per step
      for (int s = 0; s < nsteps; s++) {
        const bool more = s + 1 < nsteps;
        zero_stage((s + 2) % 3);
        Words wd;
        KvSlot m;
        if (more) {
          stage_rows(s + 1);
          gather_load(s + 1, wd, m);
        }
        KvSlot next;
        next.tok = -1;
        if (tid < kKvQ && s + 2 < nsteps) next = load_slot(s + 2);

        if (myk < g.Hp) {
          const unsigned short* tgs = tg[s % 3] + wr * 16 * TS;
          const unsigned short* tbs = tb[s % 3] + wr * 16 * TS;
          const unsigned short* qsb = qs[s & 1];
          const unsigned short* osb = os[s & 1];
          const int rr = (lane & 7) + 8 * ((lane >> 3) & 1), cc = 8 * (lane >> 4);
#pragma unroll
          for (int kq = 0; kq < kKvQ / 16; kq++) {  // k-steps over the step's queries
            unsigned agm[4], abt[4];
            ldsm_x4(agm, tgs + rr * TS + 16 * kq + cc);
            ldsm_x4(abt, tbs + rr * TS + 16 * kq + cc);
#pragma unroll
            for (int j2 = 0; j2 < NTH / 2; j2++) {
              // B fragments of n-tiles 2*j2, 2*j2+1: rows = queries (k), cols = dims (n)
              const int dcol = half * HALF + 16 * j2 + 8 * (lane >> 4);
              unsigned bq[4], bo[4];
              ldsm_x4_trans(bq, qsb + (16 * kq + rr) * RS + dcol);
              ldsm_x4_trans(bo, osb + (16 * kq + rr) * RS + dcol);
              mma_bf16_16816(ak[2 * j2], agm[0], agm[1], agm[2], agm[3], bq[0], bq[1]);
              mma_bf16_16816(ak[2 * j2 + 1], agm[0], agm[1], agm[2], agm[3], bq[2], bq[3]);
              mma_bf16_16816(av[2 * j2], abt[0], abt[1], abt[2], abt[3], bo[0], bo[1]);
              mma_bf16_16816(av[2 * j2 + 1], abt[0], abt[1], abt[2], abt[3], bo[2], bo[3]);
            }
          }
        }

        if (more) gather_store((s + 1) % 3, wd, m);
        if (tid < kKvQ && s + 2 < nsteps) meta[s & 1][tid] = next;
        cp_async_wait_all();
        __syncthreads();
      }
    }
    // write this warp's key row: keys g, g+8 of the block; n-tile j col c -> dim half*HALF + 8j + c
    if (myk < g.Hp) {
#pragma unroll
      for (int hf = 0; hf < 2; hf++) {
        const int x = x_lo + gq + 8 * hf;
        if (x >= g.Wp) continue;
        const int64_t tokk = ((int64_t)tk * g.Hp + myk) * g.Wp + x;
        __nv_bfloat16* dkr = dk + (tokk * g.heads + h) * DH + half * HALF;
        __nv_bfloat16* dvr = dv + (tokk * g.heads + h) * DH + half * HALF;
#pragma unroll
        for (int j = 0; j < NTH; j++) {
          *reinterpret_cast<__nv_bfloat162*>(dkr + 8 * j + 2 * qq) =
              __floats2bfloat162_rn(ak[j][2 * hf] * g.scale, ak[j][2 * hf + 1] * g.scale);
          *reinterpret_cast<__nv_bfloat162*>(dvr + 8 * j + 2 * qq) =
              __floats2bfloat162_rn(av[j][2 * hf], av[j][2 * hf + 1]);
        }
      }
    }
  }
}

}  // namespace dsa3d
