// dsa3d_fwd_mma.cuh -- 3D-DSA forward on tensor cores (bf16 I/O, dh 64 or 128, k_w <= 15).
//
// Input: queries sorted by box origin (dsa3d_sort.cuh).  One warp pair takes one bucket row (all
// queries sharing the origin's t and y) and cuts it into chunks of at most 16 queries whose
// x-origins differ by at most chunk_span(kw) = 30 - kw.  For a chunk, box row (bt, by) of every
// query lies in key row (o_t + bt, o_y + by) inside the 32-key segment [X0, X0 + 32), X0 = the
// chunk's smallest x-origin (and inside the 32 keys from the even key at or below X0, which the
// value products use).  Per tap plane u and box row by:
//   S_t  = (1-f_t) * Q.K[u, by]^T + f_t * Q.K[u+1, by]^T        (m16n8k16 MMAs, fp32 blend)
//   taps of row ty = by-1:  s = x-lerp(y-lerp(S_t[by-1], S_t[by]))  masked per query
//   online softmax (base 2) over the taps, P = exp2(s - m)
//   value weights of box row ty: beta = y-mix of the x-transposed P of tap rows ty and ty-1
//   O += [(1-f_t) beta | f_t beta] . [V[u, ty]; V[u+1, ty]]     (MMAs, beta as bf16 A operand)
// The pair is warp-specialised (see dsa3d_fwd_mma_kernel): the scores warp writes the blended
// raw scores of each box row to a two-row ring in shared memory, and two of its lanes per query
// evaluate only that query's taps (online softmax per query); the taps' P go through a tap ring
// to the values warp, which writes the value weights of the box row as two bf16 tiles (scaled by
// 1-f_t and f_t) that ldmatrix turns back into A operands of the P.V MMAs.  Only rows of valid
// queries exist here (the sort drops the rest).
//
// Operand layouts.  S = Q.K^T contracts dh: in k-step s, lane quad position q supplies words 2s
// and 2s+1 of its dim slice (qk_off), for the Q rows (A) and the key rows (B) alike -- any fixed
// permutation of dh applied to both operands leaves the dot products unchanged.  O = P.V reads
// the value rows in key pairs (dsa3d_pair_v_kernel) and maps output column n of n-tile j to dim
// 32 (j / 4) + 4n + j % 4 (pv_word), so lane (g, q) owns output dims 32c + 8q + [0, 8).
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

__device__ __forceinline__ uint4 ldg16(const void* p) { return __ldg(reinterpret_cast<const uint4*>(p)); }

// Largest difference of x-origins within a chunk: box columns ox - X0 + [0, kw] then stay below
// 31, so they fit the 32-key segment from X0 and, shifted by X0's parity, the one from the even key
// below it.  segment_keys(kw) = keys of the segment any box column can reach.
__host__ __device__ constexpr int chunk_span(int kw) { return 30 - kw; }
__host__ __device__ constexpr int segment_keys(int kw) { return chunk_span(kw) + kw + 1; }

// Per-row state of a chunk (rows g and g+8 of the lane).
struct MmaRow {
  bool live;        // row holds a query
  int n;            // token
  int ox;           // x-origin minus X0, in [0, chunk_span(kw)]
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

// Dim slices of the Q.K^T operands, chosen so that one 16-byte load instruction of a warp
// touches as few cache lines as possible: quad position q holds dims {32c + 8q + [0, 8)},
// c < DH/32 (the four q lanes of a key read one contiguous 64-byte span per instruction).
__device__ __forceinline__ int qk_off(int c, int qq) { return 32 * c + 8 * qq; }

__device__ __forceinline__ unsigned short bf16_bits(float x) {
  const __nv_bfloat16 b = __float2bfloat16_rn(x);
  return *reinterpret_cast<const unsigned short*>(&b);
}

// two floats as packed bf16 (round to nearest even), x in the low half
__device__ __forceinline__ unsigned bf16x2_bits(float x, float y) {
  const __nv_bfloat162 b = __floats2bfloat162_rn(x, y);
  return *reinterpret_cast<const unsigned*>(&b);
}

__device__ __forceinline__ void ldsm_x4(unsigned (&r)[4], const void* p) {
  const unsigned a = (unsigned)__cvta_generic_to_shared(p);
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(a));
}

__device__ __forceinline__ void ldsm_x4_trans(unsigned (&r)[4], const void* p) {
  const unsigned a = (unsigned)__cvta_generic_to_shared(p);
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(a));
}

// 16-byte asynchronous global -> shared copy; copies zeros instead when !valid (src is not read).
__device__ __forceinline__ void cp_async16_zfill(void* dst, const void* src, bool valid) {
  const unsigned d = (unsigned)__cvta_generic_to_shared(dst);
  const int n = valid ? 16 : 0;
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(d), "l"(src), "r"(n) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;\n" ::: "memory"); }
// wait until at most the most recent commit group is still in flight
__device__ __forceinline__ void cp_async_wait_group1() { asm volatile("cp.async.wait_group 1;\n" ::: "memory"); }

// Paired value rows.  The P.V products take V as the B operand with the keys as the contraction
// dimension, so each B register holds two consecutive keys of one dim.  The forward first copies
// the value rows of its head group into that form:
//   vp[((t * Hp + y) * Wp2 + xp) * hg + hh][d] = (V[(t, y, 2xp)][h0 + hh][d], V[(t, y, 2xp + 1)][..][d])
// as bf16 pairs (32-bit words), Wp2 = ceil(Wp / 2), zero where 2xp + 1 == Wp.  One thread moves
// 8 dims of one pair of keys: two 16-byte loads, two 16-byte stores.
template <int DH>
__global__ void dsa3d_pair_v_kernel(const __nv_bfloat16* __restrict__ v, unsigned* __restrict__ vp,
                                    const Geo g, const int Wp2, const int h0, const int hg) {
  constexpr int CH = DH / 8;
  const int64_t items = (int64_t)g.F * g.Hp * Wp2 * hg * CH;
  for (int64_t it = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; it < items;
       it += (int64_t)gridDim.x * blockDim.x) {
    const int c = (int)(it % CH);
    int64_t r = it / CH;
    const int hh = (int)(r % hg);
    r /= hg;
    const int xp = (int)(r % Wp2);
    const int64_t ty = r / Wp2;  // t * Hp + y
    const int64_t n0 = ty * g.Wp + 2 * xp;
    const uint4 a = ldg16(v + (n0 * g.heads + h0 + hh) * DH + 8 * c);
    const uint4 b = (2 * xp + 1 < g.Wp) ? ldg16(v + ((n0 + 1) * g.heads + h0 + hh) * DH + 8 * c)
                                        : make_uint4(0, 0, 0, 0);
    uint4 lo, hi;
    lo.x = __byte_perm(a.x, b.x, 0x5410); lo.y = __byte_perm(a.x, b.x, 0x7632);
    lo.z = __byte_perm(a.y, b.y, 0x5410); lo.w = __byte_perm(a.y, b.y, 0x7632);
    hi.x = __byte_perm(a.z, b.z, 0x5410); hi.y = __byte_perm(a.z, b.z, 0x7632);
    hi.z = __byte_perm(a.w, b.w, 0x5410); hi.w = __byte_perm(a.w, b.w, 0x7632);
    uint4* dst = reinterpret_cast<uint4*>(vp + (r * hg + hh) * DH + 8 * c);
    dst[0] = lo;
    dst[1] = hi;
  }
}

// P.V n-tile j, column n <-> dim 32 (j / 4) + 4 n + j % 4: lane group g then reads words
// 32c + 4g + [0, 4) of a paired row (eight lanes cover 128 contiguous bytes per instruction), and
// lane (g, q) owns output dims 32c + 8q + [0, 8).
__device__ __forceinline__ int pv_word(int c, int gq) { return 32 * c + 4 * gq; }

// O += tile0 . V[t0, y, seg] + tile1 . V[t0+1, y, seg]: the two bf16 value-weight tiles
// (16 queries x 32 segment keys from the even key X0e, row stride 40) as A operands (ldmatrix),
// the paired value rows as B operands (one 16-byte load per four n-tiles).
template <int DH>
__device__ __forceinline__ void dsa3d_pv_tile(float (&o)[MmaShape<DH>::NT][4], const unsigned short* tile,
                                              int t0, int y, int X0e, const unsigned* vph, int Wp2,
                                              int hg, const Geo& g, int lane) {
  using S = MmaShape<DH>;
  const int gq = lane >> 2, qq = lane & 3;
  if (y < 0 || y >= g.Hp) return;
  const int64_t prs = (int64_t)hg * DH;  // words per pair of keys
#pragma unroll
  for (int pl = 0; pl < 2; pl++) {
    const int t = t0 + pl;
    if (t < 0 || t >= g.F) continue;
    const unsigned* rowp = vph + (int64_t)(t * g.Hp + y) * Wp2 * prs;
#pragma unroll
    for (int kk = 0; kk < 2; kk++) {
      unsigned a[4];
      const int rr = (lane & 7) + 8 * ((lane >> 3) & 1), cc = 8 * (lane >> 4) + 16 * kk;
      ldsm_x4(a, tile + (pl * 16 + rr) * 40 + cc);
      unsigned vw[2][S::NT];  // [keys 2q, 2q+1 | keys 2q+8, 2q+9][n-tile]
#pragma unroll
      for (int hb = 0; hb < 2; hb++) {
        const int xp = (X0e >> 1) + 8 * kk + qq + 4 * hb;
        const bool ok = xp >= 0 && xp < Wp2;
        const unsigned* src = rowp + (int64_t)max(xp, 0) * prs;
#pragma unroll
        for (int c = 0; c < DH / 32; c++) {
          const uint4 w = ok ? ldg16(src + pv_word(c, gq)) : make_uint4(0, 0, 0, 0);
          vw[hb][4 * c] = w.x; vw[hb][4 * c + 1] = w.y; vw[hb][4 * c + 2] = w.z; vw[hb][4 * c + 3] = w.w;
        }
      }
#pragma unroll
      for (int j = 0; j < S::NT; j++) mma_bf16_16816(o[j], a[0], a[1], a[2], a[3], vw[0][j], vw[1][j]);
    }
  }
}

// Shared memory of one warp pair of the forward (scores warp S, values warp P):
//   S only:  raw-score ring [2][16][kFwdRaw]; raw scores of box plane u+1 of the first
//            kFwdCacheRows box rows in fragment order [row][16 values][32 lanes] (computed for tap
//            plane u and reused as the lower plane of tap plane u+1, so those rows' Q.K^T runs
//            once per box plane; rows beyond the cache recompute)
//   shared:  tap ring [kFwdSlots][16 rows][kFwdTap] of P, each slot followed by 16 floats: the
//            rows' rescale factors of that tap row, or, in a chunk's last entry, the row sums
//   P only:  two bf16 value-weight tiles [2][16][kFwdTile]
constexpr int kFwdRaw = 40;   // conflict-free float2 stores of MMA fragments
constexpr int kFwdTap = 18;   // kw <= 15; 18 keeps the two lanes per query row on distinct banks
constexpr int kFwdTile = 40;  // bf16 per row: 32 columns + pad (conflict-free ldmatrix)
#ifndef DSA3D_FWD_CACHE_ROWS
#define DSA3D_FWD_CACHE_ROWS 10
#endif
#ifndef DSA3D_FWD_SLOTS
#define DSA3D_FWD_SLOTS 4
#endif
constexpr int kFwdCacheRows = DSA3D_FWD_CACHE_ROWS;
constexpr int kFwdSlots = DSA3D_FWD_SLOTS;  // tap-ring entries: P holds two (tap rows ty-1, ty)
static_assert(kFwdSlots >= 3 && 2 * 2 * kFwdSlots <= 16, "two pairs' full and empty barriers fit the 16 ids");
constexpr int kFwdSlotFloats = 16 * kFwdTap + 16;
__host__ __device__ constexpr int fwd_pair_bytes() {
  return (2 * 16 * kFwdRaw + kFwdCacheRows * 16 * 32 + kFwdSlots * kFwdSlotFloats) * 4 +
         2 * 16 * kFwdTile * 2;
}

__device__ __forceinline__ void named_sync(unsigned id) { asm volatile("bar.sync %0, 64;\n" ::"r"(id) : "memory"); }
__device__ __forceinline__ void named_arrive(unsigned id) {
  __threadfence_block();
  asm volatile("bar.arrive %0, 64;\n" ::"r"(id) : "memory");
}

// Two warps per chunk, specialised.  The scores warp S computes the t-blended raw scores of each
// box row (Q.K^T on tensor cores, the plane cache above), then the taps of the previous tap row:
// y/x blends, the online softmax (base 2) and P, which it hands to the values warp P through the
// tap ring together with the rows' rescale factors.  P rescales O, forms the value weights of the
// box row (x-splat of the tap row, y-mix with the previous one scaled by the factor) as two bf16
// tiles and adds [(1-f_t) beta | f_t beta] . [V[u, ty]; V[u+1, ty]] on tensor cores.  Ring entry n
// lives in slot n % kFwdSlots; named barriers full[s] (S arrives, P waits) and empty[s] (P
// arrives, S waits) order them.  Both warps walk the same chunks and skip the same planes.
// RUN: the longest run of taps a lane of the scores warp evaluates, ceil(kw / 2) <= RUN
template <int DH, int RUN>
__global__ void __launch_bounds__(128, DSA3D_MMA_MINB)
    dsa3d_fwd_mma_kernel(const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k,
                         const __nv_bfloat16* __restrict__ v, const float* __restrict__ off,
                         __nv_bfloat16* __restrict__ out, float* __restrict__ lse,
                         const int* __restrict__ start, const int* __restrict__ sorted_n,
                         const int* __restrict__ sorted_ex, const unsigned* __restrict__ vp,
                         const int Wp2, const Geo g, const SortGeo sg, const int h0, const int hg) {
  using S = MmaShape<DH>;
  extern __shared__ __align__(16) unsigned char fwd_sh[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int pair = warp >> 1, role = warp & 1;  // role 0: scores warp, role 1: values warp
  const int gq = lane >> 2, qq = lane & 3;      // fragment row group / quad position
  float* raw = reinterpret_cast<float*>(fwd_sh + pair * fwd_pair_bytes());
  float* scache = raw + 2 * 16 * kFwdRaw;
  float* ring = scache + kFwdCacheRows * 16 * 32;
  unsigned short* tile = reinterpret_cast<unsigned short*>(ring + kFwdSlots * kFwdSlotFloats);
  // named barrier ids (this kernel uses no __syncthreads, so id 0 is free when 16 ids are needed)
  const unsigned full0 = (2 * 2 * kFwdSlots < 16 ? 1 : 0) + 2 * kFwdSlots * pair, empty0 = full0 + kFwdSlots;
  const int er = lane >> 1, side = lane & 1;  // epilogue / tile rows: query row, tap parity
  const int64_t rs = (int64_t)g.heads * DH;
  const float sc = g.scale * kLog2e;
  const int segw = segment_keys(g.kw);
  const int64_t rows = (int64_t)hg * sg.Et * sg.Ey;
  int n = 0;  // tap-ring entries of this pair so far

  for (int64_t row = (int64_t)blockIdx.x * 2 + pair; row < rows; row += (int64_t)gridDim.x * 2) {
    const int hh = (int)(row / ((int64_t)sg.Et * sg.Ey));
    const int rem = (int)(row - (int64_t)hh * sg.Et * sg.Ey);
    const int et = rem / sg.Ey, ey = rem % sg.Ey;
    const int h = h0 + hh;
    const int64_t b0 = (int64_t)hh * sg.E1 + ((int64_t)et * sg.Ey + ey) * sg.Ex;
    const int qbeg = start[b0], qend = start[b0 + sg.Ex];
    const int ot = et - g.kt, oy = ey - g.kh;

    for (int pos = qbeg; pos < qend;) {
      // ---- chunk: <= 16 consecutive queries whose x-origins differ by <= chunk_span(kw)
      const int ex_l = (lane < 16 && pos + lane < qend) ? sorted_ex[pos + lane] : 0x7fffffff;
      const int ex0 = __shfl_sync(kFull, ex_l, 0);
      const unsigned bal =
          __ballot_sync(kFull, lane < 16 && pos + lane < qend && ex_l - ex0 <= chunk_span(g.kw));
      const int cnt = __popc(bal);
      const int X0 = ex0 - g.kw;

      // fragment rows g, g+8: token, f_t and tap-plane range (the same in both warps)
      int fn[2];
      float fft[2];
      bool flive[2];
      int flo_t[2], fhi_t[2];
#pragma unroll
      for (int hf = 0; hf < 2; hf++) {
        const int r = gq + 8 * hf;
        flive[hf] = r < cnt;
        fn[hf] = flive[hf] ? sorted_n[pos + r] : 0;
        const Query Fq = decode_query(g, off, h, fn[hf]);
        fft[hf] = flive[hf] ? Fq.f[0] : 0.f;
        flo_t[hf] = Fq.lo[0];
        fhi_t[hf] = flive[hf] ? Fq.hi[0] : -1;
      }
      // epilogue / tile row er
      const bool elive = er < cnt;
      const int en = elive ? sorted_n[pos + er] : 0;
      const Query EQ = decode_query(g, off, h, en);
      DSA3D_DEVICE_CHECK(!elive || (EQ.ok && EQ.o[0] == ot && EQ.o[1] == oy && EQ.o[2] - X0 >= 0 && EQ.o[2] - X0 <= chunk_span(g.kw)));
      const int eox = EQ.o[2] - X0;
      const float eft = EQ.f[0], efy = EQ.f[1], efx = EQ.f[2];

      if (role == 0) {
        // ================= scores warp =================
        const __nv_bfloat16* kh_ = k + (int64_t)h * DH;
        unsigned qa[S::KS][4];
        {
          unsigned w0[S::QW], w1[S::QW];
#pragma unroll
          for (int c = 0; c < S::QW / 4; c++) {
            uint4 a = make_uint4(0, 0, 0, 0), b = make_uint4(0, 0, 0, 0);
            if (flive[0]) a = ldg16(q + ((int64_t)fn[0] * g.heads + h) * DH + qk_off(c, qq));
            if (flive[1]) b = ldg16(q + ((int64_t)fn[1] * g.heads + h) * DH + qk_off(c, qq));
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
        const int hi_t = elive ? EQ.hi[0] : -1;
        float m = -INFINITY, l = 0.f;  // running max (base 2) and partial sum of row er
        int cached_plane = -1;         // box plane whose raw scores scache holds
        for (int u = 0; u < g.kt; u++) {
          const bool fpl = (flo_t[0] <= u && u <= fhi_t[0]) || (flo_t[1] <= u && u <= fhi_t[1]);
          if (!__any_sync(kFull, fpl)) continue;
          const bool eplane = EQ.lo[0] <= u && u <= hi_t;
          const bool have_u = cached_plane == u;
          for (int by = 0; by <= g.kh; by++) {
            const int y = oy + by;
            float* rc = raw + (by & 1) * 16 * kFwdRaw;
            const bool cache_row = by < kFwdCacheRows;
            float* cr = scache + (cache_row ? by : 0) * 16 * 32 + lane;  // + 32 * (4 * jt + e)
            // t-blended raw scores of box row by -> ring; raw scores of plane u+1 -> cache
            {
              float st[4][4];
#pragma unroll
              for (int jt = 0; jt < 4; jt++) st[jt][0] = st[jt][1] = st[jt][2] = st[jt][3] = 0.f;
#pragma unroll
              for (int pl = 0; pl < 2; pl++) {
                const int t = ot + u + pl;
                if (pl == 0 && have_u && cache_row) {  // plane u was computed for tap plane u-1
#pragma unroll
                  for (int jt = 0; jt < 4; jt++)
#pragma unroll
                    for (int e = 0; e < 4; e++) st[jt][e] = (1.f - fft[e >> 1]) * cr[32 * (4 * jt + e)];
                  continue;
                }
                if (t < 0 || t >= g.F || y < 0 || y >= g.Hp) {
                  if (pl == 1 && cache_row) {
#pragma unroll
                    for (int i = 0; i < 16; i++) cr[32 * i] = 0.f;
                  }
                  continue;
                }
#pragma unroll
                for (int jt = 0; jt < 4; jt++) {
                  const int col = 8 * jt + gq;
                  const int x = X0 + col;
                  const bool ok = col < segw && x >= 0 && x < g.Wp;
                  const __nv_bfloat16* kr = kh_ + ((int64_t)(t * g.Hp + y) * g.Wp + max(x, 0)) * rs;
                  unsigned kw_[S::QW];
#pragma unroll
                  for (int c = 0; c < S::QW / 4; c++) {
                    const uint4 a = ok ? ldg16(kr + qk_off(c, qq)) : make_uint4(0, 0, 0, 0);
                    kw_[4 * c] = a.x; kw_[4 * c + 1] = a.y; kw_[4 * c + 2] = a.z; kw_[4 * c + 3] = a.w;
                  }
                  float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                  for (int s = 0; s < S::KS; s++)
                    mma_bf16_16816(acc, qa[s][0], qa[s][1], qa[s][2], qa[s][3], kw_[2 * s], kw_[2 * s + 1]);
#pragma unroll
                  for (int e = 0; e < 4; e++) {
                    const float w = pl ? fft[e >> 1] : 1.f - fft[e >> 1];
                    st[jt][e] = fmaf(w, acc[e], st[jt][e]);
                    if (pl == 1 && cache_row) cr[32 * (4 * jt + e)] = acc[e];
                  }
                }
              }
#pragma unroll
              for (int jt = 0; jt < 4; jt++)
#pragma unroll
                for (int hf = 0; hf < 2; hf++)
                  *reinterpret_cast<float2*>(rc + (gq + 8 * hf) * kFwdRaw + 8 * jt + 2 * qq) =
                      make_float2(st[jt][2 * hf], st[jt][2 * hf + 1]);
            }
            __syncwarp();
            if (by >= 1) {
              const int ty = by - 1;
              const float* rp = raw + ((by - 1) & 1) * 16 * kFwdRaw;
              const int slot = n % kFwdSlots;
              if (n >= kFwdSlots) named_sync(empty0 + slot);  // P is done with entry n - slots
              float* tp = ring + slot * kFwdSlotFloats;
              const bool erow = eplane && EQ.lo[1] <= ty && ty <= EQ.hi[1];
              // scores of this lane's taps, a run [t0, t1) of the tap row (tap wx blends columns
              // wx and wx+1, so each column is read and y-blended once), and the row max
              const int t0 = side ? (g.kw + 1) >> 1 : 0, t1 = side ? g.kw : (g.kw + 1) >> 1;
              float sv[RUN];
              float mx = -INFINITY;
              float Yp;
              {
                const int c = er * kFwdRaw + eox + t0;
                Yp = fmaf(efy, rc[c] - rp[c], rp[c]);
              }
#pragma unroll
              for (int i = 0; i < RUN; i++) {
                const int wx = t0 + i;
                sv[i] = -INFINITY;
                if (wx < t1) {
                  const int c = er * kFwdRaw + eox + wx + 1;
                  const float Y = fmaf(efy, rc[c] - rp[c], rp[c]);
                  if (erow && wx >= EQ.lo[2] && wx <= EQ.hi[2]) {
                    sv[i] = fmaf(efx, Y - Yp, Yp) * sc;
                    mx = fmaxf(mx, sv[i]);
                  }
                  Yp = Y;
                }
              }
              mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 1));
              float alpha = 1.f;
              if (mx > m) {
                alpha = exp2f(m - mx);  // 0 when m was -inf
                m = mx;
              }
              float ls = 0.f;
#pragma unroll
              for (int i = 0; i < RUN; i++) {
                const int wx = t0 + i;
                if (wx < t1) {
                  const float p = (sv[i] == -INFINITY) ? 0.f : exp2f(sv[i] - m);
                  tp[er * kFwdTap + wx] = p;
                  ls += p;
                }
              }
              l = fmaf(l, alpha, ls);
              if (side == 0) tp[16 * kFwdTap + er] = alpha;
              __syncwarp();
              named_arrive(full0 + slot);
              n++;
            }
          }
          cached_plane = u + 1;
        }
        // the chunk's last entry: row sums (and lse)
        const float lt_e = l + __shfl_xor_sync(kFull, l, 1);
        if (elive && side == 0 && lse) lse[(int64_t)h * g.N + en] = (m + log2f(lt_e)) * kLn2;
        const int slot = n % kFwdSlots;
        if (n >= kFwdSlots) named_sync(empty0 + slot);
        if (side == 0) ring[slot * kFwdSlotFloats + 16 * kFwdTap + er] = lt_e;
        __syncwarp();
        named_arrive(full0 + slot);
        n++;
      } else {
        // ================= values warp =================
        const unsigned* vph = vp + (int64_t)hh * DH;
        const int X0e = X0 - (X0 & 1);  // even start of the value segment (covers [X0, X0 + 16 + kw))
        const int vcol = X0 - X0e + eox;  // value-tile column of box column 0 of row er
        float o[S::NT][4];
#pragma unroll
        for (int j = 0; j < S::NT; j++) o[j][0] = o[j][1] = o[j][2] = o[j][3] = 0.f;
        for (int u = 0; u < g.kt; u++) {
          const bool fpl = (flo_t[0] <= u && u <= fhi_t[0]) || (flo_t[1] <= u && u <= fhi_t[1]);
          if (!__any_sync(kFull, fpl)) continue;
          for (int ty = 0; ty <= g.kh; ty++) {
            // box row ty: tap rows ty (entry n, none for ty == kh) and ty-1 (entry n-1, none for ty == 0)
            const bool has_cur = ty < g.kh;
            const float* tp = ring + (n % kFwdSlots) * kFwdSlotFloats;
            const float* tq = ring + ((n + kFwdSlots - 1) % kFwdSlots) * kFwdSlotFloats;
            float a_er = 1.f;
            if (has_cur) {
              named_sync(full0 + n % kFwdSlots);
              // O rows g, g+8 rescale by the tap row's factors
              const float a0 = tp[16 * kFwdTap + gq], a1 = tp[16 * kFwdTap + gq + 8];
              if (__any_sync(kFull, a0 != 1.f || a1 != 1.f)) {
#pragma unroll
                for (int j = 0; j < S::NT; j++) {
                  o[j][0] *= a0; o[j][1] *= a0;
                  o[j][2] *= a1; o[j][3] *= a1;
                }
              }
              a_er = tp[16 * kFwdTap + er];
            }
            // value weights of box row ty, scaled for box planes u (1 - f_t) and u+1 (f_t)
            for (int i = lane; i < 2 * 16 * kFwdTile / 8; i += 32)
              reinterpret_cast<uint4*>(tile)[i] = make_uint4(0, 0, 0, 0);
            __syncwarp();
            if (elive) {
              // this lane's run [b0, b1) of the kw + 1 box columns; column bx takes taps bx and
              // bx-1 of each tap row, so tap values roll from one column to the next
              const int hb = (g.kw + 2) >> 1;
              const int b0 = side ? hb : 0, b1 = side ? g.kw + 1 : hb;
              const bool prev_in = b0 >= 1;
              float pq = (has_cur && prev_in) ? tp[er * kFwdTap + b0 - 1] : 0.f;
              float pr = (ty >= 1 && prev_in) ? tq[er * kFwdTap + b0 - 1] : 0.f;
              for (int bx = b0; bx < b1; bx++) {
                const bool in = bx < g.kw;
                const float cq = (has_cur && in) ? tp[er * kFwdTap + bx] : 0.f;
                const float cr = (ty >= 1 && in) ? tq[er * kFwdTap + bx] : 0.f;
                const float bxc = fmaf(efx, pq - cq, cq);
                const float bxp = a_er * fmaf(efx, pr - cr, cr);
                const float beta = fmaf(efy, bxp - bxc, bxc);
                tile[er * kFwdTile + vcol + bx] = bf16_bits((1.f - eft) * beta);
                tile[(16 + er) * kFwdTile + vcol + bx] = bf16_bits(eft * beta);
                pq = cq;
                pr = cr;
              }
            }
            __syncwarp();
            if (ty >= 1) named_arrive(empty0 + (n + kFwdSlots - 1) % kFwdSlots);  // tap row ty-1 done
            if (has_cur) n++;
            dsa3d_pv_tile<DH>(o, tile, ot + u, oy + ty, X0e, vph, Wp2, hg, g, lane);
            __syncwarp();
          }
        }
        // the chunk's last entry: row sums; normalise and store
        const int slot = n % kFwdSlots;
        named_sync(full0 + slot);
        const float* lsum = ring + slot * kFwdSlotFloats + 16 * kFwdTap;
#pragma unroll
        for (int hf = 0; hf < 2; hf++) {
          if (!flive[hf]) continue;
          const float inv = 1.f / lsum[gq + 8 * hf];
          __nv_bfloat16* orow = out + ((int64_t)fn[hf] * g.heads + h) * DH;
#pragma unroll
          for (int c = 0; c < DH / 32; c++) {
            float vals[8];  // dims 32c + 8q + [0, 8): column 2q then 2q+1 of n-tiles 4c..4c+3
#pragma unroll
            for (int i = 0; i < 4; i++) {
              vals[i] = o[4 * c + i][2 * hf] * inv;
              vals[4 + i] = o[4 * c + i][2 * hf + 1] * inv;
            }
            store16(orow + 32 * c + 8 * qq, vals);
          }
        }
        __syncwarp();
        named_arrive(empty0 + slot);
        n++;
      }
      pos += cnt;
    }
  }
  // the scores warp takes the values warp's last releases, so every barrier phase completes
  if (role == 0)
    for (int m = max(0, n - kFwdSlots); m < n; m++) named_sync(empty0 + m % kFwdSlots);
}

}  // namespace dsa3d
