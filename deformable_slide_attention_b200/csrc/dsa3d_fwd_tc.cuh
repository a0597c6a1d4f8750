// dsa3d_fwd_tc.cuh -- 3D-DSA forward on the 5th-generation tensor cores (tcgen05 UMMA with
// operands and accumulators in tensor memory, K/V tiles by TMA), bf16 I/O, dh 64 or 128,
// k_w <= 15.
//
// Work unit: a tile of the window-origin sort (dsa3d_sort.cuh) -- the queries of one head whose
// extended origins e = o + k share e_t, have e_y in [Y0, Y0 + Ry) and e_x in [X0, X0 + Wx),
// Wx = 32 - k_w.  Their boxes (MegaSlide-DiT, arXiv 2607.22696, 3D-DSA definition: the 8
// trilinear corners of all taps of a query fall on one integer box of (k_t+1)(k_h+1)(k_w+1)
// tokens) all lie inside the box planes o_t .. o_t + k_t, the U = k_h + Ry "union rows"
// Y0 - k_h .. Y0 + Ry - 1 and the 32-key segment X0 - k_w .. X0 - k_w + 31.  Up to 128 queries
// of a tile are processed at once, one per tensor-memory lane (more: further passes).
//
// For tap plane u and union row j (box planes u, u+1 of the tile's planes): the raw box dots
//   D[q][p * 32 + c] = q . K[o_t + u + p, row j, key c]     (p = 0, 1; c < 32)
// are one UMMA chain (M = 128 queries, N = 64 keys of the two planes, K = dh) with the query rows
// in tensor memory (A) and the K "pair" of the row in shared memory (B, loaded by TMA), into an
// fp32 accumulator in tensor memory.  The epilogue thread of query q (thread = tensor-memory lane)
// reads its row, blends along t (1 - f_t, f_t) and along y with the previous row (tap row j-1 of
// the union uses rows j-1 and j), blends along x (tap column c uses keys c and c+1 with 1 - f_x,
// f_x), masks the taps outside the query's valid range, and runs an online softmax in base 2 --
// the oracle's arithmetic on the same bf16 inputs, in fp32.  The value weights of box row j-1
// (x-splat of the tap row's P, y-mix with the previous tap row's) scaled by 1 - f_t and f_t
// become the A operand (bf16, tensor memory) of O += [beta_a | beta_b] . [V[u, j-1]; V[u+1, j-1]]
// (K = 64 keys, N = dh; O in tensor memory).  The running max is raised lazily: O is rescaled
// only when a tap row's max exceeds the max in use by more than 2^8 (exact either way: P and O
// share the max in use).  At the end of a pass each thread divides its row of O by the softmax
// sum and writes out and lse.
//
// Roles (256 threads): warps 0-3 the epilogue (tensor-memory lane quarter w), warps 4 and 6 the TMA
// producers of K and of V, warp 5 the UMMA issuer of the raw dots (the warp also allocates tensor
// memory), warp 7 the UMMA issuer of the value products (one lane each).
// Rings of shared-memory stages hold K and V "pairs" (one union row, two planes, 32 keys, dh):
// per 64 dims, a 5-D box (64 dims, 1 head half, 32 keys, 1 row, 2 planes) of the tensor map over
// [T][H'][W'][heads * dh / 64][64] with the 128-byte swizzle, so each half is 64 rows (plane-major
// keys) of 128 bytes -- the layout the UMMA reads as K-major B (keys = N) for the dots and as
// MN-major B (dims = N, keys = K) for P.V.  Out-of-volume keys, rows and planes read as zero.
// mbarriers order everything; every wait is bounded (dsa3d_tc.cuh).
#pragma once

#include "dsa3d_bwd_mma.cuh"  // bf16 helpers
#include "dsa3d_sort.cuh"
#include "dsa3d_tc.cuh"

namespace dsa3d {

constexpr int kTcThreads = 256;  // 4 epilogue warps, K producer, dots issuer, V producer, P.V issuer
constexpr int kTcKWarp = 4, kTcMmaWarp = 5, kTcVWarp = 6, kTcPvWarp = 7;
constexpr int kTcSeg = 32;         // keys per segment
constexpr int kTcRyMax = 8;        // bucket rows per tile (Ry <= kTcRyMax)
constexpr int kTcKStages = 4;      // K pair ring
constexpr int kTcVStages = 3;      // V pair ring
constexpr float kTcRescale = 8.f;  // lazy-rescale threshold (base-2 units)

template <int DH>
struct FwdTcCfg {
  static constexpr int HALVES = DH / 64;                  // 128-byte row halves of a key
  static constexpr int PAIR_BYTES = 2 * kTcSeg * DH * 2;  // two planes x 32 keys x dh bf16
  static constexpr int KSTEPS = DH / 16;                  // UMMA K-steps of S
  static constexpr int A_COLS = DH / 2;                   // the query tile (bf16 pairs)
  static constexpr int COL_A = 0;
  static constexpr int COL_S = A_COLS;                    // 2 raw-dot buffers x 64 fp32 columns
  static constexpr int COL_P = COL_S + 128;               // 2 value-weight buffers x 32 columns
  static constexpr int COL_O = COL_P + 64;                // O: dh fp32 columns
  static constexpr int COLS = 512;                        // allocation (power of two >= COL_O + DH)
  static_assert(COL_O + DH <= COLS, "tensor memory budget");
  static constexpr int STAGE_BYTES = (kTcKStages + kTcVStages) * PAIR_BYTES;
  static constexpr int BAR_BYTES = 256;
  // at least 116 KB so that one CTA (and its 512 tensor-memory columns) owns an SM
  static constexpr int SMEM_BYTES =
      (STAGE_BYTES + BAR_BYTES + 1024 > 118784) ? STAGE_BYTES + BAR_BYTES + 1024 : 118784;
  static constexpr uint32_t IDESC_S = umma_idesc_bf16(128, 2 * kTcSeg, false, false);
  static constexpr uint32_t IDESC_PV = umma_idesc_bf16(128, DH, false, true);
};

// Tile geometry shared by the three roles (all derive it from the same global data).
struct TcTileGeo {
  int Ry, Wx, nYb, nXb;
  int64_t tiles;
};

struct TcTile {
  int hh, et, Y0, X0;
  int cnt;                   // queries of the tile
  int r0[kTcRyMax], rn[kTcRyMax];  // sorted ranges of its bucket rows
};

__device__ __forceinline__ void tc_tile(const TcTileGeo& tg, const SortGeo& sg, const int* __restrict__ start,
                                        int64_t t, TcTile& T) {
  const int xb = (int)(t % tg.nXb);
  t /= tg.nXb;
  const int yb = (int)(t % tg.nYb);
  t /= tg.nYb;
  T.et = (int)(t % sg.Et);
  T.hh = (int)(t / sg.Et);
  T.Y0 = yb * tg.Ry;
  T.X0 = xb * tg.Wx;
  const int xe = min(T.X0 + tg.Wx, sg.Ex);
  T.cnt = 0;
#pragma unroll
  for (int i = 0; i < kTcRyMax; i++) {
    T.r0[i] = 0;
    T.rn[i] = 0;
    const int ey = T.Y0 + i;
    if (i < tg.Ry && ey < sg.Ey) {
      const int64_t b = (int64_t)T.hh * sg.E1 + ((int64_t)T.et * sg.Ey + ey) * sg.Ex;
      T.r0[i] = start[b + T.X0];
      T.rn[i] = start[b + xe] - T.r0[i];
      T.cnt += T.rn[i];
    }
  }
}

template <int DH>
__global__ void __launch_bounds__(kTcThreads, 1)
    dsa3d_fwd_tc_kernel(const __grid_constant__ CUtensorMap tmk, const __grid_constant__ CUtensorMap tmv,
                        const __nv_bfloat16* __restrict__ q, const float* __restrict__ off,
                        __nv_bfloat16* __restrict__ out, float* __restrict__ lse,
                        const int* __restrict__ start, const int* __restrict__ sorted_n,
                        const int* __restrict__ sorted_ex, const Geo g, const SortGeo sg,
                        const TcTileGeo tg, const int h0) {
  using C = FwdTcCfg<DH>;
  extern __shared__ __align__(1024) unsigned char tc_smem[];
  unsigned char* stages = tc_smem + ((1024 - (smem_u32(tc_smem) & 1023)) & 1023);
  const uint32_t kst = smem_u32(stages);
  const uint32_t vst = kst + kTcKStages * C::PAIR_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(stages + C::STAGE_BYTES);
  // barrier slots
  const uint32_t b0 = smem_u32(bars);
  auto k_full = [&](int s) { return b0 + 8u * s; };
  auto k_empty = [&](int s) { return b0 + 8u * (kTcKStages + s); };
  auto v_full = [&](int s) { return b0 + 8u * (2 * kTcKStages + s); };
  auto v_empty = [&](int s) { return b0 + 8u * (2 * kTcKStages + kTcVStages + s); };
  const uint32_t bx = b0 + 8u * (2 * kTcKStages + 2 * kTcVStages);
  auto s_full = [&](int s) { return bx + 8u * s; };
  auto s_empty = [&](int s) { return bx + 8u * (2 + s); };
  auto p_full = [&](int s) { return bx + 8u * (4 + s); };
  auto p_empty = [&](int s) { return bx + 8u * (6 + s); };
  const uint32_t a_full = bx + 8u * 8, o_full = bx + 8u * 9, o_empty = bx + 8u * 10;
  const uint32_t m_done = bx + 8u * 11, m_done2 = bx + 8u * 12;  // the UMMA issuers' own exit drains
  uint32_t* tslot = reinterpret_cast<uint32_t*>(stages + C::STAGE_BYTES + 8 * 32);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tslot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kTcKStages; s++) {
      mbar_init(k_full(s), 1);
      mbar_init(k_empty(s), 1);
    }
    for (int s = 0; s < kTcVStages; s++) {
      mbar_init(v_full(s), 1);
      mbar_init(v_empty(s), 1);
    }
    for (int s = 0; s < 2; s++) {
      mbar_init(s_full(s), 1);
      mbar_init(s_empty(s), 4);
      mbar_init(p_full(s), 4);
      mbar_init(p_empty(s), 1);
    }
    mbar_init(a_full, 4);
    mbar_init(o_full, 1);
    mbar_init(o_empty, 4);
    mbar_init(m_done, 1);
    mbar_init(m_done2, 1);
    *abort_flag = 0;
    mbar_fence_init();
  }
  if (warp == kTcMmaWarp) tmem_alloc(smem_u32(tslot), C::COLS);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tslot;
  const int U = g.kh + tg.Ry;  // union rows per tile

  if (warp == kTcKWarp || warp == kTcVWarp) {
    // ===================== TMA producers: K pairs (warp kTcKWarp) and V pairs (warp kTcVWarp) ==
    // Each ring has its own thread, so that neither waits behind the other's free slots.
    if (lane == 0) {
      const bool is_k = warp == kTcKWarp;
      const CUtensorMap* tm = is_k ? &tmk : &tmv;
      const int nst = is_k ? kTcKStages : kTcVStages;
      const uint32_t base = is_k ? kst : vst;
      tma_prefetch_desc(tm);
      uint32_t cnt = 0;
      bool ok = true;
      auto load = [&](int t0, int y, int X, int hd) {
        const int s = (int)(cnt % nst);
        const uint32_t full = is_k ? k_full(s) : v_full(s), empty = is_k ? k_empty(s) : v_empty(s);
        if (cnt >= (uint32_t)nst && !mbar_wait(empty, ((cnt / nst) - 1) & 1, abort_flag)) return false;
        mbar_arrive_expect_tx(full, C::PAIR_BYTES);
#pragma unroll
        for (int hv = 0; hv < C::HALVES; hv++)
          tma_load_5d(base + s * C::PAIR_BYTES + hv * (C::PAIR_BYTES / C::HALVES), tm, full, 0, hd + hv, X, y, t0);
        cnt++;
        return true;
      };
      for (int64_t t = blockIdx.x; t < tg.tiles && ok; t += gridDim.x) {
        TcTile T;
        tc_tile(tg, sg, start, t, T);
        const int passes = (T.cnt + 127) / 128;
        const int ot = T.et - g.kt, Xs = T.X0 - g.kw, hd = (h0 + T.hh) * C::HALVES;
        // per tap plane u: the pairs (planes u, u+1) of union rows 0 .. U-1, in the order of use
        for (int ps = 0; ps < passes && ok; ps++)
          for (int u = 0; u < g.kt && ok; u++)
            for (int j = 0; j < U && ok; j++) ok = load(ot + u, T.Y0 - g.kh + j, Xs, hd);
      }
      // every issued copy has landed before the CTA can exit (bounded; the last copy of each
      // stage completes its phase last)
      for (uint32_t i = (cnt > (uint32_t)nst ? cnt - nst : 0); i < cnt; i++)
        mbar_drain(is_k ? k_full(i % nst) : v_full(i % nst), (i / nst) & 1, abort_flag);
    }
  } else if (warp == kTcMmaWarp) {
    // ===================== UMMA issuer of the raw dots =====================
    // Raw dots of union row j, planes u and u+1 (K pair (u, j), released when done), into the
    // S buffer j % 2 once the epilogue has read the row two back.
    if (lane == 0) {
      uint32_t kc = 0, sc = 0, npass = 0;
      bool ok = true;
      const uint32_t tA = tmem + C::COL_A, tS = tmem + C::COL_S;
      const uint64_t kd0 = umma_sdesc_sw128(kst, 16, 1024);
      for (int64_t t = blockIdx.x; t < tg.tiles && ok; t += gridDim.x) {
        TcTile T;
        tc_tile(tg, sg, start, t, T);
        const int passes = (T.cnt + 127) / 128;
        for (int ps = 0; ps < passes && ok; ps++, npass++) {
          ok = mbar_wait(a_full, npass & 1, abort_flag);
          if (!ok) break;
          const int rows = g.kt * U;
          for (int r = 0; r < rows && ok; r++, kc++, sc++) {
            const int ks_ = (int)(kc % kTcKStages), sb = (int)(sc & 1);
            if (!mbar_wait(k_full(ks_), (kc / kTcKStages) & 1, abort_flag) ||
                (sc >= 2 && !mbar_wait(s_empty(sb), ((sc - 2) >> 1) & 1, abort_flag))) {
              ok = false;
              break;
            }
            tc_fence_after();
            // B, K-major: 64 keys (plane 0 then plane 1) = 64 rows of 128 bytes per 64-dim half;
            // dims 16 ks .. 16 ks + 15 are 32 bytes into the rows of half ks / 4.  The descriptors
            // differ only in their start address (bits 0-13, 16-byte units): constant adds.
            const uint64_t bd0 = kd0 + (uint64_t)((ks_ * C::PAIR_BYTES) >> 4);
            const uint32_t d = tS + sb * 64;
            umma_ts_c<false>(d, tA, bd0, C::IDESC_S);
#pragma unroll
            for (int ks = 1; ks < C::KSTEPS; ks++)
              umma_ts_c<true>(d, tA + ks * 8, bd0 + (uint64_t)(((ks >> 2) * (C::PAIR_BYTES / C::HALVES) + (ks & 3) * 32) >> 4),
                              C::IDESC_S);
            umma_commit(s_full(sb));
            umma_commit(k_empty(ks_));
          }
        }
      }
      // nothing of this thread's may still run when tensor memory is released
      umma_commit(m_done);
      mbar_drain(m_done, 0, abort_flag);
    }
  } else if (warp == kTcPvWarp) {
    // ===================== UMMA issuer of the value products =====================
    // O += [beta_a | beta_b] . [V[u, j]; V[u+1, j]] once the epilogue has written box row j's
    // weights; the first product of a pass overwrites O (after the epilogue read the previous
    // pass's), the last one signals o_full.
    if (lane == 0) {
      uint32_t vc = 0, pc = 0, npass = 0;
      bool ok = true;
      const uint32_t tP = tmem + C::COL_P, tO = tmem + C::COL_O;
      const uint64_t vd0 = umma_sdesc_sw128(vst, C::PAIR_BYTES / C::HALVES, 1024);
      for (int64_t t = blockIdx.x; t < tg.tiles && ok; t += gridDim.x) {
        TcTile T;
        tc_tile(tg, sg, start, t, T);
        const int passes = (T.cnt + 127) / 128;
        for (int ps = 0; ps < passes && ok; ps++, npass++) {
          const int rows = g.kt * U;
          for (int r = 0; r < rows && ok; r++, vc++, pc++) {
            const int pb = (int)(pc & 1), vs = (int)(vc % kTcVStages);
            if (!mbar_wait(p_full(pb), (pc >> 1) & 1, abort_flag)) { ok = false; break; }
            if (!mbar_wait(v_full(vs), (vc / kTcVStages) & 1, abort_flag) ||
                (r == 0 && npass > 0 && !mbar_wait(o_empty, (npass - 1) & 1, abort_flag))) {
              ok = false;
              break;
            }
            tc_fence_after();
            // B, MN-major: keys 16 ks .. 16 ks + 15 are rows 16 ks ..; 64-dim halves apart by
            // PAIR_BYTES / HALVES
            const uint64_t bd0 = vd0 + (uint64_t)((vs * C::PAIR_BYTES) >> 4);
            const uint32_t a = tP + pb * 32;
            umma_ts(tO, a, bd0, C::IDESC_PV, r == 0 ? 0u : 1u);
#pragma unroll
            for (int ks = 1; ks < 4; ks++) umma_ts_c<true>(tO, a + ks * 8, bd0 + (uint64_t)((ks * 2048) >> 4), C::IDESC_PV);
            umma_commit(p_empty(pb));
            umma_commit(v_empty(vs));
          }
          if (ok) umma_commit(o_full);
        }
      }
      // nothing of this thread's may still run when tensor memory is released (a barrier of its
      // own: a further phase of o_full could be mistaken by an epilogue warp still waiting on it)
      umma_commit(m_done2);
      mbar_drain(m_done2, 0, abort_flag);
    }
  } else {
    // ===================== epilogue: thread = tensor-memory lane = query of the pass =====================
    const uint32_t lq = (uint32_t)(32 * warp) << 16;  // this warp's lane quarter
    const uint32_t tA = tmem + lq + C::COL_A, tS = tmem + lq + C::COL_S, tP = tmem + lq + C::COL_P,
                   tO = tmem + lq + C::COL_O;
    const float sc2 = g.scale * kLog2e;
    uint32_t sc = 0, pc = 0, npass = 0;
    bool ok = true;
    // lane 0 waits, the warp follows
    auto wwait = [&](uint32_t bar, uint32_t parity) {
      int r = 1;
      if (lane == 0) r = mbar_wait(bar, parity, abort_flag) ? 1 : 0;
      return __shfl_sync(kFull, r, 0) != 0;
    };
    for (int64_t t = blockIdx.x; t < tg.tiles && ok; t += gridDim.x) {
      TcTile T;
      tc_tile(tg, sg, start, t, T);
      const int passes = (T.cnt + 127) / 128;
      const int h = h0 + T.hh;
      for (int ps = 0; ps < passes && ok; ps++, npass++) {
        // ---- this thread's query
        const int qi = ps * 128 + warp * 32 + lane;
        const bool live = qi < T.cnt;
        int n = 0, eox = 0, dy = 0;
        float ft = 0.f, fy = 0.f, fx = 0.f;
        int lo[3] = {1, 1, 1}, hi[3] = {0, 0, 0};
        if (live) {
          int r = qi, i = 0;
          while (i < kTcRyMax - 1 && r >= T.rn[i]) r -= T.rn[i++];
          const int pos = T.r0[i] + r;
          n = sorted_n[pos];
          const Query Qd = decode_query(g, off, h, n);
          eox = sorted_ex[pos] - T.X0;
          dy = Qd.o[1] + g.kh - T.Y0;
          DSA3D_DEVICE_CHECK(Qd.ok && Qd.o[0] + g.kt == T.et && dy == i && eox >= 0 && eox < tg.Wx);
          ft = Qd.f[0];
          fy = Qd.f[1];
          fx = Qd.f[2];
#pragma unroll
          for (int a = 0; a < 3; a++) {
            lo[a] = Qd.lo[a];
            hi[a] = Qd.hi[a];
          }
        }
        // ---- the query tile (A operand of the raw dots): the thread's q row, bf16 pairs
        {
          const uint4* qr = reinterpret_cast<const uint4*>(q + ((int64_t)n * g.heads + h) * DH);
#pragma unroll
          for (int part = 0; part < DH / 64; part++) {
            uint32_t qw[32];
#pragma unroll
            for (int c = 0; c < 8; c++) {
              const uint4 v4 = live ? __ldg(qr + 8 * part + c) : make_uint4(0, 0, 0, 0);
              qw[4 * c] = v4.x; qw[4 * c + 1] = v4.y; qw[4 * c + 2] = v4.z; qw[4 * c + 3] = v4.w;
            }
            tmem_st32(tA + 32 * part, qw);
          }
          tmem_st_wait();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(a_full);
        }
        const int cmin = eox + lo[2], cmax = eox + hi[2];
        float m_used = -INFINITY, l = 0.f;
        float xsp[32];  // x-splat of the previous tap row's P
        float tprev[32];  // t-blended raw dots of the previous union row
        for (int u = 0; u < g.kt && ok; u++) {
          const bool plane_ok = live && lo[0] <= u && u <= hi[0];
#pragma unroll
          for (int c = 0; c < 32; c++) xsp[c] = 0.f;
          // step j: the raw dots of union row j (j < U), then tap row j-1 and the value weights of
          // box row j-1 (j >= 1)
          for (int j = 0; j <= U && ok; j++) {
            float tcur[32];
            if (j < U) {
              ok = wwait(s_full(sc & 1), (sc >> 1) & 1);
              if (!ok) break;
              tc_fence_after();
              uint32_t d0[32], d1[32];
              tmem_ld32(tS + (sc & 1) * 64, d0);
              tmem_ld32(tS + (sc & 1) * 64 + 32, d1);
              tmem_ld_wait(d0);
              tmem_ld_wait(d1);
              tc_fence_before();
              __syncwarp();
              if (lane == 0) mbar_arrive(s_empty(sc & 1));
              sc++;
#pragma unroll
              for (int c = 0; c < 32; c++) {
                const float a = __uint_as_float(d0[c]), b = __uint_as_float(d1[c]);
                tcur[c] = fmaf(ft, b - a, a);  // (1 - f_t) plane u + f_t plane u+1
              }
            } else {
#pragma unroll
              for (int c = 0; c < 32; c++) tcur[c] = 0.f;
            }
            if (j == 0) {
#pragma unroll
              for (int c = 0; c < 32; c++) tprev[c] = tcur[c];
              continue;
            }
            float p[32];
            const int v = j - 1 - dy;  // this query's tap row
            const bool row_ok = plane_ok && j < U && lo[1] <= v && v <= hi[1];
            float mx = -INFINITY;
            if (row_ok) {
              // y-blend of rows j-1 and j, then tap column c: keys c, c+1 blended along x; masked
              // outside [cmin, cmax]
              float yb[32];
#pragma unroll
              for (int c = 0; c < 32; c++) yb[c] = fmaf(fy, tcur[c] - tprev[c], tprev[c]);
#pragma unroll
              for (int c = 0; c < 31; c++) {
                const float sv = fmaf(fx, yb[c + 1] - yb[c], yb[c]) * sc2;
                p[c] = (c >= cmin && c <= cmax) ? sv : -INFINITY;
              }
              p[31] = -INFINITY;
              float m16[16];
#pragma unroll
              for (int c = 0; c < 16; c++) m16[c] = fmaxf(p[c], p[c + 16]);
#pragma unroll
              for (int w = 8; w >= 1; w >>= 1)
#pragma unroll
                for (int c = 0; c < w; c++) m16[c] = fmaxf(m16[c], m16[c + w]);
              mx = m16[0];
            } else {
#pragma unroll
              for (int c = 0; c < 32; c++) p[c] = -INFINITY;
            }
#pragma unroll
            for (int c = 0; c < 32; c++) tprev[c] = tcur[c];
            // lazy rescale: raise the max in use only when this row's max exceeds it by 2^8
            float alpha = 1.f;
            bool resc = false;
            if (mx > m_used + kTcRescale) {
              if (m_used == -INFINITY) {
                m_used = mx;  // nothing accumulated yet
              } else {
                alpha = ex2_approx(m_used - mx);
                m_used = mx;
                resc = true;
              }
            }
            if (__any_sync(kFull, resc)) {
              // every P.V issued so far must be done (the previous step's is the last one)
              if (pc >= 1) {
                ok = wwait(p_empty((pc - 1) & 1), ((pc - 1) >> 1) & 1);
                if (!ok) break;
              }
              tc_fence_after();
#pragma unroll
              for (int part = 0; part < DH / 32; part++) {
                uint32_t orow[32];
                tmem_ld32(tO + 32 * part, orow);
                tmem_ld_wait(orow);
#pragma unroll
                for (int i = 0; i < 32; i++) orow[i] = __float_as_uint(__uint_as_float(orow[i]) * alpha);
                tmem_st32(tO + 32 * part, orow);
              }
              tmem_st_wait();
              l *= alpha;
#pragma unroll
              for (int c = 0; c < 32; c++) xsp[c] *= alpha;
            }
            // P, its sum, the x-splat, and the value weights of box row j-1
            const float mu = (m_used == -INFINITY) ? 0.f : m_used;  // no valid tap yet: every p is 0
#pragma unroll
            for (int c = 0; c < 32; c++) p[c] = ex2_approx(p[c] - mu);  // -inf -> 0
            {
              float s16[16];
#pragma unroll
              for (int c = 0; c < 16; c++) s16[c] = p[c] + p[c + 16];
#pragma unroll
              for (int w = 8; w >= 1; w >>= 1)
#pragma unroll
                for (int c = 0; c < w; c++) s16[c] += s16[c + w];
              l += s16[0];
            }
            uint32_t pw[32];
            float prev = 0.f;
#pragma unroll
            for (int c = 0; c < 32; c += 2) {
              float be[2];
#pragma unroll
              for (int e = 0; e < 2; e++) {
                const float cur = p[c + e];
                const float xs = fmaf(fx, prev - cur, cur);  // (1 - fx) p[c] + fx p[c-1]
                be[e] = fmaf(fy, xsp[c + e] - xs, xs);       // (1 - fy) xs + fy xs_prev
                xsp[c + e] = xs;
                prev = cur;
              }
              pw[c >> 1] = bf16x2_bits((1.f - ft) * be[0], (1.f - ft) * be[1]);
              pw[16 + (c >> 1)] = bf16x2_bits(ft * be[0], ft * be[1]);
            }
            // the buffer's previous P.V (two steps back) must be done before it is rewritten
            if (pc >= 2) {
              ok = wwait(p_empty(pc & 1), ((pc - 2) >> 1) & 1);
              if (!ok) break;
            }
            tc_fence_after();
            tmem_st32(tP + (pc & 1) * 32, pw);
            tmem_st_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(p_full(pc & 1));
            pc++;
          }
        }
        if (!ok) break;
        // ---- normalise and store this pass's rows
        ok = wwait(o_full, npass & 1);
        if (!ok) break;
        tc_fence_after();
        const float inv = (l > 0.f) ? 1.f / l : 0.f;
#pragma unroll
        for (int part = 0; part < DH / 32; part++) {
          uint32_t orow[32];
          tmem_ld32(tO + 32 * part, orow);
          tmem_ld_wait(orow);
          if (live) {
            uint4* dst = reinterpret_cast<uint4*>(out + ((int64_t)n * g.heads + h) * DH + 32 * part);
#pragma unroll
            for (int i = 0; i < 4; i++) {
              uint4 w4;
              w4.x = bf16x2_bits(__uint_as_float(orow[8 * i]) * inv, __uint_as_float(orow[8 * i + 1]) * inv);
              w4.y = bf16x2_bits(__uint_as_float(orow[8 * i + 2]) * inv, __uint_as_float(orow[8 * i + 3]) * inv);
              w4.z = bf16x2_bits(__uint_as_float(orow[8 * i + 4]) * inv, __uint_as_float(orow[8 * i + 5]) * inv);
              w4.w = bf16x2_bits(__uint_as_float(orow[8 * i + 6]) * inv, __uint_as_float(orow[8 * i + 7]) * inv);
              dst[i] = w4;
            }
          }
        }
        if (live && lse) lse[(int64_t)h * g.N + n] = (m_used + log2f(l)) * kLn2;
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(o_empty);
      }
    }
  }

  // release tensor memory once no role can touch it
  tc_fence_before();
  __syncthreads();
  if (warp == kTcMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, C::COLS);
  }
}

}  // namespace dsa3d
