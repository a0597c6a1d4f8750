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
// of a tile are processed at once, one per tensor-memory lane (more: further passes); a pass
// walks only the union rows of the bucket rows its queries fall in.
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
// sum and writes out and lse.  A step in which no lane of an epilogue warp has a tap row or a
// y-carry on the box row skips the arithmetic and hands the UMMA zero weights.
//
// Roles (384 threads): warps 0-7 the epilogue (warp e: tensor-memory lane quarter e % 4, half e / 4
// of the segment's taps, each half with its own online softmax and its own O accumulator, merged
// at the end of a pass), warps 8 and 10 the TMA producers of K and of V, warp 9 the UMMA issuer
// of the raw dots (the warp also allocates tensor memory), warp 11 the UMMA issuer of the value
// products (one lane each).
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

constexpr int kTcThreads = 384;  // 8 epilogue warps, K producer, dots issuer, V producer, P.V issuer
constexpr int kTcEpiWarps = 8;
constexpr int kTcKWarp = 8, kTcMmaWarp = 9, kTcVWarp = 10, kTcPvWarp = 11;
constexpr int kTcSeg = 32;         // keys per segment
constexpr int kTcRyMax = 12;       // bucket rows per tile (Ry <= kTcRyMax)
constexpr int kTcKStages = 4;      // K pair ring
constexpr int kTcVStages = 3;      // V pair ring
constexpr int kTcTileRing = 4;     // tiles drawn ahead of the slowest role
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
  static constexpr int COL_OA = COL_P + 64;               // O of keys 0 .. 15: dh fp32 columns
  static constexpr int COL_OB = COL_OA + DH;              // O of keys 16 .. 31
  static constexpr int COLS = 512;                        // allocation (power of two >= COL_OB + DH)
  static_assert(COL_OB + DH <= COLS, "tensor memory budget");
  static_assert((2 * kTcKStages + 2 * kTcVStages + 17 + 2 * kTcTileRing) * 8 <= 448,
                "mbarriers below the allocation slot");
  static constexpr int STAGE_BYTES = (kTcKStages + kTcVStages) * PAIR_BYTES;
  static constexpr int BAR_BYTES = 512;                   // mbarriers, then the allocation slot, abort flag
  static constexpr int XCH_BYTES = 2 * 2 * 128 * 8;       // (max, sum) per pass parity, half, lane
  static constexpr int SMEM_NEED = STAGE_BYTES + BAR_BYTES + XCH_BYTES + 1024;  // + alignment slack
  // at least 116 KB so that one CTA (and its 512 tensor-memory columns) owns an SM
  static constexpr int SMEM_BYTES = SMEM_NEED > 118784 ? SMEM_NEED : 118784;
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

// Union rows of pass ps of a tile (its queries 128 ps .. 128 ps + 127, in bucket-row order): the
// bucket rows i0 .. i1 they fall in have their boxes in union rows i0 .. i1 + kh, so the pass
// walks up = i1 - i0 + kh + 1 rows from j0 = i0 (union row j is key row Y0 - kh + j).
__device__ __forceinline__ void tc_pass_rows(const TcTile& T, int ps, int kh, int& j0, int& up) {
  const int qa = 128 * ps, qb = min(qa + 128, T.cnt) - 1;
  int i0 = -1, i1 = 0, acc = 0;
#pragma unroll
  for (int i = 0; i < kTcRyMax; i++) {
    if (T.rn[i] > 0 && acc <= qb && acc + T.rn[i] > qa) {
      if (i0 < 0) i0 = i;
      i1 = i;
    }
    acc += T.rn[i];
  }
  j0 = max(i0, 0);
  up = i1 - j0 + kh + 1;
}

template <int DH>
__global__ void __launch_bounds__(kTcThreads, 1)
    dsa3d_fwd_tc_kernel(const __grid_constant__ CUtensorMap tmk, const __grid_constant__ CUtensorMap tmv,
                        const __nv_bfloat16* __restrict__ q, const float* __restrict__ off,
                        __nv_bfloat16* __restrict__ out, float* __restrict__ lse,
                        const int* __restrict__ start, const int* __restrict__ sorted_n,
                        const int* __restrict__ sorted_ex, int* __restrict__ tile_counter, const Geo g,
                        const SortGeo sg, const TcTileGeo tg, const int h0) {
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
  auto x_bar = [&](int qtr) { return bx + 8u * (13 + qtr); };       // end-of-pass exchange of a lane quarter
  auto tile_full = [&](int s) { return bx + 8u * (17 + s); };
  auto tile_empty = [&](int s) { return bx + 8u * (17 + kTcTileRing + s); };
  uint32_t* tslot = reinterpret_cast<uint32_t*>(stages + C::STAGE_BYTES + 448);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tslot + 1);
  volatile int* tile_ring = reinterpret_cast<volatile int*>(tslot + 2);  // kTcTileRing tile indices
  float2* xch = reinterpret_cast<float2*>(stages + C::STAGE_BYTES + C::BAR_BYTES);

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
      mbar_init(s_empty(s), kTcEpiWarps);
      mbar_init(p_full(s), kTcEpiWarps);
      mbar_init(p_empty(s), 1);
    }
    mbar_init(a_full, kTcEpiWarps);
    mbar_init(o_full, 1);
    mbar_init(o_empty, kTcEpiWarps);
    mbar_init(m_done, 1);
    mbar_init(m_done2, 1);
    for (int qtr = 0; qtr < 4; qtr++) mbar_init(x_bar(qtr), 2);
    for (int s = 0; s < kTcTileRing; s++) {
      mbar_init(tile_full(s), 1);
      mbar_init(tile_empty(s), kTcThreads / 32);
    }
    *abort_flag = 0;
    mbar_fence_init();
  }
  if (warp == kTcMmaWarp) tmem_alloc(smem_u32(tslot), C::COLS);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tslot;
  // Tiles are taken in order from a counter shared by the CTAs, so that the tiles in flight stay
  // close together and their K and V rows stay in L2: the K producer draws the CTA's k-th tile into
  // slot k % kTcTileRing of a ring that one thread of every warp reads (-1: no tile left).
  auto tile_at = [&](uint32_t k, bool fetch, bool& ok) -> int64_t {
    const int s = (int)(k % kTcTileRing);
    if (fetch) {
      if (k >= (uint32_t)kTcTileRing && !mbar_wait(tile_empty(s), ((k / kTcTileRing) - 1) & 1, abort_flag)) {
        ok = false;
        return -1;
      }
      const int v = atomicAdd(tile_counter, 1);
      tile_ring[s] = (v < tg.tiles) ? v : -1;
      mbar_arrive(tile_full(s));
    }
    if (!mbar_wait(tile_full(s), (k / kTcTileRing) & 1, abort_flag)) {
      ok = false;
      return -1;
    }
    const int t = tile_ring[s];
    mbar_arrive(tile_empty(s));
    return t;
  };

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
        if (cnt < 1024) TC_CLK((is_k ? 8192 : 10240) + 2 * cnt);
        if (cnt >= (uint32_t)nst && !mbar_wait(empty, ((cnt / nst) - 1) & 1, abort_flag)) return false;
        if (cnt < 1024) TC_CLK((is_k ? 8192 : 10240) + 2 * cnt + 1);
        mbar_arrive_expect_tx(full, C::PAIR_BYTES);
#pragma unroll
        for (int hv = 0; hv < C::HALVES; hv++)
          tma_load_5d(base + s * C::PAIR_BYTES + hv * (C::PAIR_BYTES / C::HALVES), tm, full, 0, hd + hv, X, y, t0);
        cnt++;
        return true;
      };
      for (uint32_t k = 0; ok; k++) {
        const int64_t t = tile_at(k, is_k, ok);
        if (t < 0) break;
        TcTile T;
        tc_tile(tg, sg, start, t, T);
        const int passes = (T.cnt + 127) / 128;
        const int ot = T.et - g.kt, Xs = T.X0 - g.kw, hd = (h0 + T.hh) * C::HALVES;
        // per pass and tap plane u: the pairs (planes u, u+1) of the pass's union rows, in the
        // order of use
        for (int ps = 0; ps < passes && ok; ps++) {
          int j0, up;
          tc_pass_rows(T, ps, g.kh, j0, up);
          for (int u = 0; u < g.kt && ok; u++)
            for (int j = 0; j < up && ok; j++) ok = load(ot + u, T.Y0 - g.kh + j0 + j, Xs, hd);
        }
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
      for (uint32_t k = 0; ok; k++) {
        const int64_t t = tile_at(k, false, ok);
        if (t < 0) break;
        TcTile T;
        tc_tile(tg, sg, start, t, T);
        const int passes = (T.cnt + 127) / 128;
        for (int ps = 0; ps < passes && ok; ps++, npass++) {
          ok = mbar_wait(a_full, npass & 1, abort_flag);
          if (!ok) break;
          int j0, up;
          tc_pass_rows(T, ps, g.kh, j0, up);
          const int rows = g.kt * up;
          for (int r = 0; r < rows && ok; r++, kc++, sc++) {
            const int ks_ = (int)(kc % kTcKStages), sb = (int)(sc & 1);
            if (kc < 680) TC_CLK(4096 + 3 * kc);
            if (!mbar_wait(k_full(ks_), (kc / kTcKStages) & 1, abort_flag) ||
                (sc >= 2 && !mbar_wait(s_empty(sb), ((sc - 2) >> 1) & 1, abort_flag))) {
              ok = false;
              break;
            }
            if (kc < 680) TC_CLK(4096 + 3 * kc + 1);
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
            if (kc < 680) TC_CLK(4096 + 3 * kc + 2);
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
      const uint32_t tP = tmem + C::COL_P, tOa = tmem + C::COL_OA, tOb = tmem + C::COL_OB;
      const uint64_t vd0 = umma_sdesc_sw128(vst, C::PAIR_BYTES / C::HALVES, 1024);
      for (uint32_t k = 0; ok; k++) {
        const int64_t t = tile_at(k, false, ok);
        if (t < 0) break;
        TcTile T;
        tc_tile(tg, sg, start, t, T);
        const int passes = (T.cnt + 127) / 128;
        for (int ps = 0; ps < passes && ok; ps++, npass++) {
          int j0, up;
          tc_pass_rows(T, ps, g.kh, j0, up);
          const int rows = g.kt * up;
          for (int r = 0; r < rows && ok; r++, vc++, pc++) {
            const int pb = (int)(pc & 1), vs = (int)(vc % kTcVStages);
            if (pc < 512) TC_CLK(6144 + 4 * pc);
            if (!mbar_wait(p_full(pb), (pc >> 1) & 1, abort_flag)) { ok = false; break; }
            if (pc < 512) TC_CLK(6144 + 4 * pc + 1);
            if (!mbar_wait(v_full(vs), (vc / kTcVStages) & 1, abort_flag) ||
                (r == 0 && npass > 0 && !mbar_wait(o_empty, (npass - 1) & 1, abort_flag))) {
              ok = false;
              break;
            }
            if (pc < 512) TC_CLK(6144 + 4 * pc + 2);
            tc_fence_after();
            // B, MN-major: keys 16 ks .. 16 ks + 15 are rows 16 ks ..; 64-dim halves apart by
            // PAIR_BYTES / HALVES
            const uint64_t bd0 = vd0 + (uint64_t)((vs * C::PAIR_BYTES) >> 4);
            // K-steps 0 and 2 (keys 0 .. 15 of planes u, u+1) into O_a, 1 and 3 (keys 16 .. 31) into O_b
            const uint32_t a = tP + pb * 32;
            umma_ts(tOa, a, bd0, C::IDESC_PV, r == 0 ? 0u : 1u);
            umma_ts(tOb, a + 8, bd0 + (uint64_t)(2048 >> 4), C::IDESC_PV, r == 0 ? 0u : 1u);
            umma_ts_c<true>(tOa, a + 16, bd0 + (uint64_t)((2 * 2048) >> 4), C::IDESC_PV);
            umma_ts_c<true>(tOb, a + 24, bd0 + (uint64_t)((3 * 2048) >> 4), C::IDESC_PV);
            umma_commit(p_empty(pb));
            umma_commit(v_empty(vs));
            if (pc < 512) TC_CLK(6144 + 4 * pc + 3);
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
    // Warp e reads lane quarter e % 4 and takes half e / 4 of the segment: half 0 the taps 0 .. 15
    // (keys 0 .. 16), half 1 the taps 15 .. 30 (keys 15 .. 31).  Each half runs its own online
    // softmax into its own accumulator (O_a: keys 0 .. 15, O_b: keys 16 .. 31): key c's weight
    // takes taps c - 1 and c, so half 1 also evaluates tap 15, for key 16 only, and leaves it out
    // of its sum.  At the end of a pass the halves exchange (max, sum) and each writes half of the
    // output dims: out = (2^(m_a - M) O_a + 2^(m_b - M) O_b) / (2^(m_a - M) l_a + 2^(m_b - M) l_b).
    const int quarter = warp & 3, half = warp >> 2;
    const uint32_t lq = (uint32_t)(32 * quarter) << 16;  // this warp's lane quarter
    const uint32_t tA = tmem + lq + C::COL_A, tS = tmem + lq + C::COL_S, tP = tmem + lq + C::COL_P;
    const uint32_t tOa = tmem + lq + C::COL_OA, tOb = tmem + lq + C::COL_OB;
    const uint32_t tO = half ? tOb : tOa;  // this half's accumulator
    const int c0 = 15 * half;             // this half's first tap (segment column)
    const float sc2 = g.scale * kLog2e;
    const int slot = quarter * 32 + lane;
    uint32_t sc = 0, pc = 0, npass = 0, est = 0;
    bool ok = true;
#define DSA3D_EP_CLK(k) \
  if (quarter == 0 && lane == 0 && e_ < 340) TC_CLK((half ? 2048 : 0) + 6 * e_ + (k))
    // lane 0 waits, the warp follows
    auto wwait = [&](uint32_t bar, uint32_t parity) {
      int r = 1;
      if (lane == 0) r = mbar_wait(bar, parity, abort_flag) ? 1 : 0;
      return __shfl_sync(kFull, r, 0) != 0;
    };
    for (uint32_t k = 0; ok; k++) {
      int tv = -1, okv = 1;
      if (lane == 0) {
        bool o = true;
        tv = (int)tile_at(k, false, o);
        okv = o ? 1 : 0;
      }
      ok = __shfl_sync(kFull, okv, 0) != 0;
      const int64_t t = __shfl_sync(kFull, tv, 0);
      if (!ok || t < 0) break;
      TcTile T;
      tc_tile(tg, sg, start, t, T);
      const int passes = (T.cnt + 127) / 128;
      const int h = h0 + T.hh;
      for (int ps = 0; ps < passes && ok; ps++, npass++) {
        // ---- this thread's query
        const int qi = ps * 128 + slot;
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
        // ---- the query tile (A operand of the raw dots): this half's dims of the q row, bf16 pairs
        {
          const uint4* qr = reinterpret_cast<const uint4*>(q + ((int64_t)n * g.heads + h) * DH + half * (DH / 2));
#pragma unroll
          for (int part = 0; part < DH / 64; part++) {
            uint32_t qw[16];
#pragma unroll
            for (int c = 0; c < 4; c++) {
              const uint4 v4 = live ? __ldg(qr + 4 * part + c) : make_uint4(0, 0, 0, 0);
              qw[4 * c] = v4.x; qw[4 * c + 1] = v4.y; qw[4 * c + 2] = v4.z; qw[4 * c + 3] = v4.w;
            }
            tmem_st16(tA + half * (DH / 4) + 16 * part, qw);
          }
          tmem_st_wait();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(a_full);
        }
        int j0, up;
        tc_pass_rows(T, ps, g.kh, j0, up);
        // this lane's tap rows lo[1] .. hi[1] are the steps rlo .. rhi (empty when rlo > rhi); the
        // steps in which some lane of the warp has a tap row or a y-carry on box row j-1 form the
        // hull [wlo, whi]: outside it no lane has a weight, and no lane reads the raw dots of row
        // j unless step jj + 1 is inside it
        const int rlo = live ? lo[1] + 1 + dy - j0 : 1, rhi = live ? hi[1] + 1 + dy - j0 : 0;
        const bool any_rows = rlo <= rhi;
        const int wlo = __reduce_min_sync(kFull, any_rows ? rlo : 0x7fffffff);
        const int whi = __reduce_max_sync(kFull, any_rows ? rhi + 1 : -0x7fffffff);
        // this half's taps i = 0 .. 15 are segment columns c0 + i; valid in [lmin, lmax]
        const int lmin = eox + lo[2] - c0, lmax = eox + hi[2] - c0;
        float m_used = -INFINITY, l = 0.f;
        float xsp[16];    // x-splat of the previous tap row's P on this half's keys
        float tprev[17];  // t-blended raw dots of the previous union row, columns c0 .. c0 + 16
        for (int u = 0; u < g.kt && ok; u++) {
          const bool plane_ok = live && lo[0] <= u && u <= hi[0];
#pragma unroll
          for (int c = 0; c < 16; c++) xsp[c] = 0.f;
          // step jj (union row j = j0 + jj): the raw dots of row j (jj < up), then this query's tap
          // row v = j - 1 - dy (union rows j-1 and j) and the value weights of box row j-1
          // (jj >= 1), which take tap row v (1 - f_y) and the carry of tap row v-1 (f_y)
          for (int jj = 0; jj <= up && ok; jj++) {
            const uint32_t e_ = est++;
            (void)e_;
            DSA3D_EP_CLK(0);
            float tcur[17];
            if (jj < up) {
              ok = wwait(s_full(sc & 1), (sc >> 1) & 1);
              if (!ok) break;
              DSA3D_EP_CLK(1);
              if (jj + 1 >= wlo && jj + 1 <= whi) {
                tc_fence_after();
                const uint32_t sb = tS + (sc & 1) * 64;
                uint32_t a[16], b[16], a1, b1;
                if (half == 0) {  // columns 0 .. 16 of planes u (0 ..) and u+1 (32 ..)
                  tmem_ld16(sb, a);
                  tmem_ld1(sb + 16, a1);
                  tmem_ld16(sb + 32, b);
                  tmem_ld1(sb + 48, b1);
                } else {          // columns 15 .. 31
                  tmem_ld1(sb + 15, a1);
                  tmem_ld16(sb + 16, a);
                  tmem_ld1(sb + 47, b1);
                  tmem_ld16(sb + 48, b);
                }
                tmem_ld_wait(a, a1, b, b1);
                tc_fence_before();
                // (1 - f_t) plane u + f_t plane u+1
                auto tb = [&](uint32_t x, uint32_t y) {
                  const float xa = __uint_as_float(x), yb = __uint_as_float(y);
                  return fmaf(ft, yb - xa, xa);
                };
                if (half == 0) {
#pragma unroll
                  for (int c = 0; c < 16; c++) tcur[c] = tb(a[c], b[c]);
                  tcur[16] = tb(a1, b1);
                } else {
                  tcur[0] = tb(a1, b1);
#pragma unroll
                  for (int c = 0; c < 16; c++) tcur[c + 1] = tb(a[c], b[c]);
                }
              } else {
#pragma unroll
                for (int c = 0; c < 17; c++) tcur[c] = 0.f;  // no lane of the warp reads row j
              }
              __syncwarp();
              if (lane == 0) mbar_arrive(s_empty(sc & 1));
              sc++;
              DSA3D_EP_CLK(2);
            } else {
#pragma unroll
              for (int c = 0; c < 17; c++) tcur[c] = 0.f;
            }
            if (jj == 0) {
#pragma unroll
              for (int c = 0; c < 17; c++) tprev[c] = tcur[c];
              continue;
            }
            const uint32_t pb = tP + (pc & 1) * 32 + 8 * half;  // this half's words of planes u, u+1
            if (jj < wlo || jj > whi) {
              // no lane has a tap or a carry on box row j-1: every weight is 0 (and so is every
              // lane's x-splat carry), the softmax state is unchanged; the buffer's previous
              // product must be done before the zeros go in (which also keeps this warp within
              // one phase of the others on p_full)
#pragma unroll
              for (int c = 0; c < 17; c++) tprev[c] = tcur[c];
              if (pc >= 2) {
                ok = wwait(p_empty(pc & 1), ((pc - 2) >> 1) & 1);
                if (!ok) break;
              }
              tc_fence_after();
              uint32_t zw[8];
#pragma unroll
              for (int c = 0; c < 8; c++) zw[c] = 0u;
              tmem_st8(pb, zw);
              tmem_st8(pb + 16, zw);
              tmem_st_wait();
              tc_fence_before();
              __syncwarp();
              if (lane == 0) mbar_arrive(p_full(pc & 1));
              pc++;
              continue;
            }
            float p[17];  // this half's taps 0 .. 15 (p[16]: tap 31 for half 1, never valid)
            const bool row_ok = plane_ok && jj < up && rlo <= jj && jj <= rhi;
            float mx = -INFINITY;
            if (row_ok) {
              // y-blend of rows j-1 and j, then tap i: columns i, i+1 blended along x; masked
              // outside [lmin, lmax]
              float yb[17];
#pragma unroll
              for (int c = 0; c < 17; c++) yb[c] = fmaf(fy, tcur[c] - tprev[c], tprev[c]);
#pragma unroll
              for (int c = 0; c < 16; c++) {
                const float sv = fmaf(fx, yb[c + 1] - yb[c], yb[c]) * sc2;
                p[c] = (c >= lmin && c <= lmax) ? sv : -INFINITY;
              }
              p[16] = -INFINITY;
              float m8[8];
#pragma unroll
              for (int c = 0; c < 8; c++) m8[c] = fmaxf(p[c], p[c + 8]);
#pragma unroll
              for (int w = 4; w >= 1; w >>= 1)
#pragma unroll
                for (int c = 0; c < w; c++) m8[c] = fmaxf(m8[c], m8[c + w]);
              mx = m8[0];
            } else {
#pragma unroll
              for (int c = 0; c < 17; c++) p[c] = -INFINITY;
            }
#pragma unroll
            for (int c = 0; c < 17; c++) tprev[c] = tcur[c];
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
              // 16 columns at a time: the step's arrays are live here
#pragma unroll 1
              for (int part = 0; part < DH / 16; part++) {
                uint32_t orow[16], o1;
                tmem_ld16(tO + 16 * part, orow);
                tmem_ld_wait16(orow, o1);
#pragma unroll
                for (int i = 0; i < 16; i++) orow[i] = __float_as_uint(__uint_as_float(orow[i]) * alpha);
                tmem_st16(tO + 16 * part, orow);
              }
              tmem_st_wait();
              l *= alpha;
#pragma unroll
              for (int c = 0; c < 16; c++) xsp[c] *= alpha;
            }
            // P, its sum (half 1 leaves out tap 15, which half 0 counts), the x-splat onto this
            // half's keys, and the value weights of box row j-1
            DSA3D_EP_CLK(3);
            const float mu = (m_used == -INFINITY) ? 0.f : m_used;  // no valid tap yet: every p is 0
#pragma unroll
            for (int c = 0; c < 16; c++) p[c] = ex2_approx(p[c] - mu);  // -inf -> 0
            p[16] = 0.f;
            {
              float s8[8];
              s8[0] = (half ? 0.f : p[0]) + p[8];
#pragma unroll
              for (int c = 1; c < 8; c++) s8[c] = p[c] + p[c + 8];
#pragma unroll
              for (int w = 4; w >= 1; w >>= 1)
#pragma unroll
                for (int c = 0; c < w; c++) s8[c] += s8[c + w];
              l += s8[0];
            }
            // key k of the half (segment key c0 + half + k) takes taps k - 1 + half and k + half
            uint32_t pw0[8], pw1[8];
            {
              float be[16];
              if (half == 0) {
                float prev = 0.f;
#pragma unroll
                for (int k = 0; k < 16; k++) {
                  const float cur = p[k];
                  const float xs = fmaf(fx, prev - cur, cur);  // (1 - fx) p[k] + fx p[k-1]
                  be[k] = fmaf(fy, xsp[k] - xs, xs);           // (1 - fy) xs + fy xs_prev
                  xsp[k] = xs;
                  prev = cur;
                }
              } else {
#pragma unroll
                for (int k = 0; k < 16; k++) {
                  const float cur = p[k + 1], prev = p[k];
                  const float xs = fmaf(fx, prev - cur, cur);
                  be[k] = fmaf(fy, xsp[k] - xs, xs);
                  xsp[k] = xs;
                }
              }
#pragma unroll
              for (int k = 0; k < 16; k += 2) {
                pw0[k >> 1] = bf16x2_bits((1.f - ft) * be[k], (1.f - ft) * be[k + 1]);
                pw1[k >> 1] = bf16x2_bits(ft * be[k], ft * be[k + 1]);
              }
            }
            // the buffer's previous P.V (two steps back) must be done before it is rewritten
            if (pc >= 2) {
              ok = wwait(p_empty(pc & 1), ((pc - 2) >> 1) & 1);
              if (!ok) break;
            }
            DSA3D_EP_CLK(4);
            tc_fence_after();
            tmem_st8(pb, pw0);
            tmem_st8(pb + 16, pw1);
            tmem_st_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(p_full(pc & 1));
            pc++;
            DSA3D_EP_CLK(5);
          }
        }
        if (!ok) break;
        // ---- merge the halves and store this pass's rows: half h writes dims h dh/2 .. (h+1) dh/2
        ok = wwait(o_full, npass & 1);
        if (!ok) break;
        tc_fence_after();
        // (max, sum) to the partner warp through a slot pair of this pass's parity: a slot is
        // written again two passes later, after the partner's next exchange, so it has been read
        float2* xs = xch + (npass & 1) * 256;
        xs[half * 128 + slot] = make_float2(m_used, l);
        __syncwarp();
        if (lane == 0) mbar_arrive(x_bar(quarter));
        ok = wwait(x_bar(quarter), npass & 1);
        if (!ok) break;
        __syncwarp();
        const float2 other = xs[(1 - half) * 128 + slot];
        const float ma = half ? other.x : m_used, la = half ? other.y : l;
        const float mb = half ? m_used : other.x, lb = half ? l : other.y;
        const float M = fmaxf(ma, mb);
        const float wa = (M == -INFINITY) ? 0.f : ex2_approx(ma - M);
        const float wb = (M == -INFINITY) ? 0.f : ex2_approx(mb - M);
        const float L = wa * la + wb * lb;
        const float inv = (L > 0.f) ? 1.f / L : 0.f;
        const float ca = wa * inv, cb = wb * inv;
        const bool warp_live = __any_sync(kFull, live);  // a warp past the pass's queries reads nothing
#pragma unroll
        for (int part = 0; part < DH / 64 && warp_live; part++) {
          const int col = half * (DH / 2) + 32 * part;
          uint32_t oa[32], ob[32];
          tmem_ld32(tOa + col, oa);
          tmem_ld32(tOb + col, ob);
          tmem_ld_wait(oa);
          tmem_ld_wait(ob);
          if (live) {
            uint4* dst = reinterpret_cast<uint4*>(out + ((int64_t)n * g.heads + h) * DH + col);
            auto o = [&](int i) { return fmaf(ca, __uint_as_float(oa[i]), cb * __uint_as_float(ob[i])); };
#pragma unroll
            for (int i = 0; i < 4; i++) {
              uint4 w4;
              w4.x = bf16x2_bits(o(8 * i), o(8 * i + 1));
              w4.y = bf16x2_bits(o(8 * i + 2), o(8 * i + 3));
              w4.z = bf16x2_bits(o(8 * i + 4), o(8 * i + 5));
              w4.w = bf16x2_bits(o(8 * i + 6), o(8 * i + 7));
              dst[i] = w4;
            }
          }
        }
        if (half == 0 && live && lse) lse[(int64_t)h * g.N + n] = (M + log2f(L)) * kLn2;
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(o_empty);
      }
    }
#undef DSA3D_EP_CLK
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
