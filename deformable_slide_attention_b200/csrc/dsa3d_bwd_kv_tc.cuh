// dsa3d_bwd_kv_tc.cuh -- key side of the 3D-DSA backward on the 5th-generation tensor cores:
// dK = scale Gamma^T Q and dV = Beta^T dO accumulated in tensor memory (bf16 I/O, dh 64 or 128).
//
// The derivative of Eq. 1 (MegaSlide-DiT, arXiv 2607.22696) with respect to a key row k_j sums,
// over every query whose box holds j, scale * gamma_j * q, and with respect to v_j the sum of
// beta_j * dO, where beta_j (gamma_j) is the query's trilinear splat of P (of P (dP - D)) onto box
// position j.  The query side (dsa3d_bwd_q_kernel) stores, per query, tap plane and box row, the
// splats of P (beta) and P dP (gamma') in bf16, and D and f_t; gamma = gamma' - D beta and the
// t-mix of the two tap planes that feed a box plane are formed here.
//
// Work unit: a key tile of kKvtRows key rows x 32 keys (M = 128, one tensor-memory lane per key)
// of one frame and head.  The queries whose boxes cover the tile lie in (kt + 1) x ney bucket-row
// ranges of the window-origin sort (box plane bt, origin row e_y, origin x range); they are
// concatenated and consumed kKvtQ per stage.  A stage holds, in shared memory with the 128-byte
// swizzle: Gamma^T and Beta^T (128 keys x kKvtQ queries, K-major: the A operands) and the stage's
// q and dO rows (kKvtQ queries x dh, MN-major: the B operands).  Per stage one thread issues
// dK += Gamma^T Q and dV += Beta^T dO (M = 128, N = dh, K = kKvtQ) into a pair of accumulators in
// tensor memory; two pairs alternate between tiles, so a tile's results are written while the
// next tile's products run.
//
// Roles (416 threads): warps 0-7 build stages, warp w the query columns 8w .. 8w + 7 of every
// stage (its slots, their q and dO rows, their columns of Gamma^T and Beta^T), each on its own;
// warps 8-11 write dK and dV (thread = key); warp 12 issues the UMMAs and owns the
// tensor-memory allocation.  mbarriers order the roles; every wait is bounded (dsa3d_tc.cuh).
#pragma once

#include "dsa3d_bwd_mma.cuh"  // BoxGeo, bf16 helpers, cp.async helpers
#include "dsa3d_sort.cuh"
#include "dsa3d_tc.cuh"

namespace dsa3d {

constexpr int kKvtRows = 4;        // key rows per tile
constexpr int kKvtKeys = 32;       // keys per key row of a tile
constexpr int kKvtQ = 64;          // queries per stage (K of the UMMAs: four K-steps of 16)
constexpr int kKvtStages = 3;
constexpr int kKvtTileRing = 4;    // tiles drawn ahead of the slowest role
constexpr int kKvtRanges = 128;    // bucket-row ranges per tile: (kt + 1) (kKvtRows + kh) <= this
constexpr int kKvtEpiWarp0 = 8, kKvtMmaWarp = 12;
constexpr int kKvtThreads = 13 * 32;

// Geometry of a tile, the same in every role.
struct KvtTile {
  int hh, tk, yk0, x_lo, ney, nranges;
};

__device__ __forceinline__ KvtTile kvt_tile(const Geo& g, const SortGeo& sg, int64_t t) {
  const int NB = (g.Wp + kKvtKeys - 1) / kKvtKeys, NY = (g.Hp + kKvtRows - 1) / kKvtRows;
  KvtTile T;
  const int b = (int)(t % NB);
  t /= NB;
  const int yb = (int)(t % NY);
  t /= NY;
  T.tk = (int)(t % g.F);
  T.hh = (int)(t / g.F);
  T.x_lo = kKvtKeys * b;
  T.yk0 = kKvtRows * yb;
  T.ney = min(T.yk0 + kKvtRows - 1 + g.kh, sg.Ey - 1) - T.yk0 + 1;
  T.nranges = (g.kt + 1) * T.ney;
  return T;
}

// Range r of a tile: box plane bt = r / ney of the covering queries, origin row e_y = yk0 + r % ney,
// origin x in [x_lo, x_lo + 32 + kw): its first sorted position and its length.
__device__ __forceinline__ void kvt_range(const Geo& g, const SortGeo& sg, const KvtTile& T,
                                          const int* __restrict__ start, int r, int& beg, int& len) {
  beg = 0;
  len = 0;
  if (r < T.nranges) {
    const int bt = r / T.ney, ey = T.yk0 + (r - bt * T.ney);
    const int64_t b0 = (int64_t)T.hh * sg.E1 + ((int64_t)(T.tk - bt + g.kt) * sg.Ey + ey) * sg.Ex;
    beg = start[b0 + T.x_lo];
    len = start[b0 + min(T.x_lo + kKvtKeys + g.kw, sg.Ex)] - beg;
  }
}

// Queries covering a tile, summed by one warp (four ranges per lane).
__device__ __forceinline__ int kvt_total(const Geo& g, const SortGeo& sg, const KvtTile& T,
                                         const int* __restrict__ start, int lane) {
  int sum = 0;
#pragma unroll
  for (int e = 0; e < kKvtRanges / 32; e++) {
    int beg, len;
    kvt_range(g, sg, T, start, lane + 32 * e, beg, len);
    sum += len;
  }
#pragma unroll
  for (int d = 16; d >= 1; d >>= 1) sum += __shfl_xor_sync(kFull, sum, d);
  return sum;
}

// One query slot of a stage.
struct KvtSlot {
  int64_t row;  // element offset of the query's q / dO row
  int64_t box;  // element offset of the query's stored splats
  int bt;       // box plane of the tile's frame in the query's box
  int by0;      // box row of the tile's first key row (may lie outside [0, kh])
  int ox;       // x-origin of the box minus the tile's first key x
  int ok;       // 0: empty slot
  float D, ft;
};

template <int DH>
struct KvtCfg {
  static constexpr int A_BYTES = 128 * kKvtQ * 2;         // Gamma^T or Beta^T: 128 keys x 64 queries
  static constexpr int B_BYTES = kKvtQ * DH * 2;          // q or dO rows
  static constexpr int HALF_BYTES = kKvtQ * 128;          // one 64-dim half of the B rows
  static constexpr int STAGE_BYTES = 2 * A_BYTES + 2 * B_BYTES;
  static constexpr int META_BYTES = kKvtStages * kKvtQ * (int)sizeof(KvtSlot);
  static constexpr int RANGE_BYTES = kKvtEpiWarp0 * (2 * kKvtRanges + 8) * 4;
  static constexpr int SCRATCH_BYTES = 16 * kKvtEpiWarp0;  // a store target per builder warp
  static constexpr int BAR_BYTES = 256;
  static constexpr int SMEM_BYTES =
      kKvtStages * STAGE_BYTES + META_BYTES + RANGE_BYTES + SCRATCH_BYTES + BAR_BYTES + 1024;
  static constexpr int COLS = (4 * DH <= 256) ? 256 : 512;  // two (dK, dV) pairs
  static constexpr uint32_t IDESC = umma_idesc_bf16(128, DH, false, true);
  static_assert(SMEM_BYTES <= 227 * 1024, "shared memory budget");
  static_assert(A_BYTES % 1024 == 0 && B_BYTES % 1024 == 0, "1024-byte swizzle atoms");
};

// The A tiles are K-major with the 128-byte swizzle: key m's row of 64 queries is the 128 bytes at
// 128 m, and its 16-byte chunk of queries 8 c .. 8 c + 7 sits at chunk c ^ (m & 7) (TMA's
// CU_TENSOR_MAP_SWIZZLE_128B pattern, 1024-byte atoms).  The B rows are MN-major: the 16-byte
// chunk c (dims 64 hv + 8 c ..) of query row k is at kvt_b_off(k, hv, c).
__device__ __forceinline__ uint32_t kvt_b_off(int k, int hv, int c) {
  return (uint32_t)(hv * (kKvtQ * 128) + k * 128 + ((c ^ (k & 7)) << 4));
}



template <int DH>
__global__ void __launch_bounds__(kKvtThreads, 1)
    dsa3d_bwd_kv_tc_kernel(const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ dout,
                           __nv_bfloat16* __restrict__ dk, __nv_bfloat16* __restrict__ dv,
                           const int* __restrict__ start, const int* __restrict__ sorted_n,
                           const int* __restrict__ sorted_ex, const unsigned short* __restrict__ gbox,
                           const unsigned short* __restrict__ bbox, const float2* __restrict__ dft,
                           int* __restrict__ tile_counter, const Geo g, const SortGeo sg, const BoxGeo bg,
                           const int h0, const int hg) {
  using C = KvtCfg<DH>;
  extern __shared__ __align__(1024) unsigned char kvt_smem[];
  unsigned char* stages = kvt_smem + ((1024 - (smem_u32(kvt_smem) & 1023)) & 1023);
  KvtSlot* meta = reinterpret_cast<KvtSlot*>(stages + kKvtStages * C::STAGE_BYTES);
  int* ranges = reinterpret_cast<int*>(stages + kKvtStages * C::STAGE_BYTES + C::META_BYTES);
  unsigned char* scratch = stages + kKvtStages * C::STAGE_BYTES + C::META_BYTES + C::RANGE_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(scratch + C::SCRATCH_BYTES);
  const uint32_t st0 = smem_u32(stages);
  const uint32_t b0 = smem_u32(bars);
  auto full = [&](int s) { return b0 + 8u * s; };
  auto empty = [&](int s) { return b0 + 8u * (kKvtStages + s); };
  auto acc_full = [&](int s) { return b0 + 8u * (2 * kKvtStages + s); };
  auto acc_empty = [&](int s) { return b0 + 8u * (2 * kKvtStages + 2 + s); };
  const uint32_t m_done = b0 + 8u * (2 * kKvtStages + 4);
  auto tile_full = [&](int s) { return b0 + 8u * (2 * kKvtStages + 5 + s); };
  auto tile_empty = [&](int s) { return b0 + 8u * (2 * kKvtStages + 5 + kKvtTileRing + s); };
  uint32_t* tslot = reinterpret_cast<uint32_t*>(bars + 24);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tslot + 1);
  volatile int* tile_ring = reinterpret_cast<volatile int*>(tslot + 2);  // kKvtTileRing tile indices
  static_assert((2 * kKvtStages + 5 + 2 * kKvtTileRing) * 8 <= 192 && 192 + 8 + 4 * kKvtTileRing <= C::BAR_BYTES,
                "barrier slots");

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kKvtStages; s++) {
      mbar_init(full(s), kKvtEpiWarp0 * 32);
      mbar_init(empty(s), 1);
    }
    for (int s = 0; s < 2; s++) {
      mbar_init(acc_full(s), 1);
      mbar_init(acc_empty(s), 4);
    }
    mbar_init(m_done, 1);
    for (int s = 0; s < kKvtTileRing; s++) {
      mbar_init(tile_full(s), 1);
      mbar_init(tile_empty(s), kKvtThreads / 32);
    }
    *abort_flag = 0;
    mbar_fence_init();
  }
  if (warp == kKvtMmaWarp) tmem_alloc(smem_u32(tslot), C::COLS);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tslot;
  const int NB = (g.Wp + kKvtKeys - 1) / kKvtKeys, NY = (g.Hp + kKvtRows - 1) / kKvtRows;
  const int64_t tiles = (int64_t)hg * g.F * NY * NB;
  // Tiles are taken in order from a counter shared by the CTAs (so that the tiles in flight stay
  // close together and their query rows and splats stay in L2): builder warp 0's lane 0 draws the
  // CTA's k-th tile into slot k % kKvtTileRing of a ring every warp reads (-1: no tile left).
  auto next_tile = [&](uint32_t k, bool& ok) -> int64_t {
    const int s = (int)(k % kKvtTileRing);
    int64_t t = -1;
    if (lane == 0) {
      if (warp == 0) {
        if (k >= (uint32_t)kKvtTileRing && !mbar_wait(tile_empty(s), ((k / kKvtTileRing) - 1) & 1, abort_flag)) ok = false;
        if (ok) {
          const int v = atomicAdd(tile_counter, 1);
          tile_ring[s] = (v < tiles) ? v : -1;
          mbar_arrive(tile_full(s));
        }
      }
      if (ok && !mbar_wait(tile_full(s), (k / kKvtTileRing) & 1, abort_flag)) ok = false;
      if (ok) {
        t = tile_ring[s];
        mbar_arrive(tile_empty(s));
      }
    }
    ok = __shfl_sync(kFull, ok ? 1 : 0, 0) != 0;
    t = __shfl_sync(kFull, (int)t, 0);
    return ok ? t : -1;
  };

  if (warp < kKvtEpiWarp0) {
    // ===================== stage builders: warp w builds query columns 8w .. 8w + 7 of every stage =====================
    // Each warp works on its own: the tile's ranges (its own copy), its 8 slots, their q and dO
    // rows, the zeros and splats of its 8 columns of Gamma^T and Beta^T; every thread arrives on
    // the stage's full barrier once its copies and stores are done and fenced.
    int* r_beg = ranges + warp * (2 * kKvtRanges + 8);
    int* r_pre = r_beg + kKvtRanges;  // kKvtRanges + 1 entries
    KvtSlot* mw = meta;               // stage buffers' slots
    uint32_t gs = 0;                  // stages of the tiles before this one
    bool ok = true;
    for (uint32_t kt_ = 0; ok; kt_++) {
      const int64_t t = next_tile(kt_, ok);
      if (t < 0) break;
      const KvtTile T = kvt_tile(g, sg, t);
      const int h = h0 + T.hh;
      // ranges 4 lane .. 4 lane + 3 and their exclusive prefix
      int beg[4], len[4], sum = 0;
#pragma unroll
      for (int e = 0; e < 4; e++) {
        kvt_range(g, sg, T, start, 4 * lane + e, beg[e], len[e]);
        sum += len[e];
      }
      int incl = sum;
#pragma unroll
      for (int d = 1; d < 32; d <<= 1) {
        const int y = __shfl_up_sync(kFull, incl, d);
        if (lane >= d) incl += y;
      }
      const int total = __shfl_sync(kFull, incl, 31);
      __syncwarp();  // the previous tile's ranges are read
      {
        int run = incl - sum;
#pragma unroll
        for (int e = 0; e < 4; e++) {
          r_beg[4 * lane + e] = beg[e];
          r_pre[4 * lane + e] = run;
          run += len[e];
        }
        if (lane == 0) r_pre[kKvtRanges] = total;
      }
      __syncwarp();
      const int nst = (total + kKvtQ - 1) / kKvtQ;
      // slot i = kKvtQ ls + 8 warp + lane of the concatenated ranges (lanes 0 .. 7): its range and
      // sorted position, and the loads it needs, left raw so that nothing waits for them until
      // the slot is written out a stage later
      struct SlotRaw {
        int lo, pos, ex, n;
        float2 d;
      };
      auto slot_load = [&](int ls) {
        SlotRaw sr;
        sr.lo = -1;
        sr.pos = 0;
        sr.ex = 0;
        sr.n = 0;
        sr.d = make_float2(0.f, 0.f);
        const int i = kKvtQ * ls + 8 * warp + lane;
        if (lane < 8 && i < total) {
          int lo = 0, hi = kKvtRanges;  // largest r with r_pre[r] <= i (a non-empty range)
          while (hi - lo > 1) {
            const int mid = (lo + hi) >> 1;
            if (r_pre[mid] <= i) lo = mid; else hi = mid;
          }
          sr.lo = lo;
          sr.pos = r_beg[lo] + (i - r_pre[lo]);
          sr.ex = sorted_ex[sr.pos];
          sr.n = sorted_n[sr.pos];
          sr.d = dft[sr.pos];
        }
        return sr;
      };
      auto slot_of = [&](const SlotRaw& sr) {
        KvtSlot m;
        m.ok = sr.lo >= 0 ? 1 : 0;
        const int bt = m.ok ? sr.lo / T.ney : 0;
        m.bt = bt;
        m.by0 = g.kh - (sr.lo - bt * T.ney);  // yk0 - e_y + kh
        m.ox = sr.ex - g.kw - T.x_lo;
        m.row = ((int64_t)sr.n * g.heads + h) * DH;
        m.box = (int64_t)sr.pos * bg.per_q;
        m.D = sr.d.x;
        m.ft = sr.d.y;
        return m;
      };
      // software pipeline: the slots of stage ls + 1 and the splat words of stage ls are loaded
      // while stage ls's buffer is awaited, copied into and zeroed
      SlotRaw snext = slot_load(0);
      for (int ls = 0; ls < nst && ok; ls++) {
        const uint32_t G = gs + (uint32_t)ls;
        const int buf = (int)(G % kKvtStages);
        KvtSlot* ms = mw + buf * kKvtQ + 8 * warp;  // this warp's 8 slots
#define DSA3D_KV_CLK(k) \
  if (lane == 0 && warp == 0 && G < 500) TC_CLK(8 * G + (k))
        DSA3D_KV_CLK(0);
        if (lane < 8) ms[lane] = slot_of(snext);
        __syncwarp();
        DSA3D_KV_CLK(1);
        // item lane: slot lane / 4, key row lane % 4; its box row's words (at most 8: k_w <= 15)
        // are loaded before the buffer wait and used after the zeros
        const int kl = lane >> 2, r = lane & 3;
        const KvtSlot m = ms[kl];
        const int by = m.by0 + r;
        const bool live = m.ok && by >= 0 && by <= g.kh && T.yk0 + r < g.Hp;
        const int words = bg.width >> 1;
        unsigned gw0[8], ew0[8], gw1[8], ew1[8];
        {
          const int64_t o0 = m.box + (int64_t)(m.bt * (g.kh + 1) + by) * bg.width;  // tap plane bt
          const int64_t o1 = o0 - (int64_t)(g.kh + 1) * bg.width;                    // tap plane bt - 1
          const bool has0 = live && m.bt < g.kt, has1 = live && m.bt >= 1;
          const unsigned* pg0 = reinterpret_cast<const unsigned*>(gbox + (has0 ? o0 : 0));
          const unsigned* pe0 = reinterpret_cast<const unsigned*>(bbox + (has0 ? o0 : 0));
          const unsigned* pg1 = reinterpret_cast<const unsigned*>(gbox + (has1 ? o1 : 0));
          const unsigned* pe1 = reinterpret_cast<const unsigned*>(bbox + (has1 ? o1 : 0));
#pragma unroll
          for (int w = 0; w < 8; w++) {
            if (w >= words) break;
            const int x0 = m.ox + 2 * w;  // key of box column 2w
            const bool in = x0 + 1 >= 0 && x0 < kKvtKeys;
            gw0[w] = (in && has0) ? __ldg(pg0 + w) : 0u;
            ew0[w] = (in && has0) ? __ldg(pe0 + w) : 0u;
            gw1[w] = (in && has1) ? __ldg(pg1 + w) : 0u;
            ew1[w] = (in && has1) ? __ldg(pe1 + w) : 0u;
          }
        }
        DSA3D_KV_CLK(2);
        if (ls + 1 < nst) snext = slot_load(ls + 1);
        DSA3D_KV_CLK(3);
        // the buffer's previous stage must be consumed (lane 0 waits, the warp follows)
        int rw = 1;
        if (lane == 0 && G >= (uint32_t)kKvtStages)
          rw = mbar_wait(empty(buf), ((G / kKvtStages) - 1) & 1, abort_flag) ? 1 : 0;
        ok = __shfl_sync(kFull, rw, 0) != 0;
        if (!ok) break;
        DSA3D_KV_CLK(4);
        unsigned char* sbase = stages + buf * C::STAGE_BYTES;
        unsigned char* ag = sbase;
        unsigned char* ab = sbase + C::A_BYTES;
        unsigned char* bq = sbase + 2 * C::A_BYTES;
        unsigned char* bo = bq + C::B_BYTES;
        // q and dO rows of the 8 slots (zero for empty ones) into the MN-major B operands: lane
        // copies chunks lane % 4 + 4 j of slot lane / 4's rows
        {
          constexpr int CH = DH / 8;  // 16-byte chunks per row
          const int64_t ro = m.ok ? m.row : 0;
          const __nv_bfloat16* sq = q + ro;
          const __nv_bfloat16* so = dout + ro;
          const int kq = 8 * warp + kl;
#pragma unroll
          for (int j = 0; j < CH / 4; j++) {
            const int c = (lane & 3) + 4 * j;
            const uint32_t dof = kvt_b_off(kq, c >> 3, c & 7);
            cp_async16_zfill(bq + dof, sq + 8 * c, m.ok != 0);
            cp_async16_zfill(bo + dof, so + 8 * c, m.ok != 0);
          }
          cp_async_commit();
        }
        // zeros in the warp's 16-byte column chunk (queries 8 warp ..) of every key row
#pragma unroll
        for (int it = 0; it < 4; it++) {
          const int mr = lane + 32 * it;
          const uint32_t off = (uint32_t)((mr >> 3) * 1024 + (mr & 7) * 128 + ((warp ^ (mr & 7)) << 4));
          *reinterpret_cast<uint4*>(ag + off) = make_uint4(0, 0, 0, 0);
          *reinterpret_cast<uint4*>(ab + off) = make_uint4(0, 0, 0, 0);
        }
        __syncwarp();
        DSA3D_KV_CLK(5);
        {
          // key x of key row r is tile row mk = 4 x + r (the four key rows of a column sit in
          // rows with different swizzle phases, so the four lanes of a slot store to different
          // banks); query k = 8 warp + kl sits in chunk warp ^ (mk & 7) of the row.  A column
          // outside the tile (or an item without a box row here) stores to the warp's scratch word.
          const float D = m.D, ft = m.ft;
          const uint32_t dummy = (uint32_t)(scratch - ag) + 16u * warp;
#pragma unroll
          for (int w = 0; w < 8; w++) {
            if (w >= words) break;
#pragma unroll
            for (int e = 0; e < 2; e++) {
              const int x = m.ox + 2 * w + e;
              const bool in = live && x >= 0 && x < kKvtKeys;
              const float bb0 = __uint_as_float(e ? (ew0[w] & 0xffff0000u) : (ew0[w] << 16));
              const float gg0 = __uint_as_float(e ? (gw0[w] & 0xffff0000u) : (gw0[w] << 16));
              const float bb1 = __uint_as_float(e ? (ew1[w] & 0xffff0000u) : (ew1[w] << 16));
              const float gg1 = __uint_as_float(e ? (gw1[w] & 0xffff0000u) : (gw1[w] << 16));
              const float be = fmaf(ft, bb1 - bb0, bb0);
              const float c0 = fmaf(-D, bb0, gg0), c1 = fmaf(-D, bb1, gg1);
              const float ga = fmaf(ft, c1 - c0, c0);
              const int mk = 4 * x + r;
              const uint32_t off = in ? (uint32_t)(128 * mk + ((warp ^ (mk & 7)) << 4) + 2 * kl) : dummy;
              *reinterpret_cast<unsigned short*>(ag + off) = bf16_bits(ga);
              *reinterpret_cast<unsigned short*>(ag + off + (in ? C::A_BYTES : 0u)) = bf16_bits(be);
            }
          }
        }
        DSA3D_KV_CLK(6);
        // the thread's copies and stores become visible to the tensor cores, then full
        cp_async_wait_all();
        fence_proxy_async_smem();
        mbar_arrive(full(buf));
        DSA3D_KV_CLK(7);
#undef DSA3D_KV_CLK
      }
      gs += (uint32_t)nst;
    }
  } else if (warp < kKvtMmaWarp) {
    // ===================== dK, dV out: thread = key =====================
    const int quarter = warp - kKvtEpiWarp0;  // lanes 32 quarter ..: tile row mk = 32 quarter + lane
    const uint32_t lq = (uint32_t)(32 * quarter) << 16;
    uint32_t tc = 0;
    bool ok = true;
    for (; ok; tc++) {
      const int64_t t = next_tile(tc, ok);
      if (t < 0) break;
      const KvtTile T = kvt_tile(g, sg, t);
      const int total = kvt_total(g, sg, T, start, lane);
      const int buf = (int)(tc & 1);
      int r = 1;
      if (lane == 0) r = mbar_wait(acc_full(buf), (tc >> 1) & 1, abort_flag) ? 1 : 0;
      ok = __shfl_sync(kFull, r, 0) != 0;
      if (!ok) break;
      if (quarter == 0 && lane == 0 && tc < 1000) TC_CLK(12288 + 2 * tc);
      tc_fence_after();
      const int mk = 32 * quarter + lane;  // key x = mk / 4 of key row mk % 4
      const int yk = T.yk0 + (mk & 3), x = T.x_lo + (mk >> 2);
      const bool live = yk < g.Hp && x < g.Wp;
      const int64_t row = (((int64_t)(T.tk * g.Hp + yk) * g.Wp + x) * g.heads + (h0 + T.hh)) * DH;
      const uint32_t acc = tmem + lq + (uint32_t)(buf * 2 * DH);
#pragma unroll
      for (int which = 0; which < 2; which++) {
        const float sc = which ? 1.f : g.scale;
        __nv_bfloat16* dst_base = which ? dv : dk;
#pragma unroll 1
        for (int part = 0; part < DH / 32; part++) {
          uint32_t v[32];
          tmem_ld32(acc + which * DH + 32 * part, v);
          tmem_ld_wait(v);
          if (live) {
            uint4* dst = reinterpret_cast<uint4*>(dst_base + row + 32 * part);
            auto o = [&](int i) { return total > 0 ? sc * __uint_as_float(v[i]) : 0.f; };
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
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(acc_empty(buf));
      if (quarter == 0 && lane == 0 && tc < 1000) TC_CLK(12288 + 2 * tc + 1);
    }
  } else {
    // ===================== UMMA issuer =====================
    uint32_t gs = 0, tc = 0;
    bool ok = true;
    const uint64_t d0 = umma_sdesc_sw128(st0, 16, 1024);                     // A: K-major, 8-row groups
    const uint64_t e0 = umma_sdesc_sw128(st0, C::HALF_BYTES, 1024);          // B: MN-major, 64-dim halves
    for (; ok; tc++) {
      const int64_t t = next_tile(tc, ok);
      if (t < 0) break;
      const KvtTile T = kvt_tile(g, sg, t);
      const int total = kvt_total(g, sg, T, start, lane);
      const int nst = (total + kKvtQ - 1) / kKvtQ;
      const int buf = (int)(tc & 1);
      if (lane == 0) {
        if (tc >= 2 && !mbar_wait(acc_empty(buf), ((tc >> 1) - 1) & 1, abort_flag)) ok = false;
        const uint32_t acc = tmem + (uint32_t)(buf * 2 * DH);
        for (int ls = 0; ls < nst && ok; ls++) {
          const uint32_t G = gs + (uint32_t)ls;
          const int sb = (int)(G % kKvtStages);
          if (G < 2000) TC_CLK(8192 + 2 * G);
          if (!mbar_wait(full(sb), (G / kKvtStages) & 1, abort_flag)) {
            ok = false;
            break;
          }
          if (G < 2000) TC_CLK(8192 + 2 * G + 1);
          tc_fence_after();
          const uint32_t so = (uint32_t)(sb * C::STAGE_BYTES);
#pragma unroll
          for (int ks = 0; ks < kKvtQ / 16; ks++) {
            const uint32_t acc_flag = (ls > 0 || ks > 0) ? 1u : 0u;
            const uint64_t ag = d0 + (uint64_t)((so + 32 * ks) >> 4);
            const uint64_t abt = d0 + (uint64_t)((so + C::A_BYTES + 32 * ks) >> 4);
            const uint64_t bq = e0 + (uint64_t)((so + 2 * C::A_BYTES + 2048 * ks) >> 4);
            const uint64_t bo = e0 + (uint64_t)((so + 2 * C::A_BYTES + C::B_BYTES + 2048 * ks) >> 4);
            umma_ss(acc, ag, bq, C::IDESC, acc_flag);
            umma_ss(acc + DH, abt, bo, C::IDESC, acc_flag);
          }
          umma_commit(empty(sb));
        }
        if (ok) umma_commit(acc_full(buf));
      }
      ok = __shfl_sync(kFull, ok ? 1 : 0, 0) != 0;
      gs += (uint32_t)nst;
    }
    if (lane == 0) {
      // nothing of this thread's may still run when tensor memory is released
      umma_commit(m_done);
      mbar_drain(m_done, 0, abort_flag);
    }
    __syncwarp();
  }

  // release tensor memory once no role can touch it
  tc_fence_before();
  __syncthreads();
  if (warp == kKvtMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, C::COLS);
  }
}

}  // namespace dsa3d
