// dsa3d_bwd_dq_tc.cuh -- dq of the 3D-DSA backward on the 5th-generation tensor cores (bf16 I/O,
// dh 64 or 128, k_w <= 15).
//
// The derivative of Eq. 1 (MegaSlide-DiT, arXiv 2607.22696) with respect to a query is
//   dq = scale * sum_tau P_tau (dP_tau - D) k~_tau = scale * sum_box gamma_box K_box,
// gamma the trilinear splat of P (dP - D) onto the query's box.  The query side
// (dsa3d_bwd_q_kernel) stores, per query and tap plane u, the y/x splats of P (beta) and P dP
// (gamma') on the box rows, and D and f_t; tap plane u's gamma = gamma' - D beta feeds box plane u
// with weight 1 - f_t and box plane u + 1 with weight f_t.
//
// Work unit: the forward's tile of the window-origin sort (dsa3d_fwd_tc.cuh): up to 128 queries of
// a pass on the tensor-memory lanes, the pass's union rows, the 32-key segment.  For tap plane u
// and union row j one UMMA chain adds
//   dq[q][:] += [(1 - f_t) gamma_u | f_t gamma_u][q][64 keys] . [K[u, j]; K[u + 1, j]]
// (M = 128 queries, N = dh, K = 64 keys of the two planes), A from shared memory (each writer
// thread fills its query's row: zeros, then its box row's kw + 1 values at keys eox .. eox + kw),
// B the K pair of the forward (5-D TMA box, 128-byte swizzle, MN-major).  dq of a pass sits in
// tensor memory (two accumulators alternate between passes); the writers scale and store it.
//
// Roles (192 threads): warps 0-3 write the A rows and dq (thread = tensor-memory lane = query of
// the pass), warp 4 the TMA producer of the K pairs (it also draws the tiles), warp 5 the UMMA
// issuer (it also owns the tensor-memory allocation).  mbarriers order everything; every wait is
// bounded (dsa3d_tc.cuh).
#pragma once

#include "dsa3d_bwd_mma.cuh"
#include "dsa3d_fwd_tc.cuh"
#include "dsa3d_sort.cuh"
#include "dsa3d_tc.cuh"

namespace dsa3d {

constexpr int kDqtThreads = 192;
constexpr int kDqtKWarp = 4, kDqtMmaWarp = 5;
constexpr int kDqtKStages = 3;  // K pair ring
constexpr int kDqtABufs = 3;    // A tiles

template <int DH>
struct DqtCfg {
  static constexpr int HALVES = DH / 64;
  static constexpr int PAIR_BYTES = 2 * kTcSeg * DH * 2;
  static constexpr int A_BYTES = 128 * 64 * 2;  // 128 queries x 64 keys
  static constexpr int STAGE_BYTES = kDqtKStages * PAIR_BYTES + kDqtABufs * A_BYTES;
  static constexpr int BAR_BYTES = 256;
  static constexpr int SMEM_BYTES = STAGE_BYTES + BAR_BYTES + 1024;
  static constexpr int COLS = (2 * DH <= 128) ? 128 : 256;  // two dq accumulators
  static constexpr uint32_t IDESC = umma_idesc_bf16(128, DH, false, true);
  static_assert(SMEM_BYTES <= 113 * 1024, "two CTAs per SM");
};

template <int DH>
__global__ void __launch_bounds__(kDqtThreads, 2)
    dsa3d_bwd_dq_tc_kernel(const __grid_constant__ CUtensorMap tmk, __nv_bfloat16* __restrict__ dq,
                           const int* __restrict__ start, const int* __restrict__ sorted_n,
                           const int* __restrict__ sorted_ex, const unsigned short* __restrict__ gbox,
                           const unsigned short* __restrict__ bbox, const float2* __restrict__ dft,
                           int* __restrict__ tile_counter, const Geo g, const SortGeo sg, const BoxGeo bg,
                           const TcTileGeo tg, const int h0) {
  using C = DqtCfg<DH>;
  extern __shared__ __align__(1024) unsigned char dqt_smem[];
  unsigned char* stages = dqt_smem + ((1024 - (smem_u32(dqt_smem) & 1023)) & 1023);
  const uint32_t kst = smem_u32(stages);
  unsigned char* abuf = stages + kDqtKStages * C::PAIR_BYTES;
  const uint32_t ast = smem_u32(abuf);
  uint64_t* bars = reinterpret_cast<uint64_t*>(stages + C::STAGE_BYTES);
  const uint32_t b0 = smem_u32(bars);
  auto k_full = [&](int s) { return b0 + 8u * s; };
  auto k_empty = [&](int s) { return b0 + 8u * (kDqtKStages + s); };
  constexpr int BA = 2 * kDqtKStages, BC = BA + 2 * kDqtABufs;  // first A, first accumulator barrier
  auto a_full = [&](int s) { return b0 + 8u * (BA + s); };
  auto a_empty = [&](int s) { return b0 + 8u * (BA + kDqtABufs + s); };
  auto acc_full = [&](int s) { return b0 + 8u * (BC + s); };
  auto acc_empty = [&](int s) { return b0 + 8u * (BC + 2 + s); };
  const uint32_t m_done = b0 + 8u * (BC + 4);
  auto tile_full = [&](int s) { return b0 + 8u * (BC + 5 + s); };
  auto tile_empty = [&](int s) { return b0 + 8u * (BC + 5 + kTcTileRing + s); };
  uint32_t* tslot = reinterpret_cast<uint32_t*>(bars + 28);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tslot + 1);
  volatile int* tile_ring = reinterpret_cast<volatile int*>(tslot + 2);
  static_assert((BC + 5 + 2 * kTcTileRing) * 8 <= 224 && 232 + 4 * kTcTileRing <= C::BAR_BYTES,
                "barrier slots");

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kDqtKStages; s++) {
      mbar_init(k_full(s), 1);
      mbar_init(k_empty(s), 1);
    }
    for (int s = 0; s < kDqtABufs; s++) {
      mbar_init(a_full(s), 128);
      mbar_init(a_empty(s), 1);
    }
    for (int s = 0; s < 2; s++) {
      mbar_init(acc_full(s), 1);
      mbar_init(acc_empty(s), 4);
    }
    mbar_init(m_done, 1);
    for (int s = 0; s < kTcTileRing; s++) {
      mbar_init(tile_full(s), 1);
      mbar_init(tile_empty(s), kDqtThreads / 32);
    }
    *abort_flag = 0;
    mbar_fence_init();
  }
  if (warp == kDqtMmaWarp) tmem_alloc(smem_u32(tslot), C::COLS);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tslot;
  // tiles in order from a counter shared by the CTAs (as in the forward): the K producer draws the
  // CTA's k-th tile into slot k % kTcTileRing of a ring that one thread of every warp reads
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

  if (warp == kDqtKWarp) {
    // ===================== TMA producer of the K pairs (and the tile draws) =====================
    if (lane == 0) {
      tma_prefetch_desc(&tmk);
      uint32_t cnt = 0;
      bool ok = true;
      for (uint32_t k = 0; ok; k++) {
        const int64_t t = tile_at(k, true, ok);
        if (t < 0) break;
        TcTile T;
        tc_tile(tg, sg, start, t, T);
        const int passes = (T.cnt + 127) / 128;
        const int ot = T.et - g.kt, Xs = T.X0 - g.kw, hd = (h0 + T.hh) * C::HALVES;
        for (int ps = 0; ps < passes && ok; ps++) {
          int j0, up;
          tc_pass_rows(T, ps, g.kh, j0, up);
          for (int u = 0; u < g.kt && ok; u++)
            for (int j = 0; j < up && ok; j++, cnt++) {
              const int s = (int)(cnt % kDqtKStages);
              if (cnt >= (uint32_t)kDqtKStages &&
                  !mbar_wait(k_empty(s), ((cnt / kDqtKStages) - 1) & 1, abort_flag)) {
                ok = false;
                break;
              }
              mbar_arrive_expect_tx(k_full(s), C::PAIR_BYTES);
#pragma unroll
              for (int hv = 0; hv < C::HALVES; hv++)
                tma_load_5d(kst + s * C::PAIR_BYTES + hv * (C::PAIR_BYTES / C::HALVES), &tmk, k_full(s), 0,
                            hd + hv, Xs, T.Y0 - g.kh + j0 + j, ot + u);
            }
        }
      }
      for (uint32_t i = (cnt > (uint32_t)kDqtKStages ? cnt - kDqtKStages : 0); i < cnt; i++)
        mbar_drain(k_full(i % kDqtKStages), (i / kDqtKStages) & 1, abort_flag);
    }
  } else if (warp == kDqtMmaWarp) {
    // ===================== UMMA issuer =====================
    if (lane == 0) {
      uint32_t kc = 0, ac = 0, npass = 0;
      bool ok = true;
      const uint64_t ad0 = umma_sdesc_sw128(ast, 16, 1024);                             // A: K-major
      const uint64_t bd0 = umma_sdesc_sw128(kst, C::PAIR_BYTES / C::HALVES, 1024);      // B: MN-major
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
          const int ab = (int)(npass & 1);
          const uint32_t acc = tmem + (uint32_t)(ab * DH);
          if (npass >= 2 && !mbar_wait(acc_empty(ab), ((npass >> 1) - 1) & 1, abort_flag)) {
            ok = false;
            break;
          }
          for (int r = 0; r < rows && ok; r++, kc++, ac++) {
            const int ks_ = (int)(kc % kDqtKStages), as_ = (int)(ac % kDqtABufs);
            if (!mbar_wait(k_full(ks_), (kc / kDqtKStages) & 1, abort_flag) ||
                !mbar_wait(a_full(as_), (ac / kDqtABufs) & 1, abort_flag)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint64_t a0 = ad0 + (uint64_t)((as_ * C::A_BYTES) >> 4);
            const uint64_t bq = bd0 + (uint64_t)((ks_ * C::PAIR_BYTES) >> 4);
#pragma unroll
            for (int ks = 0; ks < 4; ks++)
              umma_ss(acc, a0 + (uint64_t)((32 * ks) >> 4), bq + (uint64_t)((2048 * ks) >> 4), C::IDESC,
                      (r > 0 || ks > 0) ? 1u : 0u);
            umma_commit(k_empty(ks_));
            umma_commit(a_empty(as_));
          }
          if (ok) umma_commit(acc_full(ab));
        }
      }
      umma_commit(m_done);
      mbar_drain(m_done, 0, abort_flag);
    }
  } else {
    // ===================== A rows and dq: thread = tensor-memory lane = query of the pass =====================
    const uint32_t lq = (uint32_t)(32 * warp) << 16;
    const int qslot = 32 * warp + lane;
    const float sc = g.scale;
    uint32_t ac = 0, npass = 0;
    bool ok = true;
    auto wwait = [&](uint32_t bar, uint32_t parity) {
      int r = 1;
      if (lane == 0) r = mbar_wait(bar, parity, abort_flag) ? 1 : 0;
      return __shfl_sync(kFull, r, 0) != 0;
    };
    // this thread's row of an A tile: 128 bytes at 128 qslot, 16-byte chunk c at c ^ (qslot & 7)
    auto a_off = [&](int key) {
      return (uint32_t)(128 * qslot + ((((key >> 3) ^ (qslot & 7)) << 4) | ((key & 7) << 1)));
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
        const int qi = ps * 128 + qslot;
        const bool live = qi < T.cnt;
        int n = 0, eox = 0, dy = 0;
        int64_t box = 0;
        float D = 0.f, ft = 0.f;
        if (live) {
          int r = qi, i = 0;
          while (i < kTcRyMax - 1 && r >= T.rn[i]) r -= T.rn[i++];
          const int pos = T.r0[i] + r;
          n = sorted_n[pos];
          eox = sorted_ex[pos] - T.X0;
          dy = i;
          box = (int64_t)pos * bg.per_q;
          const float2 d = dft[pos];
          D = d.x;
          ft = d.y;
        }
        int j0, up;
        tc_pass_rows(T, ps, g.kh, j0, up);
        const int words = bg.width >> 1;
        // the box row of step (u, jj) is by = j0 + jj - dy; its words are loaded one step ahead
        auto load_row = [&](int u, int jj, unsigned (&gw)[8], unsigned (&bw)[8]) {
          const int by = j0 + jj - dy;
          const bool has = live && by >= 0 && by <= g.kh;
          const int64_t o = box + (int64_t)(u * (g.kh + 1) + (has ? by : 0)) * bg.width;
          const unsigned* pg = reinterpret_cast<const unsigned*>(gbox + o);
          const unsigned* pb = reinterpret_cast<const unsigned*>(bbox + o);
#pragma unroll
          for (int w = 0; w < 8; w++) {
            gw[w] = (has && w < words) ? __ldg(pg + w) : 0u;
            bw[w] = (has && w < words) ? __ldg(pb + w) : 0u;
          }
        };
        unsigned gn[8], bn[8];
        load_row(0, 0, gn, bn);
        for (int u = 0; u < g.kt && ok; u++) {
          for (int jj = 0; jj < up && ok; jj++, ac++) {
            unsigned gw[8], bw[8];
#pragma unroll
            for (int w = 0; w < 8; w++) {
              gw[w] = gn[w];
              bw[w] = bn[w];
            }
            {
              const int nu = (jj + 1 < up) ? u : u + 1, nj = (jj + 1 < up) ? jj + 1 : 0;
              if (nu < g.kt) load_row(nu, nj, gn, bn);
            }
            const int as_ = (int)(ac % kDqtABufs);
            if (ac >= (uint32_t)kDqtABufs) {
              ok = wwait(a_empty(as_), ((ac / kDqtABufs) - 1) & 1);
              if (!ok) break;
            }
            unsigned char* arow = abuf + as_ * C::A_BYTES;
            {
              // chunk c ^ (qslot & 7) in round c: eight consecutive lanes cover all 32 banks
              unsigned char* z = arow + 128 * qslot;
#pragma unroll
              for (int c = 0; c < 8; c++)
                *reinterpret_cast<uint4*>(z + ((c ^ (qslot & 7)) << 4)) = make_uint4(0, 0, 0, 0);
            }
            const int by = j0 + jj - dy;
            if (live && by >= 0 && by <= g.kh) {
              const float w0 = 1.f - ft;
              // box column c is key eox + c (eox + kw <= 31).  The values go out as 32-bit key
              // pairs from the even key at or below eox: pair m holds columns 2m, 2m + 1 (eox even)
              // or 2m - 1, 2m (eox odd; the columns -1 and kw + 1 are the zeros beside the box row,
              // keys eox - 1 >= 0 and eox + kw + 1 <= 31)
              auto lo = [&](int w) { return fmaf(-D, __uint_as_float(bw[w] << 16), __uint_as_float(gw[w] << 16)); };
              auto hi = [&](int w) {
                return fmaf(-D, __uint_as_float(bw[w] & 0xffff0000u), __uint_as_float(gw[w] & 0xffff0000u));
              };
              const bool odd = (eox & 1) != 0;
              const int np = words + (odd ? 1 : 0), k0 = eox & ~1;
#pragma unroll
              for (int m = 0; m < 9; m++) {
                if (m >= np) continue;
                const float a = odd ? (m > 0 ? hi(m > 0 ? m - 1 : 0) : 0.f) : lo(m < 8 ? m : 7);
                const float b = odd ? (m < words ? lo(m < 8 ? m : 7) : 0.f) : hi(m < 8 ? m : 7);
                const int key = k0 + 2 * m;
                *reinterpret_cast<unsigned*>(arow + a_off(key)) = bf16x2_bits(w0 * a, w0 * b);
                *reinterpret_cast<unsigned*>(arow + a_off(32 + key)) = bf16x2_bits(ft * a, ft * b);
              }
            }
            // this thread's stores become visible to the tensor cores, then it arrives
            fence_proxy_async_smem();
            mbar_arrive(a_full(as_));
          }
        }
        if (!ok) break;
        // ---- this pass's dq rows
        const int ab = (int)(npass & 1);
        ok = wwait(acc_full(ab), (npass >> 1) & 1);
        if (!ok) break;
        tc_fence_after();
        const uint32_t acc = tmem + lq + (uint32_t)(ab * DH);
#pragma unroll 1
        for (int part = 0; part < DH / 32; part++) {
          uint32_t v[32];
          tmem_ld32(acc + 32 * part, v);
          tmem_ld_wait(v);
          if (live) {
            uint4* dst = reinterpret_cast<uint4*>(dq + ((int64_t)n * g.heads + h) * DH + 32 * part);
#pragma unroll
            for (int i = 0; i < 4; i++) {
              uint4 w4;
              w4.x = bf16x2_bits(sc * __uint_as_float(v[8 * i]), sc * __uint_as_float(v[8 * i + 1]));
              w4.y = bf16x2_bits(sc * __uint_as_float(v[8 * i + 2]), sc * __uint_as_float(v[8 * i + 3]));
              w4.z = bf16x2_bits(sc * __uint_as_float(v[8 * i + 4]), sc * __uint_as_float(v[8 * i + 5]));
              w4.w = bf16x2_bits(sc * __uint_as_float(v[8 * i + 6]), sc * __uint_as_float(v[8 * i + 7]));
              dst[i] = w4;
            }
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(acc_empty(ab));
      }
    }
  }

  // release tensor memory once no role can touch it
  tc_fence_before();
  __syncthreads();
  if (warp == kDqtMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, C::COLS);
  }
}

}  // namespace dsa3d
