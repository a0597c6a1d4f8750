// dsa3d_dq_tc.cuh -- the dq pass of the 3D-DSA backward on the 5th-generation tensor cores
// (tcgen05 UMMA with the accumulator in tensor memory), dh = 128.
//
// dq = scale * sum_j gamma[j] K[j] over the box tokens j of each query (MegaSlide-DiT,
// arXiv 2607.22696, Eq. 1, differentiated with respect to q; gamma = gamma' - D beta and the t-mix
// of the two tap planes feeding each box plane, from the query-side pass's stored splats).  For one
// chunk of <= 16 queries (the forward's chunks) the transposed product
//     dq^T [dh = 128 dims x 16 queries] = sum over box rows  K_seg^T [128 x 32 keys] . gamma^T [32 x 16]
// is an M = 128, N = 16 UMMA per box row (two K = 16 halves), accumulated in 16 columns of tensor
// memory (lane = dim, column = query).  The four warps of a CTA work on one chunk at a time: per box
// row they copy the 32-key segment of K (cp.async, in the UMMA's MN-major layout) and build the gamma
// tile (K-major layout) into one of two shared buffers; one thread issues the two MMAs and commits
// them to that buffer's mbarrier, which gates the buffer's next refill.  At the end of a chunk each
// warp reads its 32 lanes (dims) of the accumulator and writes dq.
//
// Layouts (no swizzle; "core matrix" = 8 rows of 16 bytes, 128 contiguous bytes):
//   A = K_seg^T, MN-major: core matrix (dim group g, key group c) holds keys 8c..8c+7 as rows, each
//       row the 8 dims 8g..8g+7 of that key; offset g * kTcSbo + c * 128 + (key % 8) * 16.
//   B = gamma^T, K-major: core matrix (query group r, key group c) holds queries 8r..8r+7 as rows,
//       each row the 8 keys 8c..8c+7; offset r * 512 + c * 128 + (query % 8) * 16.
// The leading byte offset (between key groups) is 128 for both; the stride byte offsets (between
// dim groups / query groups) are kTcSbo and 512.  kTcSbo = 528 spreads the 16 dim groups of one
// key over distinct bank slots for the copies.
#pragma once

#include "dsa3d_bwd_mma.cuh"

namespace dsa3d {

constexpr int kTcSbo = 528;                 // bytes between dim groups of the A tile
constexpr int kTcABytes = 16 * kTcSbo;      // one A buffer (16 dim groups)
constexpr int kTcBBytes = 2 * 512;          // one B buffer (2 query groups x 4 key groups)
constexpr int kTcCols = 32;                 // tensor-memory columns allocated per CTA (>= 16)
constexpr unsigned kTcWaitLimit = 1u << 26; // polls of an mbarrier before giving up
constexpr int kTcCtasPerSm = 8;             // resident CTAs per SM: 8 x kTcCols <= 512 TMEM columns

__host__ __device__ constexpr int dq_tc_smem_bytes() {
  return 2 * kTcABytes + 2 * kTcBBytes + 16 * 16 + 64;
}

// UMMA shared-memory descriptor, no swizzle: start address, leading / stride byte offsets (all in
// 16-byte units), descriptor version 1.
__device__ __forceinline__ uint64_t umma_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
  d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
  d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
  d |= (uint64_t)1 << 46;  // version
  return d;                // base offset 0, leading-offset mode 0, layout type 0 (no swizzle)
}

// Instruction descriptor of kind::f16: bf16 A and B, fp32 accumulator, A MN-major, B K-major,
// N = 16, M = 128.
constexpr uint32_t kTcIdesc = (1u << 4)      // accumulator format f32
                              | (1u << 7)    // A format bf16
                              | (1u << 10)   // B format bf16
                              | (1u << 15)   // A major: MN
                              | (0u << 16)   // B major: K
                              | (2u << 17)   // N >> 3
                              | (8u << 24);  // M >> 4

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t .reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// Wait for the phase of parity `parity` of the mbarrier to complete, at most kTcWaitLimit polls;
// on timeout the device check flag records it (dsa3d_check_device reports it) and false returns.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity) {
  for (unsigned i = 0; i < kTcWaitLimit; i++)
    if (mbar_try_wait(bar, parity)) return true;
  atomicExch(&g_dsa3d_check, 2);
  return false;
}

template <int DH>
__global__ void __launch_bounds__(128, kTcCtasPerSm)
    dsa3d_bwd_dq_tc_kernel(const __nv_bfloat16* __restrict__ k, __nv_bfloat16* __restrict__ dq,
                           const int* __restrict__ start, const int* __restrict__ sorted_n,
                           const int* __restrict__ sorted_ex, const unsigned short* __restrict__ gbox,
                           const unsigned short* __restrict__ bbox, const float2* __restrict__ dft,
                           const Geo g, const SortGeo sg, const BoxGeo bg, const int h0, const int hg) {
  static_assert(DH == 128, "M = 128 dims per UMMA");
  extern __shared__ __align__(1024) unsigned char tc_sh[];
  unsigned char* abuf = tc_sh;                                   // [2][kTcABytes]
  unsigned char* bbuf = tc_sh + 2 * kTcABytes;                   // [2][kTcBBytes]
  int4* qinfo = reinterpret_cast<int4*>(bbuf + 2 * kTcBBytes);   // [16]: token, col0, D, f_t
  uint64_t* mbar = reinterpret_cast<uint64_t*>(qinfo + 16);      // [2]
  uint32_t* tslot = reinterpret_cast<uint32_t*>(mbar + 2);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t a_s = (uint32_t)__cvta_generic_to_shared(abuf);
  const uint32_t b_s = (uint32_t)__cvta_generic_to_shared(bbuf);
  const uint32_t bar_s = (uint32_t)__cvta_generic_to_shared(mbar);

  // tensor memory: warp 0 allocates kTcCols columns for the CTA's accumulator
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     (uint32_t)__cvta_generic_to_shared(tslot)),
                 "r"(kTcCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  if (tid == 0) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(bar_s) : "memory");
    asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(bar_s + 8) : "memory");
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
  const uint32_t tmem = *tslot;

  const int64_t rs = (int64_t)g.heads * DH;
  const int segw = segment_keys(g.kw);
  const int64_t rows = (int64_t)hg * sg.Et * sg.Ey;
  uint32_t commits[2] = {0u, 0u};  // commits issued on each buffer's mbarrier (same in every thread)
  bool ok = true;                  // false after a wait gave up: the CTA then stops issuing work
  // thread 0 waits for a commit; the barrier hands the outcome (the same in every thread) and the
  // ordering to the whole CTA
  auto wait_commit = [&](int b) {
    const bool mine = (tid == 0) ? mbar_wait(bar_s + 8 * b, (commits[b] - 1) & 1) : true;
    return __syncthreads_and(mine) != 0;
  };

  for (int64_t row = blockIdx.x; row < rows && ok; row += gridDim.x) {
    const int hh = (int)(row / ((int64_t)sg.Et * sg.Ey));
    const int rem = (int)(row - (int64_t)hh * sg.Et * sg.Ey);
    const int et = rem / sg.Ey, ey = rem % sg.Ey;
    const int h = h0 + hh;
    const int64_t b0 = (int64_t)hh * sg.E1 + ((int64_t)et * sg.Ey + ey) * sg.Ex;
    const int qbeg = start[b0], qend = start[b0 + sg.Ex];
    const int ot = et - g.kt, oy = ey - g.kh;
    const __nv_bfloat16* kh_ = k + (int64_t)h * DH;
    const int bt0 = max(0, -ot), bt1 = min(g.kt, g.F - 1 - ot);
    const int by0 = max(0, -oy), by1 = min(g.kh, g.Hp - 1 - oy);
    const int nby = by1 - by0 + 1;
    const int nsteps = (bt1 >= bt0 && by1 >= by0) ? (bt1 - bt0 + 1) * nby : 0;

    for (int pos = qbeg; pos < qend && ok;) {
      int X0;
      const int cnt = chunk_len(sorted_ex, pos, qend, g.kw, lane, X0);  // the same in every warp
      if (tid < 16) {
        int4 qi = make_int4(-1, 0, 0, 0);
        if (tid < cnt) {
          const float2 d = dft[pos + tid];
          qi = make_int4(sorted_n[pos + tid], sorted_ex[pos + tid] - g.kw - X0, __float_as_int(d.x),
                         __float_as_int(d.y));
        }
        qinfo[tid] = qi;
      }
      __syncthreads();

      for (int s = 0; s < nsteps && ok; s++) {
        const int b = s & 1;
        const int bt = bt0 + s / nby, by = by0 + s % nby;
        // the MMAs that last read buffer b are done before it is refilled
        if (commits[b] > 0) ok = wait_commit(b);
        if (!ok) break;
        // A: the K segment of key row (ot + bt, oy + by), keys X0 .. X0 + 31; thread t copies the
        // 16-byte chunks (key, dim group) = (t / 16 + 8 i, t % 16)
        {
          const __nv_bfloat16* krow = kh_ + (int64_t)((ot + bt) * g.Hp + oy + by) * g.Wp * rs;
          unsigned char* dst = abuf + b * kTcABytes;
#pragma unroll
          for (int i = 0; i < 4; i++) {
            const int key = tid / 16 + 8 * i, dg = tid % 16;
            const int x = X0 + key;
            const bool in = key < segw && x >= 0 && x < g.Wp;
            const __nv_bfloat16* src = in ? krow + (int64_t)x * rs + 8 * dg : krow;
            cp_async16_zfill(dst + dg * kTcSbo + (key >> 3) * 128 + (key & 7) * 16, src, in);
          }
          cp_async_commit();
        }
        // B: gamma of (query r, keys 8c .. 8c+7) for thread t < 64 = (r, c) = (t / 4, t % 4)
        if (tid < 64) {
          const int r = tid >> 2, c = tid & 3;
          const int4 qi = qinfo[r];
          float gv[8];
#pragma unroll
          for (int e = 0; e < 8; e++) gv[e] = 0.f;
          if (qi.x >= 0) {
            const float D = __int_as_float(qi.z), ft = __int_as_float(qi.w);
            const int64_t qb = (int64_t)(pos + r) * bg.per_q;
            const int o0 = (bt * (g.kh + 1) + by) * bg.width, o1 = o0 - (g.kh + 1) * bg.width;
#pragma unroll
            for (int e = 0; e < 8; e++) {
              const int bx = 8 * c + e - qi.y;
              if (bx < 0 || bx >= bg.width) continue;
              float c0 = 0.f, c1 = 0.f;
              if (bt < g.kt) c0 = fmaf(-D, bf16_val(bbox[qb + o0 + bx]), bf16_val(gbox[qb + o0 + bx]));
              if (bt >= 1) c1 = fmaf(-D, bf16_val(bbox[qb + o1 + bx]), bf16_val(gbox[qb + o1 + bx]));
              gv[e] = fmaf(ft, c1 - c0, c0);
            }
          }
          uint4 w;
          w.x = bf16x2_bits(gv[0], gv[1]);
          w.y = bf16x2_bits(gv[2], gv[3]);
          w.z = bf16x2_bits(gv[4], gv[5]);
          w.w = bf16x2_bits(gv[6], gv[7]);
          *reinterpret_cast<uint4*>(bbuf + b * kTcBBytes + (r >> 3) * 512 + c * 128 + (r & 7) * 16) = w;
        }
        cp_async_wait_all();
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // make the tiles visible to UMMA
        __syncthreads();
        if (tid == 0) {
          asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
#pragma unroll
          for (int half = 0; half < 2; half++) {  // keys 16 half .. 16 half + 15
            const uint64_t ad = umma_desc(a_s + b * kTcABytes + half * 256, 128, kTcSbo);
            const uint64_t bd = umma_desc(b_s + b * kTcBBytes + half * 256, 128, 512);
            const uint32_t acc = (s > 0 || half > 0) ? 1u : 0u;
            asm volatile(
                "{\n\t .reg .pred p;\n\t"
                "setp.ne.b32 p, %4, 0;\n\t"
                "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}"
                ::"r"(tmem), "l"(ad), "l"(bd), "r"(kTcIdesc), "r"(acc)
                : "memory");
          }
          asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                           bar_s + 8 * b)
                       : "memory");
        }
        commits[b]++;
      }
      if (!ok) break;

      // epilogue: wait for the chunk's last MMAs, then warp w reads dims 32w + lane of the 16 queries
      float v[16];
#pragma unroll
      for (int j = 0; j < 16; j++) v[j] = 0.f;
      if (nsteps > 0) {
        ok = wait_commit((nsteps - 1) & 1);
        if (ok) {
          asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
          uint32_t r[16];
          asm volatile(
              "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, "
              "%12, %13, %14, %15}, [%16];"
              : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
                "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
                "=r"(r[14]), "=r"(r[15])
              : "r"(tmem + ((uint32_t)(32 * warp) << 16)));
          asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
          for (int j = 0; j < 16; j++) v[j] = __uint_as_float(r[j]);
        }
      }
      const int dim = 32 * warp + lane;
#pragma unroll
      for (int j = 0; j < 16; j++) {
        const int n = qinfo[j].x;
        if (n >= 0) dq[((int64_t)n * g.heads + h) * DH + dim] = __float2bfloat16_rn(v[j] * g.scale);
      }
      asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
      __syncthreads();  // the accumulator and the query slots are free for the next chunk
      pos += cnt;
    }
  }

  // every commit has been waited on (the last one of each chunk covers the earlier ones); free the
  // tensor memory
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  if (warp == 0) {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTcCols)
                 : "memory");
  }
}

}  // namespace dsa3d
