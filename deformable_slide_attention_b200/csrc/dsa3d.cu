// dsa3d.cu -- C ABI of the 3D-DSA library: argument validation, launch configuration and the
// extern "C" entry points declared in include/dsa3d.h.  All device work is in the kernels of
// dsa3d_*.cuh headers; this file allocates no device memory.
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cmath>
#include <cstdlib>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "dsa3d.h"
#include "dsa3d_bwd.cuh"
#include "dsa3d_bwd_dq_tc.cuh"
#include "dsa3d_bwd_kv_tc.cuh"
#include "dsa3d_bwd_mma.cuh"
#include "dsa3d_fwd.cuh"
#include "dsa3d_fwd_mma.cuh"
#include "dsa3d_fwd_tc.cuh"
#include "dsa3d_sort.cuh"
#include "dsa3d_taps.cuh"
#include "dsa3d_timing.cuh"

namespace dsa3d {
namespace {

constexpr int kWarps = 4;  // warps per CTA (one (head, query) item per warp at a time)

struct Shape {
  int F, Hp, Wp, heads, dh, kt, kh, kw;
  int64_t N;
};

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

struct Range {
  uintptr_t lo, hi;
};
Range range_of(const void* p, size_t bytes) {
  const uintptr_t a = reinterpret_cast<uintptr_t>(p);
  return {a, a + bytes};
}
bool overlap(Range a, Range b) { return a.lo < b.hi && b.lo < a.hi; }

size_t elem_size(dsa3d_dtype_t t) { return t == DSA3D_F32 ? 4 : 2; }

Geo make_geo(const Shape& s) {
  Geo g;
  g.F = s.F; g.Hp = s.Hp; g.Wp = s.Wp; g.heads = s.heads;
  g.kt = s.kt; g.kh = s.kh; g.kw = s.kw;
  g.Bt = s.kt + 1; g.Bh = s.kh + 1; g.Bw = s.kw + 1;
  g.B = g.Bt * g.Bh * g.Bw;
  g.K = s.kt * s.kh * s.kw;
  g.HW = s.Hp * s.Wp;
  g.N = s.N;
  g.scale = 1.0f / std::sqrt((float)s.dh);
  return g;
}

// Shape checks shared by every entry point.
dsa3d_status_t check_shape(const Shape& s, dsa3d_dtype_t dtype, int warp_bytes_per_box_elem) {
  (void)warp_bytes_per_box_elem;
  if (dtype != DSA3D_F32 && dtype != DSA3D_BF16) return DSA3D_ERR_INVALID_ARGUMENT;
  if (s.F < 1 || s.Hp < 1 || s.Wp < 1 || s.heads < 1 || s.dh < 1) return DSA3D_ERR_INVALID_ARGUMENT;
  const int dims[3] = {s.F, s.Hp, s.Wp}, win[3] = {s.kt, s.kh, s.kw};
  for (int a = 0; a < 3; a++) {
    if (win[a] < 1 || (win[a] & 1) == 0) return DSA3D_ERR_INVALID_ARGUMENT;
    if ((int64_t)win[a] > 2 * (int64_t)dims[a] - 1 || win[a] > 1022) return DSA3D_ERR_UNSUPPORTED;
  }
  if (s.dh != 32 && s.dh != 64 && s.dh != 128) return DSA3D_ERR_UNSUPPORTED;
  const int64_t N = (int64_t)s.F * s.Hp * s.Wp;
  if (N >= (int64_t(1) << 31)) return DSA3D_ERR_UNSUPPORTED;
  if ((double)N * s.heads * s.dh >= 4.0e18) return DSA3D_ERR_UNSUPPORTED;
  const int64_t B = (int64_t)(s.kt + 1) * (s.kh + 1) * (s.kw + 1);
  if (B > 32767) return DSA3D_ERR_UNSUPPORTED;  // box indices are stored as int16
  return DSA3D_OK;
}

int smem_bytes(const Geo& g, int warps, bool backward) {
  return table_smem(g.B, g.K) + warps * (backward ? bwd_warp_smem(g.B, g.K) : fwd_warp_smem(g.B, g.K));
}

// Choose warps per CTA so that the dynamic shared memory fits; 0 if even one warp does not.
int pick_warps(const Geo& g, bool backward, int max_smem) {
  for (int w = kWarps; w >= 1; w >>= 1)
    if (smem_bytes(g, w, backward) <= max_smem) return w;
  return 0;
}

struct DeviceInfo {
  int sms = 0;
  int max_smem = 0;
};
DeviceInfo device_info() {
  DeviceInfo d;
  int dev = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev);
  cudaDeviceGetAttribute(&d.max_smem, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
  return d;
}

template <typename Kern>
dsa3d_status_t launch_persistent(Kern kern, int warps, int smem, int64_t items, cudaStream_t st,
                                 int& grid_out) {
  const DeviceInfo d = device_info();
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
    return DSA3D_ERR_CUDA;
  int per_sm = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, warps * 32, smem) != cudaSuccess)
    return DSA3D_ERR_CUDA;
  if (per_sm < 1) return DSA3D_ERR_UNSUPPORTED;
  const int64_t need = (items + warps - 1) / warps;
  int64_t grid = (int64_t)d.sms * per_sm;
  if (need < grid) grid = need;
  if (grid < 1) grid = 1;
  grid_out = (int)grid;
  (void)st;
  return DSA3D_OK;
}

template <typename T, int DH, int W>
dsa3d_status_t fwd_launch(const Shape& s, const void* q, const void* k, const void* v,
                          const float* off, void* out, float* lse, cudaStream_t st) {
  const Geo g = make_geo(s);
  const int smem = smem_bytes(g, W, false);
  auto kern = dsa3d_fwd_kernel<T, DH, W>;
  int grid = 0;
  const int64_t items = (int64_t)s.heads * s.N;
  dsa3d_status_t rc = launch_persistent(kern, W, smem, items, st, grid);
  if (rc != DSA3D_OK) return rc;
  TimedLaunch tl(kKernFwd, st);
  kern<<<grid, W * 32, smem, st>>>(static_cast<const T*>(q), static_cast<const T*>(k),
                                   static_cast<const T*>(v), off, static_cast<T*>(out), lse, g, items);
  const bool launched = cudaGetLastError() == cudaSuccess;
  return (tl.finish() && launched) ? DSA3D_OK : DSA3D_ERR_CUDA;
}

template <typename T, int DH>
dsa3d_status_t fwd_dispatch_w(const Shape& s, int warps, const void* q, const void* k,
                              const void* v, const float* off, void* out, float* lse,
                              cudaStream_t st) {
  switch (warps) {
    case 4: return fwd_launch<T, DH, 4>(s, q, k, v, off, out, lse, st);
    case 2: return fwd_launch<T, DH, 2>(s, q, k, v, off, out, lse, st);
    case 1: return fwd_launch<T, DH, 1>(s, q, k, v, off, out, lse, st);
    default: return DSA3D_ERR_UNSUPPORTED;
  }
}

template <typename T>
dsa3d_status_t fwd_dispatch(const Shape& s, int warps, const void* q, const void* k, const void* v,
                            const float* off, void* out, float* lse, cudaStream_t st) {
  switch (s.dh) {
    case 32: return fwd_dispatch_w<T, 32>(s, warps, q, k, v, off, out, lse, st);
    case 64: return fwd_dispatch_w<T, 64>(s, warps, q, k, v, off, out, lse, st);
    case 128: return fwd_dispatch_w<T, 128>(s, warps, q, k, v, off, out, lse, st);
    default: return DSA3D_ERR_UNSUPPORTED;
  }
}

// --- sorted tensor-core forward ---------------------------------------------------------------
bool mma_forward_ok(const Shape& s, dsa3d_dtype_t dtype) {
  return dtype == DSA3D_BF16 && (s.dh == 64 || s.dh == 128) && s.kw <= 15;
}

SortGeo make_sort_geo(const Shape& s) {
  SortGeo sg;
  sg.Et = s.F + s.kt;
  sg.Ey = s.Hp + s.kh;
  sg.Ex = s.Wp + s.kw;
  sg.E1 = (int64_t)sg.Et * sg.Ey * sg.Ex + 1;
  return sg;
}

// Workspace layout for hg heads: cnt/start [hg*E1] | qkey [hg*N] | qrank [hg*N] |
// sorted_n [hg*N] | sorted_ex [hg*N] | block sums; every part 16-byte aligned.
struct SortWs {
  int *cnt, *qkey, *qrank, *sorted_n, *sorted_ex, *bsum;
  int64_t cnt_elems, nb;
};
size_t align16(size_t b) { return (b + 15) & ~size_t(15); }
size_t sort_ws_bytes(const Shape& s, int hg) {
  const SortGeo sg = make_sort_geo(s);
  const int64_t cnt = (int64_t)hg * sg.E1;
  const int64_t nb = (cnt + kScanTile - 1) / kScanTile;
  return align16(cnt * 4) + 4 * align16((size_t)hg * s.N * 4) + align16(nb * 4);
}
// Forward workspace of a head group: the sort arrays, then the paired value rows
// (F * Hp * ceil(Wp / 2) pairs of keys x hg heads x dh words).
int pair_width(const Shape& s) { return (s.Wp + 1) / 2; }
size_t vpair_bytes(const Shape& s, int hg) {
  return align16((size_t)s.F * s.Hp * pair_width(s) * hg * s.dh * 4);
}
size_t fwd_ws_bytes(const Shape& s, int hg) { return sort_ws_bytes(s, hg) + vpair_bytes(s, hg); }
SortWs carve_sort_ws(const Shape& s, int hg, void* base) {
  const SortGeo sg = make_sort_geo(s);
  SortWs w;
  w.cnt_elems = (int64_t)hg * sg.E1;
  w.nb = (w.cnt_elems + kScanTile - 1) / kScanTile;
  char* p = static_cast<char*>(base);
  w.cnt = reinterpret_cast<int*>(p);
  p += align16(w.cnt_elems * 4);
  const size_t qb = align16((size_t)hg * s.N * 4);
  w.qkey = reinterpret_cast<int*>(p);
  p += qb;
  w.qrank = reinterpret_cast<int*>(p);
  p += qb;
  w.sorted_n = reinterpret_cast<int*>(p);
  p += qb;
  w.sorted_ex = reinterpret_cast<int*>(p);
  p += qb;
  w.bsum = reinterpret_cast<int*>(p);
  return w;
}

int grid_for(int64_t work, int threads, int per_sm_cap) {
  const DeviceInfo d = device_info();
  int64_t grid = (work + threads - 1) / threads;
  const int64_t cap = (int64_t)d.sms * per_sm_cap;
  if (grid > cap) grid = cap;
  if (grid < 1) grid = 1;
  return (int)grid;
}

// Argument checks of the forward entry points (after check_shape): pointers present and aligned,
// outputs disjoint from the inputs and from each other.  off_bytes: size of the offsets.
dsa3d_status_t check_forward_args(const Shape& s, dsa3d_dtype_t dtype, const void* q, const void* k,
                                  const void* v, const float* offsets, size_t off_bytes,
                                  const void* out, const float* lse) {
  if (!q || !k || !v || !offsets || !out) return DSA3D_ERR_INVALID_ARGUMENT;
  const void* al[] = {q, k, v, offsets, out};
  for (const void* p : al)
    if (!aligned16(p)) return DSA3D_ERR_INVALID_ARGUMENT;
  if (lse && (reinterpret_cast<uintptr_t>(lse) & 3u)) return DSA3D_ERR_INVALID_ARGUMENT;
  const size_t tb = (size_t)s.N * s.heads * s.dh * elem_size(dtype);
  const Range in[] = {range_of(q, tb), range_of(k, tb), range_of(v, tb), range_of(offsets, off_bytes)};
  const Range ro = range_of(out, tb);
  const Range rl = range_of(lse, lse ? (size_t)s.heads * s.N * 4 : 0);
  for (const Range& r : in)
    if (overlap(r, ro) || (lse && overlap(r, rl))) return DSA3D_ERR_INVALID_ARGUMENT;
  if (lse && overlap(ro, rl)) return DSA3D_ERR_INVALID_ARGUMENT;
  return DSA3D_OK;
}

// The same for the backward entry points; fills the input and output ranges for the workspace
// checks.  off_bytes: size of the offsets (and of their gradient).
dsa3d_status_t check_backward_args(const Shape& s, dsa3d_dtype_t dtype, const void* q, const void* k,
                                   const void* v, const float* offsets, const float* lse,
                                   const void* dout, const void* dq, const void* dk, const void* dv,
                                   const float* doffsets, size_t off_bytes, Range ins[6],
                                   Range outs[4]) {
  if (!q || !k || !v || !offsets || !lse || !dout || !dq || !dk || !dv || !doffsets)
    return DSA3D_ERR_INVALID_ARGUMENT;
  const void* al[] = {q, k, v, offsets, dout, dq, dk, dv, doffsets};
  for (const void* p : al)
    if (!aligned16(p)) return DSA3D_ERR_INVALID_ARGUMENT;
  if (reinterpret_cast<uintptr_t>(lse) & 3u) return DSA3D_ERR_INVALID_ARGUMENT;
  const size_t tb = (size_t)s.N * s.heads * s.dh * elem_size(dtype);
  ins[0] = range_of(q, tb);
  ins[1] = range_of(k, tb);
  ins[2] = range_of(v, tb);
  ins[3] = range_of(offsets, off_bytes);
  ins[4] = range_of(lse, (size_t)s.heads * s.N * 4);
  ins[5] = range_of(dout, tb);
  outs[0] = range_of(dq, tb);
  outs[1] = range_of(dk, tb);
  outs[2] = range_of(dv, tb);
  outs[3] = range_of(doffsets, off_bytes);
  for (int i = 0; i < 4; i++) {
    for (int j = 0; j < 6; j++)
      if (overlap(ins[j], outs[i])) return DSA3D_ERR_INVALID_ARGUMENT;
    for (int j = i + 1; j < 4; j++)
      if (overlap(outs[i], outs[j])) return DSA3D_ERR_INVALID_ARGUMENT;
  }
  return DSA3D_OK;
}

// A caller workspace must be aligned and disjoint from every tensor argument.
dsa3d_status_t check_workspace(const void* ws, size_t bytes, const Range* ins, int n_in,
                               const Range* outs, int n_out) {
  if (!aligned16(ws)) return DSA3D_ERR_INVALID_ARGUMENT;
  const Range rw = range_of(ws, bytes);
  for (int i = 0; i < n_in; i++)
    if (overlap(ins[i], rw)) return DSA3D_ERR_INVALID_ARGUMENT;
  for (int i = 0; i < n_out; i++)
    if (overlap(outs[i], rw)) return DSA3D_ERR_INVALID_ARGUMENT;
  return DSA3D_OK;
}

dsa3d_status_t zero16(void* p, size_t n16, cudaStream_t st);

// Sort the queries of heads [h0, h0 + hg) by window origin into w (dsa3d_sort.cuh): zero the
// bucket counts, count, scan, fill, then order each bucket by token index so that the sorted
// arrays are the same in every run.  Queries without a valid tap get zero rows of zrow (the
// forward's out or the backward's dq), lse = -inf (when lse is given) and zero doff (when given).
template <int DH>
dsa3d_status_t sort_queries(const Shape& s, const float* off, const SortWs& w, int h0, int hg,
                            __nv_bfloat16* zrow, float* lse, float* doff, cudaStream_t st) {
  const Geo g = make_geo(s);
  const SortGeo sg = make_sort_geo(s);
  dsa3d_status_t rc = zero16(w.cnt, align16(w.cnt_elems * 4) / 16, st);
  if (rc != DSA3D_OK) return rc;
  const int64_t items = (int64_t)hg * s.N;
  {
    TimedLaunch tl(kKernSortCount, st);
    dsa3d_sort_count_kernel<__nv_bfloat16, DH><<<grid_for(items, 256, 16), 256, 0, st>>>(
        off, g, sg, h0, hg, w.cnt, w.qkey, w.qrank, zrow, lse, doff);
    if (cudaGetLastError() != cudaSuccess || !tl.finish()) return DSA3D_ERR_CUDA;
  }
  {
    TimedLaunch tl(kKernScan, st);
    dsa3d_scan_blocks_kernel<<<(unsigned)w.nb, kScanThreads, 0, st>>>(w.cnt, w.cnt_elems, w.bsum);
    dsa3d_scan_sums_kernel<<<1, kScanThreads, 0, st>>>(w.bsum, (int)w.nb);
    dsa3d_scan_apply_kernel<<<(unsigned)w.nb, kScanThreads, 0, st>>>(w.cnt, w.cnt_elems, w.bsum);
    if (cudaGetLastError() != cudaSuccess || !tl.finish()) return DSA3D_ERR_CUDA;
  }
  {
    TimedLaunch tl(kKernSortFill, st);
    dsa3d_sort_fill_kernel<<<grid_for(items, 256, 16), 256, 0, st>>>(w.cnt, w.qkey, w.qrank, g, sg, hg,
                                                                     w.sorted_n, w.sorted_ex);
    if (cudaGetLastError() != cudaSuccess || !tl.finish()) return DSA3D_ERR_CUDA;
  }
  // order: the scan's block sums are spent, so bsum[0] counts the large buckets (listed in qkey,
  // whose keys are spent too) and qrank is the merge scratch of their runs
  if ((rc = zero16(w.bsum, 1, st)) != DSA3D_OK) return rc;
  {
    TimedLaunch tl(kKernSortOrder, st);
    dsa3d_sort_order_kernel<<<grid_for(w.cnt_elems - 1, 256, 16), 256, 0, st>>>(
        w.cnt, w.cnt_elems - 1, w.sorted_n, w.qkey, w.bsum);
    dsa3d_sort_order_big_kernel<<<device_info().sms, kBigThreads, 0, st>>>(w.cnt, w.qkey, w.bsum,
                                                                           w.sorted_n, w.qrank);
    if (cudaGetLastError() != cudaSuccess || !tl.finish()) return DSA3D_ERR_CUDA;
  }
  return DSA3D_OK;
}

template <int DH>
dsa3d_status_t fwd_mma_group(const Shape& s, const void* q, const void* k, const void* v,
                             const float* off, void* out, float* lse, const SortWs& w,
                             unsigned* vp, int h0, int hg, cudaStream_t st) {
  const Geo g = make_geo(s);
  const SortGeo sg = make_sort_geo(s);
  const int Wp2 = pair_width(s);
  {
    TimedLaunch tl(kKernPairV, st);
    const int64_t pitems = (int64_t)s.F * s.Hp * Wp2 * hg * (DH / 8);
    dsa3d_pair_v_kernel<DH><<<grid_for(pitems, 256, 16), 256, 0, st>>>(
        static_cast<const __nv_bfloat16*>(v), vp, g, Wp2, h0, hg);
    if (cudaGetLastError() != cudaSuccess || !tl.finish()) return DSA3D_ERR_CUDA;
  }
  dsa3d_status_t rc = sort_queries<DH>(s, off, w, h0, hg, static_cast<__nv_bfloat16*>(out), lse, nullptr, st);
  if (rc != DSA3D_OK) return rc;
  {
    // the scores warp's tap loops sized for the window: two lanes per query, ceil(kw / 2) taps each
    auto kern = (s.kw <= 9) ? dsa3d_fwd_mma_kernel<DH, 5> : dsa3d_fwd_mma_kernel<DH, 8>;
    const int smem = 2 * fwd_pair_bytes();  // two warp pairs per CTA
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
      return DSA3D_ERR_CUDA;
    const int64_t rows = (int64_t)hg * sg.Et * sg.Ey;
    const int grid = grid_for(rows, 2, 1 << 20);  // one row per warp pair; the scheduler balances rows
    TimedLaunch tl(kKernFwdMma, st);
    kern<<<grid, 128, smem, st>>>(static_cast<const __nv_bfloat16*>(q), static_cast<const __nv_bfloat16*>(k),
                               static_cast<const __nv_bfloat16*>(v), off,
                               static_cast<__nv_bfloat16*>(out), lse, w.cnt, w.sorted_n, w.sorted_ex, vp,
                               Wp2, g, sg, h0, hg);
    if (cudaGetLastError() != cudaSuccess || !tl.finish()) return DSA3D_ERR_CUDA;
  }
  return DSA3D_OK;
}

// --- tcgen05 forward ---------------------------------------------------------------------------
// cuTensorMapEncodeTiled through the runtime's driver entry point (no link to the driver library).
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// Tensor map over a [T][H'][W'][heads][dh] bf16 tensor (k or v) viewed as the 5-D
// (64 dims, heads * dh / 64 head halves, x, y, t), box (64, 1, 32 keys, 1 row, 2 planes) with the
// 128-byte swizzle: one TMA copy per 64 dims brings half of a K or V "pair" (one row, two planes,
// 32 keys) into the layout the tcgen05 forward's UMMAs read (dsa3d_fwd_tc.cuh).
bool make_pair_map(CUtensorMap* m, const void* base, const Shape& s) {
  PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
  if (!enc) return false;
  const cuuint64_t row = (cuuint64_t)s.heads * s.dh * 2;  // bytes per token
  const cuuint64_t dims[5] = {64, (cuuint64_t)s.heads * s.dh / 64, (cuuint64_t)s.Wp, (cuuint64_t)s.Hp,
                              (cuuint64_t)s.F};
  const cuuint64_t strides[4] = {128, row, row * s.Wp, row * s.Wp * s.Hp};
  const cuuint32_t box[5] = {64, 1, (cuuint32_t)kTcSeg, 1, 2};
  const cuuint32_t es[5] = {1, 1, 1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, const_cast<void*>(base), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Bucket rows per tile: about 225 queries per tile at the volume's average density (one query
// per bucket, spread over (F+kt)(H'+kh)(W'+kw) buckets), 1..kTcRyMax; DSA3D_TC_RY overrides it.
// A tile of more than 128 queries takes a second pass, but each pass walks only its own union
// rows and each epilogue warp skips the rows none of its queries touch, so tall tiles still win
// (1080p: 309, 293, 286, 277 ms at 6, 8, 10, 12 rows; 720p: 9.5, 8.8, 8.1, 8.3 ms).
TcTileGeo make_tile_geo(const Shape& s, int hg) {
  const SortGeo sg = make_sort_geo(s);
  TcTileGeo tg;
  tg.Wx = kTcSeg - s.kw;
  const double dens = (double)s.N / ((double)sg.Et * sg.Ey * sg.Ex);
  int ry = (int)std::lround(225.0 / (dens * tg.Wx));
  if (const char* e = std::getenv("DSA3D_TC_RY")) ry = std::atoi(e);
  tg.Ry = ry < 1 ? 1 : (ry > kTcRyMax ? kTcRyMax : ry);
  tg.nYb = (sg.Ey + tg.Ry - 1) / tg.Ry;
  tg.nXb = (sg.Ex + tg.Wx - 1) / tg.Wx;
  tg.tiles = (int64_t)hg * sg.Et * tg.nYb * tg.nXb;
  return tg;
}

// The tcgen05 forward runs unless DSA3D_FWD_KERNEL=mma selects the mma.sync forward.
bool use_tc_forward() {
  const char* e = std::getenv("DSA3D_FWD_KERNEL");
  return !(e && std::strcmp(e, "mma") == 0);
}

template <int DH>
dsa3d_status_t fwd_tc_group(const Shape& s, const void* q, const void* k, const void* v,
                            const float* off, void* out, float* lse, const SortWs& w, int h0, int hg,
                            cudaStream_t st) {
  using C = FwdTcCfg<DH>;
  const Geo g = make_geo(s);
  const SortGeo sg = make_sort_geo(s);
  CUtensorMap tmk, tmv;
  if (!make_pair_map(&tmk, k, s) || !make_pair_map(&tmv, v, s)) return DSA3D_ERR_CUDA;
  dsa3d_status_t rc = sort_queries<DH>(s, off, w, h0, hg, static_cast<__nv_bfloat16*>(out), lse, nullptr, st);
  if (rc != DSA3D_OK) return rc;
  const TcTileGeo tg = make_tile_geo(s, hg);
  auto kern = dsa3d_fwd_tc_kernel<DH>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES) != cudaSuccess)
    return DSA3D_ERR_CUDA;
  const DeviceInfo d = device_info();
  int64_t grid = d.sms;
  if (grid > tg.tiles) grid = tg.tiles;
  if (grid < 1) grid = 1;
  // the tile counter: the scan's block sums, dead once the sort is done (at least 16 bytes)
  if (cudaMemsetAsync(w.bsum, 0, sizeof(int), st) != cudaSuccess) return DSA3D_ERR_CUDA;
  TimedLaunch tl(kKernFwdTc, st);
  kern<<<(int)grid, kTcThreads, C::SMEM_BYTES, st>>>(tmk, tmv, static_cast<const __nv_bfloat16*>(q), off,
                                                     static_cast<__nv_bfloat16*>(out), lse, w.cnt, w.sorted_n,
                                                     w.sorted_ex, w.bsum, g, sg, tg, h0);
  if (cudaGetLastError() != cudaSuccess || !tl.finish()) return DSA3D_ERR_CUDA;
  return DSA3D_OK;
}

// The tcgen05 dq pass runs unless DSA3D_DQ_KERNEL=mma selects the mma.sync one.
bool use_tc_dq() {
  const char* e = std::getenv("DSA3D_DQ_KERNEL");
  return !(e && std::strcmp(e, "mma") == 0);
}

// The tcgen05 key side runs unless DSA3D_KV_KERNEL=mma selects the mma.sync one, or a tile's
// covering queries span more bucket-row ranges than it takes ((kt + 1)(4 + kh) > 128).
bool use_tc_key_side(const Shape& s) {
  const char* e = std::getenv("DSA3D_KV_KERNEL");
  if (e && std::strcmp(e, "mma") == 0) return false;
  return (s.kt + 1) * (kKvtRows + s.kh) <= kKvtRanges;
}

struct BwdArgs {
  const void *q, *k, *v, *dout;
  const float *off, *lse;
  void *dq, *dk, *dv;
  float* doff;
  float *acc_k, *acc_v;
  int acc_heads, h0, hc;
};

// --- sorted tensor-core backward -------------------------------------------------------------
BoxGeo make_box_geo(const Shape& s) {
  BoxGeo bg;
  bg.rows = s.kt * (s.kh + 1);
  bg.width = s.kw + 1;
  bg.per_q = bg.rows * bg.width;
  return bg;
}
// Workspace for hg heads: the sort's | gamma' boxes | beta boxes | (D, f_t) per sorted query.
size_t mma_bwd_ws_bytes(const Shape& s, int hg) {
  const BoxGeo bg = make_box_geo(s);
  const size_t boxes = align16((size_t)hg * s.N * bg.per_q * 2);
  return sort_ws_bytes(s, hg) + 2 * boxes + align16((size_t)hg * s.N * 8);
}

template <int DH>
dsa3d_status_t bwd_mma_group(const Shape& s, const void* q, const void* k, const void* v,
                             const float* off, const float* lse, const void* dout, void* dq, void* dk,
                             void* dv, float* doff, void* ws, int h0, int hg, cudaStream_t st) {
  const Geo g = make_geo(s);
  const SortGeo sg = make_sort_geo(s);
  const BoxGeo bg = make_box_geo(s);
  const SortWs w = carve_sort_ws(s, hg, ws);
  char* p = static_cast<char*>(ws) + sort_ws_bytes(s, hg);
  const size_t boxes = align16((size_t)hg * s.N * bg.per_q * 2);
  unsigned short* gbox = reinterpret_cast<unsigned short*>(p);
  unsigned short* bbox = reinterpret_cast<unsigned short*>(p + boxes);
  float2* dft = reinterpret_cast<float2*>(p + 2 * boxes);
  using bf = __nv_bfloat16;
  const bf* qb = static_cast<const bf*>(q);
  const bf* kb = static_cast<const bf*>(k);
  const bf* vb = static_cast<const bf*>(v);
  const bf* ob = static_cast<const bf*>(dout);

  dsa3d_status_t rc = sort_queries<DH>(s, off, w, h0, hg, static_cast<bf*>(dq), nullptr, doff, st);
  if (rc != DSA3D_OK) return rc;
  const int64_t rows = (int64_t)hg * sg.Et * sg.Ey;
  {
    const int smem = bwdq_pair_floats() * (int)sizeof(float);  // one warp pair per CTA
    if (cudaFuncSetAttribute(dsa3d_bwd_q_kernel<DH>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) !=
        cudaSuccess)
      return DSA3D_ERR_CUDA;
    TimedLaunch tl(kKernBwdQ, st);
    dsa3d_bwd_q_kernel<DH><<<grid_for(rows, 1, 1 << 20), 64, smem, st>>>(
        qb, kb, vb, ob, off, lse, doff, w.cnt, w.sorted_n, w.sorted_ex, gbox, bbox, dft, g, sg, bg,
        h0, hg);
    if (cudaGetLastError() != cudaSuccess || !tl.finish()) return DSA3D_ERR_CUDA;
  }
  if (use_tc_dq()) {
    using C = DqtCfg<DH>;
    CUtensorMap tmk;
    if (!make_pair_map(&tmk, k, s)) return DSA3D_ERR_CUDA;
    const TcTileGeo tg = make_tile_geo(s, hg);
    auto kern = dsa3d_bwd_dq_tc_kernel<DH>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES) != cudaSuccess)
      return DSA3D_ERR_CUDA;
    const DeviceInfo d = device_info();
    int64_t grid = 2 * (int64_t)d.sms;
    if (grid > tg.tiles) grid = tg.tiles;
    if (grid < 1) grid = 1;
    // the tile counter: the scan's block sums, dead once the sort is done
    if (cudaMemsetAsync(w.bsum, 0, sizeof(int), st) != cudaSuccess) return DSA3D_ERR_CUDA;
    TimedLaunch tl(kKernBwdDqTc, st);
    kern<<<(int)grid, kDqtThreads, C::SMEM_BYTES, st>>>(tmk, static_cast<bf*>(dq), w.cnt, w.sorted_n, w.sorted_ex,
                                                        gbox, bbox, dft, w.bsum, g, sg, bg, tg, h0);
    if (cudaGetLastError() != cudaSuccess || !tl.finish()) return DSA3D_ERR_CUDA;
  } else {
    const int smem = 4 * dq_warp_bytes<DH>();
    if (cudaFuncSetAttribute(dsa3d_bwd_dq_kernel<DH>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) !=
        cudaSuccess)
      return DSA3D_ERR_CUDA;
    TimedLaunch tl(kKernBwdDq, st);
    dsa3d_bwd_dq_kernel<DH><<<grid_for(rows, 4, 1 << 20), 128, smem, st>>>(
        kb, static_cast<bf*>(dq), w.cnt, w.sorted_n, w.sorted_ex, gbox, bbox, dft, g, sg, bg, h0, hg);
    if (cudaGetLastError() != cudaSuccess || !tl.finish()) return DSA3D_ERR_CUDA;
  }
  if (use_tc_key_side(s)) {
    using C = KvtCfg<DH>;
    const int64_t tiles = (int64_t)hg * s.F * ((s.Hp + kKvtRows - 1) / kKvtRows) * ((s.Wp + kKvtKeys - 1) / kKvtKeys);
    auto kern = dsa3d_bwd_kv_tc_kernel<DH>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES) != cudaSuccess)
      return DSA3D_ERR_CUDA;
    const DeviceInfo d = device_info();
    int64_t grid = d.sms;
    if (grid > tiles) grid = tiles;
    if (grid < 1) grid = 1;
    // the tile counter: the scan's block sums, dead once the sort is done (at least 16 bytes)
    if (cudaMemsetAsync(w.bsum, 0, sizeof(int), st) != cudaSuccess) return DSA3D_ERR_CUDA;
    TimedLaunch tl(kKernBwdKvTc, st);
    kern<<<(int)grid, kKvtThreads, C::SMEM_BYTES, st>>>(qb, ob, static_cast<bf*>(dk), static_cast<bf*>(dv), w.cnt,
                                                       w.sorted_n, w.sorted_ex, gbox, bbox, dft, w.bsum, g, sg,
                                                       bg, h0, hg);
    if (cudaGetLastError() != cudaSuccess || !tl.finish()) return DSA3D_ERR_CUDA;
  } else {
    const int64_t tiles = (int64_t)hg * s.F * ((s.Hp + kKvRows - 1) / kKvRows) * ((s.Wp + 15) / 16);
    const int smem = kv_dyn_bytes<DH>();
    if (cudaFuncSetAttribute(dsa3d_bwd_kv_kernel<DH>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) !=
        cudaSuccess)
      return DSA3D_ERR_CUDA;
    TimedLaunch tl(kKernBwdKv, st);
    dsa3d_bwd_kv_kernel<DH><<<grid_for(tiles, 1, 1 << 20), kKvThreads, smem, st>>>(
        qb, ob, static_cast<bf*>(dk), static_cast<bf*>(dv), w.cnt, w.sorted_n, w.sorted_ex, gbox,
        bbox, dft, g, sg, bg, h0, hg);
    if (cudaGetLastError() != cudaSuccess || !tl.finish()) return DSA3D_ERR_CUDA;
  }
  return DSA3D_OK;
}

template <typename T, int DH, int W>
dsa3d_status_t bwd_launch(const Shape& s, const BwdArgs& a, cudaStream_t st) {
  const Geo g = make_geo(s);
  const int smem = smem_bytes(g, W, true);
  auto kern = dsa3d_bwd_kernel<T, DH, W>;
  int grid = 0;
  const int64_t items = (int64_t)a.hc * s.N;
  dsa3d_status_t rc = launch_persistent(kern, W, smem, items, st, grid);
  if (rc != DSA3D_OK) return rc;
  TimedLaunch tl(kKernBwd, st);
  kern<<<grid, W * 32, smem, st>>>(
      static_cast<const T*>(a.q), static_cast<const T*>(a.k), static_cast<const T*>(a.v), a.off,
      a.lse, static_cast<const T*>(a.dout), static_cast<T*>(a.dq),
      a.doff, a.acc_k, a.acc_v, a.acc_heads, a.h0, g, items);
  const bool launched = cudaGetLastError() == cudaSuccess;
  return (tl.finish() && launched) ? DSA3D_OK : DSA3D_ERR_CUDA;
}

template <typename T, int DH>
dsa3d_status_t bwd_finalize(const Shape& s, const BwdArgs& a, cudaStream_t st) {
  const DeviceInfo d = device_info();
  const int64_t chunks = s.N * a.hc * (DH / Elems<T>::kPerLoad);
  int64_t grid = (chunks + 255) / 256;
  if (grid > (int64_t)d.sms * 16) grid = (int64_t)d.sms * 16;
  if (grid < 1) grid = 1;
  TimedLaunch tl(kKernBwdFinalize, st);
  dsa3d_bwd_finalize_kernel<T, DH><<<(int)grid, 256, 0, st>>>(
      a.acc_k, a.acc_v, static_cast<T*>(a.dk), static_cast<T*>(a.dv), s.heads, a.h0, a.hc, s.N);
  const bool launched = cudaGetLastError() == cudaSuccess;
  return (tl.finish() && launched) ? DSA3D_OK : DSA3D_ERR_CUDA;
}

template <typename T, int DH>
dsa3d_status_t bwd_dispatch_w(const Shape& s, int warps, const BwdArgs& a, cudaStream_t st) {
  switch (warps) {
    case 4: return bwd_launch<T, DH, 4>(s, a, st);
    case 2: return bwd_launch<T, DH, 2>(s, a, st);
    case 1: return bwd_launch<T, DH, 1>(s, a, st);
    default: return DSA3D_ERR_UNSUPPORTED;
  }
}

template <typename T>
dsa3d_status_t bwd_dispatch(const Shape& s, int warps, const BwdArgs& a, cudaStream_t st,
                            bool finalize) {
  dsa3d_status_t rc;
  switch (s.dh) {
    case 32: rc = bwd_dispatch_w<T, 32>(s, warps, a, st); break;
    case 64: rc = bwd_dispatch_w<T, 64>(s, warps, a, st); break;
    case 128: rc = bwd_dispatch_w<T, 128>(s, warps, a, st); break;
    default: return DSA3D_ERR_UNSUPPORTED;
  }
  if (rc != DSA3D_OK || !finalize) return rc;
  switch (s.dh) {
    case 32: return bwd_finalize<T, 32>(s, a, st);
    case 64: return bwd_finalize<T, 64>(s, a, st);
    case 128: return bwd_finalize<T, 128>(s, a, st);
    default: return DSA3D_ERR_UNSUPPORTED;
  }
}

// --- per-tap offsets (CUDA cores) -----------------------------------------------------------------
template <typename T, int DH>
dsa3d_status_t fwd_taps_launch(const Shape& s, const void* q, const void* k, const void* v,
                               const float* off, void* out, float* lse, cudaStream_t st) {
  const Geo g = make_geo(s);
  constexpr int W = kTapsFwdWarps;
  auto kern = dsa3d_fwd_taps_kernel<T, DH, W>;
  int grid = 0;
  const int64_t items = (int64_t)s.heads * s.N;
  dsa3d_status_t rc = launch_persistent(kern, W, 0, items, st, grid);
  if (rc != DSA3D_OK) return rc;
  TimedLaunch tl(kKernFwdTaps, st);
  kern<<<grid, W * 32, 0, st>>>(static_cast<const T*>(q), static_cast<const T*>(k),
                                     static_cast<const T*>(v), off, static_cast<T*>(out), lse, g, items);
  const bool launched = cudaGetLastError() == cudaSuccess;
  return (tl.finish() && launched) ? DSA3D_OK : DSA3D_ERR_CUDA;
}

template <typename T>
dsa3d_status_t fwd_taps_dispatch(const Shape& s, const void* q, const void* k, const void* v,
                                 const float* off, void* out, float* lse, cudaStream_t st) {
  switch (s.dh) {
    case 32: return fwd_taps_launch<T, 32>(s, q, k, v, off, out, lse, st);
    case 64: return fwd_taps_launch<T, 64>(s, q, k, v, off, out, lse, st);
    case 128: return fwd_taps_launch<T, 128>(s, q, k, v, off, out, lse, st);
    default: return DSA3D_ERR_UNSUPPORTED;
  }
}

// Warps per CTA of the per-tap backward: its per-warp shared memory grows with K.
int pick_taps_warps(const Geo& g, int max_smem) {
  for (int w = kWarps; w >= 1; w >>= 1)
    if ((int64_t)w * bwd_taps_warp_bytes(g.K) + w * 32 * 20 <= max_smem) return w;
  return 0;
}

template <typename T, int DH, int W>
dsa3d_status_t bwd_taps_launch(const Shape& s, const BwdArgs& a, cudaStream_t st) {
  const Geo g = make_geo(s);
  const int smem = W * bwd_taps_warp_bytes(g.K);
  auto kern = dsa3d_bwd_taps_kernel<T, DH, W>;
  int grid = 0;
  const int64_t items = (int64_t)a.hc * s.N;
  dsa3d_status_t rc = launch_persistent(kern, W, smem, items, st, grid);
  if (rc != DSA3D_OK) return rc;
  TimedLaunch tl(kKernBwdTaps, st);
  kern<<<grid, W * 32, smem, st>>>(
      static_cast<const T*>(a.q), static_cast<const T*>(a.k), static_cast<const T*>(a.v), a.off,
      a.lse, static_cast<const T*>(a.dout), static_cast<T*>(a.dq), a.doff, a.acc_k, a.acc_v,
      a.acc_heads, a.h0, g, items);
  const bool launched = cudaGetLastError() == cudaSuccess;
  return (tl.finish() && launched) ? DSA3D_OK : DSA3D_ERR_CUDA;
}

template <typename T, int DH>
dsa3d_status_t bwd_taps_dispatch_w(const Shape& s, int warps, const BwdArgs& a, cudaStream_t st) {
  switch (warps) {
    case 4: return bwd_taps_launch<T, DH, 4>(s, a, st);
    case 2: return bwd_taps_launch<T, DH, 2>(s, a, st);
    case 1: return bwd_taps_launch<T, DH, 1>(s, a, st);
    default: return DSA3D_ERR_UNSUPPORTED;
  }
}

template <typename T>
dsa3d_status_t bwd_taps_dispatch(const Shape& s, int warps, const BwdArgs& a, cudaStream_t st,
                                 bool finalize) {
  dsa3d_status_t rc;
  switch (s.dh) {
    case 32: rc = bwd_taps_dispatch_w<T, 32>(s, warps, a, st); break;
    case 64: rc = bwd_taps_dispatch_w<T, 64>(s, warps, a, st); break;
    case 128: rc = bwd_taps_dispatch_w<T, 128>(s, warps, a, st); break;
    default: return DSA3D_ERR_UNSUPPORTED;
  }
  if (rc != DSA3D_OK || !finalize) return rc;
  switch (s.dh) {
    case 32: return bwd_finalize<T, 32>(s, a, st);
    case 64: return bwd_finalize<T, 64>(s, a, st);
    case 128: return bwd_finalize<T, 128>(s, a, st);
    default: return DSA3D_ERR_UNSUPPORTED;
  }
}

// Zero n16 16-byte words at p (the backward's fp32 accumulators).
dsa3d_status_t zero16(void* p, size_t n16, cudaStream_t st) {
  const DeviceInfo d = device_info();
  int64_t grid = ((int64_t)n16 + 255) / 256;
  if (grid > (int64_t)d.sms * 8) grid = (int64_t)d.sms * 8;
  if (grid < 1) grid = 1;
  TimedLaunch tl(kKernZero, st);
  dsa3d_zero_kernel<<<(int)grid, 256, 0, st>>>(static_cast<uint4*>(p), (int64_t)n16);
  const bool launched = cudaGetLastError() == cudaSuccess;
  return (tl.finish() && launched) ? DSA3D_OK : DSA3D_ERR_CUDA;
}

size_t acc_bytes_per_head(const Shape& s) { return (size_t)2 * s.N * s.dh * sizeof(float); }

// Scratch of dsa3d_backward_noalloc: a file-scope device array, so that entry point never
// allocates.  Host code must not use the symbol as an address; noalloc_scratch() looks up the
// device address once per device (with that device current) and caches it.
static __device__ __align__(256) unsigned char g_noalloc_scratch[DSA3D_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mu;
void* g_noalloc_ptr[kMaxDevices] = {};

dsa3d_status_t noalloc_scratch(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return DSA3D_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return DSA3D_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (!g_noalloc_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return DSA3D_ERR_CUDA;
    g_noalloc_ptr[dev] = p;
  }
  *out = g_noalloc_ptr[dev];
  return DSA3D_OK;
}

}  // namespace
}  // namespace dsa3d

using namespace dsa3d;

extern "C" {

int dsa3d_abi_version(void) { return DSA3D_ABI_VERSION; }

const char* dsa3d_status_string(dsa3d_status_t status) {
  switch (status) {
    case DSA3D_OK: return "ok";
    case DSA3D_ERR_INVALID_ARGUMENT: return "invalid argument";
    case DSA3D_ERR_UNSUPPORTED: return "unsupported shape or window";
    case DSA3D_ERR_WORKSPACE_TOO_SMALL: return "workspace too small";
    case DSA3D_ERR_CUDA: return "CUDA error";
    case DSA3D_ERR_DEVICE_CHECK: return "device-side check failed";
    default: return "unknown status";
  }
}

dsa3d_status_t dsa3d_forward(const void* q, const void* k, const void* v, const float* offsets,
                             void* out, float* lse, void* workspace, size_t workspace_bytes,
                             int F, int Hp, int Wp, int heads, int dh, int kt, int kh, int kw,
                             dsa3d_dtype_t dtype, cudaStream_t stream) {
  const Shape s{F, Hp, Wp, heads, dh, kt, kh, kw, (int64_t)F * Hp * Wp};
  dsa3d_status_t rc = check_shape(s, dtype, 0);
  if (rc != DSA3D_OK) return rc;
  const size_t ob = (size_t)heads * s.N * 12;
  if ((rc = check_forward_args(s, dtype, q, k, v, offsets, ob, out, lse)) != DSA3D_OK) return rc;

  if (workspace && workspace_bytes > 0 && mma_forward_ok(s, dtype)) {
    const size_t one = fwd_ws_bytes(s, 1);
    if (workspace_bytes < one) return DSA3D_ERR_WORKSPACE_TOO_SMALL;
    const size_t tb = (size_t)s.N * heads * dh * elem_size(dtype);
    const Range ins[] = {range_of(q, tb), range_of(k, tb), range_of(v, tb), range_of(offsets, ob)};
    const Range outs[] = {range_of(out, tb), range_of(lse, lse ? (size_t)heads * s.N * 4 : 0)};
    if ((rc = check_workspace(workspace, workspace_bytes, ins, 4, outs, 2)) != DSA3D_OK) return rc;
    int hg = heads;
    while (hg > 1 && fwd_ws_bytes(s, hg) > workspace_bytes) hg = (hg + 1) / 2;
    for (int h0 = 0; h0 < heads; h0 += hg) {
      const int n = (heads - h0 < hg) ? heads - h0 : hg;
      const SortWs wn = carve_sort_ws(s, n, workspace);
      unsigned* vp = reinterpret_cast<unsigned*>(static_cast<char*>(workspace) + sort_ws_bytes(s, n));
      dsa3d_status_t r;
      if (use_tc_forward())
        r = (dh == 128) ? fwd_tc_group<128>(s, q, k, v, offsets, out, lse, wn, h0, n, stream)
                        : fwd_tc_group<64>(s, q, k, v, offsets, out, lse, wn, h0, n, stream);
      else
        r = (dh == 128) ? fwd_mma_group<128>(s, q, k, v, offsets, out, lse, wn, vp, h0, n, stream)
                        : fwd_mma_group<64>(s, q, k, v, offsets, out, lse, wn, vp, h0, n, stream);
      if (r != DSA3D_OK) return r;
    }
    return DSA3D_OK;
  }

  const Geo g = make_geo(s);
  const DeviceInfo d = device_info();
  if (d.sms == 0) return DSA3D_ERR_CUDA;  // no usable device
  const int warps = pick_warps(g, false, d.max_smem);
  if (warps == 0) return DSA3D_ERR_UNSUPPORTED;
  if (dtype == DSA3D_F32)
    return fwd_dispatch<float>(s, warps, q, k, v, offsets, out, lse, stream);
  return fwd_dispatch<__nv_bfloat16>(s, warps, q, k, v, offsets, out, lse, stream);
}

size_t dsa3d_forward_workspace_bytes(int F, int Hp, int Wp, int heads, int dh, int kt, int kh,
                                     int kw, dsa3d_dtype_t dtype) {
  const Shape s{F, Hp, Wp, heads, dh, kt, kh, kw, (int64_t)F * Hp * Wp};
  if (check_shape(s, dtype, 0) != DSA3D_OK || !mma_forward_ok(s, dtype)) return 0;
  return fwd_ws_bytes(s, heads);
}

size_t dsa3d_backward_workspace_bytes(int F, int Hp, int Wp, int heads, int dh, int kt, int kh,
                                      int kw, dsa3d_dtype_t dtype) {
  const Shape s{F, Hp, Wp, heads, dh, kt, kh, kw, (int64_t)F * Hp * Wp};
  if (check_shape(s, dtype, 0) != DSA3D_OK) return 0;
  if (dtype == DSA3D_F32) return 0;
  if (mma_forward_ok(s, dtype)) return mma_bwd_ws_bytes(s, heads);
  return acc_bytes_per_head(s) * (size_t)heads;
}

dsa3d_status_t dsa3d_backward(const void* q, const void* k, const void* v, const float* offsets,
                              const float* lse, const void* dout, void* dq,
                              void* dk, void* dv, float* doffsets, void* workspace,
                              size_t workspace_bytes, int F, int Hp, int Wp, int heads, int dh,
                              int kt, int kh, int kw, dsa3d_dtype_t dtype, cudaStream_t stream) {
  const Shape s{F, Hp, Wp, heads, dh, kt, kh, kw, (int64_t)F * Hp * Wp};
  dsa3d_status_t rc = check_shape(s, dtype, 0);
  if (rc != DSA3D_OK) return rc;
  Range ins[6], outs[4];
  rc = check_backward_args(s, dtype, q, k, v, offsets, lse, dout, dq, dk, dv, doffsets,
                           (size_t)heads * s.N * 12, ins, outs);
  if (rc != DSA3D_OK) return rc;
  const size_t tb = (size_t)s.N * heads * dh * elem_size(dtype);

  if (mma_forward_ok(s, dtype) && workspace && workspace_bytes >= mma_bwd_ws_bytes(s, 1)) {
    if ((rc = check_workspace(workspace, workspace_bytes, ins, 6, outs, 4)) != DSA3D_OK) return rc;
    int hg = heads;
    while (hg > 1 && mma_bwd_ws_bytes(s, hg) > workspace_bytes) hg = (hg + 1) / 2;
    for (int h0 = 0; h0 < heads; h0 += hg) {
      const int n = (heads - h0 < hg) ? heads - h0 : hg;
      const dsa3d_status_t r =
          (dh == 128) ? bwd_mma_group<128>(s, q, k, v, offsets, lse, dout, dq, dk, dv, doffsets, workspace, h0, n, stream)
                      : bwd_mma_group<64>(s, q, k, v, offsets, lse, dout, dq, dk, dv, doffsets, workspace, h0, n, stream);
      if (r != DSA3D_OK) return r;
    }
    return DSA3D_OK;
  }

  const size_t per_head = acc_bytes_per_head(s);
  if (dtype == DSA3D_BF16) {
    if (!workspace || workspace_bytes < per_head) return DSA3D_ERR_WORKSPACE_TOO_SMALL;
    if ((rc = check_workspace(workspace, workspace_bytes, ins, 6, outs, 4)) != DSA3D_OK) return rc;
  }

  const Geo g = make_geo(s);
  const DeviceInfo d = device_info();
  if (d.sms == 0) return DSA3D_ERR_CUDA;  // no usable device
  const int warps = pick_warps(g, true, d.max_smem);
  if (warps == 0) return DSA3D_ERR_UNSUPPORTED;

  BwdArgs a;
  a.q = q; a.k = k; a.v = v; a.dout = dout; a.off = offsets; a.lse = lse;
  a.dq = dq; a.dk = dk; a.dv = dv; a.doff = doffsets;

  if (dtype == DSA3D_F32) {
    // accumulate straight into the fp32 outputs
    if ((rc = zero16(dk, tb / 16, stream)) != DSA3D_OK) return rc;
    if ((rc = zero16(dv, tb / 16, stream)) != DSA3D_OK) return rc;
    a.acc_k = static_cast<float*>(dk);
    a.acc_v = static_cast<float*>(dv);
    a.acc_heads = heads;
    a.h0 = 0;
    a.hc = heads;
    return bwd_dispatch<float>(s, warps, a, stream, false);
  }

  int hc_max = (int)(workspace_bytes / per_head);
  if (hc_max > heads) hc_max = heads;
  for (int h0 = 0; h0 < heads; h0 += hc_max) {
    const int hc = (heads - h0 < hc_max) ? heads - h0 : hc_max;
    const size_t half = (size_t)s.N * hc * dh;  // floats per accumulator
    a.acc_k = static_cast<float*>(workspace);
    a.acc_v = a.acc_k + half;
    a.acc_heads = hc;
    a.h0 = h0;
    a.hc = hc;
    if ((rc = zero16(workspace, 2 * half * sizeof(float) / 16, stream)) != DSA3D_OK) return rc;
    rc = bwd_dispatch<__nv_bfloat16>(s, warps, a, stream, true);
    if (rc != DSA3D_OK) return rc;
  }
  return DSA3D_OK;
}

dsa3d_status_t dsa3d_backward_noalloc(const void* q, const void* k, const void* v,
                                      const float* offsets, const float* lse,
                                      const void* dout, void* dq, void* dk, void* dv,
                                      float* doffsets, int F, int Hp, int Wp, int heads, int dh,
                                      int kt, int kh, int kw, dsa3d_dtype_t dtype,
                                      cudaStream_t stream) {
  const Shape s{F, Hp, Wp, heads, dh, kt, kh, kw, (int64_t)F * Hp * Wp};
  const dsa3d_status_t rc = check_shape(s, dtype, 0);
  if (rc != DSA3D_OK) return rc;
  // reject, before any device work, a problem whose single head fits neither path in the fixed
  // scratch: the tensor-core path's sort and splats, or the general path's fp32 accumulators
  if (dtype == DSA3D_BF16) {
    const bool mma_fits = mma_forward_ok(s, dtype) && mma_bwd_ws_bytes(s, 1) <= DSA3D_NOALLOC_SCRATCH_BYTES;
    if (!mma_fits && acc_bytes_per_head(s) > DSA3D_NOALLOC_SCRATCH_BYTES) return DSA3D_ERR_WORKSPACE_TOO_SMALL;
  }
  void* scratch = nullptr;
  const dsa3d_status_t sc = noalloc_scratch(&scratch);
  if (sc != DSA3D_OK) return sc;
  return dsa3d_backward(q, k, v, offsets, lse, dout, dq, dk, dv, doffsets, scratch,
                        DSA3D_NOALLOC_SCRATCH_BYTES, F, Hp, Wp, heads, dh, kt, kh, kw, dtype,
                        stream);
}

dsa3d_status_t dsa3d_forward_taps(const void* q, const void* k, const void* v, const float* offsets,
                                  void* out, float* lse, int F, int Hp, int Wp, int heads, int dh,
                                  int kt, int kh, int kw, dsa3d_dtype_t dtype, cudaStream_t stream) {
  const Shape s{F, Hp, Wp, heads, dh, kt, kh, kw, (int64_t)F * Hp * Wp};
  dsa3d_status_t rc = check_shape(s, dtype, 0);
  if (rc != DSA3D_OK) return rc;
  const size_t ob = (size_t)heads * s.N * kt * kh * kw * 12;
  if ((rc = check_forward_args(s, dtype, q, k, v, offsets, ob, out, lse)) != DSA3D_OK) return rc;
  if (dtype == DSA3D_F32) return fwd_taps_dispatch<float>(s, q, k, v, offsets, out, lse, stream);
  return fwd_taps_dispatch<__nv_bfloat16>(s, q, k, v, offsets, out, lse, stream);
}

size_t dsa3d_backward_taps_workspace_bytes(int F, int Hp, int Wp, int heads, int dh, int kt, int kh,
                                           int kw, dsa3d_dtype_t dtype) {
  const Shape s{F, Hp, Wp, heads, dh, kt, kh, kw, (int64_t)F * Hp * Wp};
  if (check_shape(s, dtype, 0) != DSA3D_OK || dtype == DSA3D_F32) return 0;
  return acc_bytes_per_head(s) * (size_t)heads;
}

dsa3d_status_t dsa3d_backward_taps(const void* q, const void* k, const void* v, const float* offsets,
                                   const float* lse, const void* dout, void* dq, void* dk, void* dv,
                                   float* doffsets, void* workspace, size_t workspace_bytes, int F,
                                   int Hp, int Wp, int heads, int dh, int kt, int kh, int kw,
                                   dsa3d_dtype_t dtype, cudaStream_t stream) {
  const Shape s{F, Hp, Wp, heads, dh, kt, kh, kw, (int64_t)F * Hp * Wp};
  dsa3d_status_t rc = check_shape(s, dtype, 0);
  if (rc != DSA3D_OK) return rc;
  Range ins[6], outs[4];
  rc = check_backward_args(s, dtype, q, k, v, offsets, lse, dout, dq, dk, dv, doffsets,
                           (size_t)heads * s.N * kt * kh * kw * 12, ins, outs);
  if (rc != DSA3D_OK) return rc;
  const size_t per_head = acc_bytes_per_head(s);
  if (dtype == DSA3D_BF16) {
    if (!workspace || workspace_bytes < per_head) return DSA3D_ERR_WORKSPACE_TOO_SMALL;
    if ((rc = check_workspace(workspace, workspace_bytes, ins, 6, outs, 4)) != DSA3D_OK) return rc;
  }
  const Geo g = make_geo(s);
  const int warps = pick_taps_warps(g, device_info().max_smem);
  if (warps == 0) return DSA3D_ERR_UNSUPPORTED;

  BwdArgs a;
  a.q = q; a.k = k; a.v = v; a.dout = dout; a.off = offsets; a.lse = lse;
  a.dq = dq; a.dk = dk; a.dv = dv; a.doff = doffsets;
  if (dtype == DSA3D_F32) {
    const size_t tb = (size_t)s.N * heads * dh * 4;
    if ((rc = zero16(dk, tb / 16, stream)) != DSA3D_OK) return rc;
    if ((rc = zero16(dv, tb / 16, stream)) != DSA3D_OK) return rc;
    a.acc_k = static_cast<float*>(dk);
    a.acc_v = static_cast<float*>(dv);
    a.acc_heads = heads;
    a.h0 = 0;
    a.hc = heads;
    return bwd_taps_dispatch<float>(s, warps, a, stream, false);
  }
  int hc_max = (int)(workspace_bytes / per_head);
  if (hc_max > heads) hc_max = heads;
  for (int h0 = 0; h0 < heads; h0 += hc_max) {
    const int hc = (heads - h0 < hc_max) ? heads - h0 : hc_max;
    const size_t half = (size_t)s.N * hc * dh;
    a.acc_k = static_cast<float*>(workspace);
    a.acc_v = a.acc_k + half;
    a.acc_heads = hc;
    a.h0 = h0;
    a.hc = hc;
    if ((rc = zero16(workspace, 2 * half * sizeof(float) / 16, stream)) != DSA3D_OK) return rc;
    if ((rc = bwd_taps_dispatch<__nv_bfloat16>(s, warps, a, stream, true)) != DSA3D_OK) return rc;
  }
  return DSA3D_OK;
}

dsa3d_status_t dsa3d_timing_enable(int enable) {
  Timing::get().enable(enable != 0);
  return DSA3D_OK;
}

int dsa3d_timing_read(dsa3d_kernel_time_t* out, int max_entries) {
  return Timing::get().read(out, max_entries);
}

void dsa3d_timing_reset(void) { Timing::get().reset(); }

#ifdef DSA3D_TC_TRACE
int dsa3d_tc_trace_read(float* host, int n) {
  return cudaMemcpyFromSymbol(host, g_tc_trace, (size_t)n * sizeof(float)) == cudaSuccess ? 0 : 1;
}
int dsa3d_tc_clk_read(unsigned* host, int n) {
  return cudaMemcpyFromSymbol(host, g_tc_clk, (size_t)n * sizeof(unsigned)) == cudaSuccess ? 0 : 1;
}
#endif

dsa3d_status_t dsa3d_check_device(cudaStream_t stream) {
  if (cudaStreamSynchronize(stream) != cudaSuccess) return DSA3D_ERR_CUDA;
  int flag = 0;
  if (cudaMemcpyFromSymbol(&flag, g_dsa3d_check, sizeof(int)) != cudaSuccess) return DSA3D_ERR_CUDA;
  if (flag) {
    const int zero = 0;
    if (cudaMemcpyToSymbol(g_dsa3d_check, &zero, sizeof(int)) != cudaSuccess) return DSA3D_ERR_CUDA;
    return DSA3D_ERR_DEVICE_CHECK;
  }
  return DSA3D_OK;
}

}  // extern "C"
