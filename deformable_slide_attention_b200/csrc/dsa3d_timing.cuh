// dsa3d_timing.cuh -- optional per-kernel timing with CUDA events on the launch stream
// (the dsa3d_timing_* entry points).  Off by default; when off, a launch costs one relaxed
// atomic load.
#pragma once

#include <cuda_runtime.h>

#include <atomic>
#include <mutex>
#include <vector>

namespace dsa3d {

enum KernelId {
  kKernFwd = 0,
  kKernBwd,
  kKernBwdFinalize,
  kKernZero,
  kKernFwdMma,
  kKernSortCount,
  kKernScan,
  kKernSortFill,
  kKernBwdQ,
  kKernBwdDq,
  kKernBwdKv,
  kKernPairV,
  kKernFwdTaps,
  kKernBwdTaps,
  kKernDwconv,
  kKernDwconvDw,
  kKernPointwise,
  kKernPointwiseDz,
  kKernPointwiseDw,
  kKernSortOrder,
  kKernFwdTc,
  kKernBwdKvTc,
  kKernBwdDqTc,
  kKernDwconvSw,
  kKernDwconvSw2,
  kKernCount
};
inline const char* kernel_name(int id) {
  static const char* names[kKernCount] = {
      "dsa3d_fwd_kernel",      "dsa3d_bwd_kernel",        "dsa3d_bwd_finalize_kernel",
      "dsa3d_zero_kernel",     "dsa3d_fwd_mma_kernel",    "dsa3d_sort_count_kernel",
      "dsa3d_scan_kernels",    "dsa3d_sort_fill_kernel",  "dsa3d_bwd_q_kernel",
      "dsa3d_bwd_dq_kernel",   "dsa3d_bwd_kv_kernel",     "dsa3d_pair_v_kernel",
      "dsa3d_fwd_taps_kernel", "dsa3d_bwd_taps_kernel", "dsa3d_dwconv3d_kernel",
      "dsa3d_dwconv3d_dw_kernel", "dsa3d_pointwise_offsets_kernel", "dsa3d_pointwise_dz_kernel",
      "dsa3d_pointwise_dw_kernel", "dsa3d_sort_order_kernels", "dsa3d_fwd_tc_kernel",
      "dsa3d_bwd_kv_tc_kernel", "dsa3d_bwd_dq_tc_kernel", "dsa3d_dwconv3d_sw_kernel",
      "dsa3d_dwconv3d_sw2_kernel"};
  return names[id];
}

class Timing {
 public:
  static Timing& get() {
    static Timing t;
    return t;
  }
  bool on() const { return on_.load(std::memory_order_relaxed); }
  void enable(bool e) { on_.store(e, std::memory_order_relaxed); }

  // Bracket a launch: begin() before, end() after.  Returns false on a CUDA error.
  bool begin(int kid, cudaStream_t st, int& slot) {
    slot = -1;
    if (!on()) return true;
    std::lock_guard<std::mutex> g(mu_);
    Pending p;
    p.kid = kid;
    if (!take(p.a) || !take(p.b)) return false;
    if (cudaEventRecord(p.a, st) != cudaSuccess) return false;
    pending_.push_back(p);
    slot = (int)pending_.size() - 1;
    return true;
  }
  bool end(int slot, cudaStream_t st) {
    if (slot < 0) return true;
    std::lock_guard<std::mutex> g(mu_);
    return cudaEventRecord(pending_[slot].b, st) == cudaSuccess;
  }
  int read(dsa3d_kernel_time_t* out, int max_entries) {
    std::lock_guard<std::mutex> g(mu_);
    for (Pending& p : pending_) {
      float ms = 0.f;
      if (cudaEventSynchronize(p.b) == cudaSuccess && cudaEventElapsedTime(&ms, p.a, p.b) == cudaSuccess) {
        total_ms_[p.kid] += ms;
        launches_[p.kid] += 1;
      }
      free_.push_back(p.a);
      free_.push_back(p.b);
    }
    pending_.clear();
    int n = 0;
    for (int k = 0; k < kKernCount; k++) {
      if (launches_[k] == 0) continue;
      if (out && n < max_entries) {
        out[n].kernel = kernel_name(k);
        out[n].launches = launches_[k];
        out[n].total_ms = total_ms_[k];
      }
      n++;
    }
    return n;
  }
  void reset() {
    std::lock_guard<std::mutex> g(mu_);
    for (int k = 0; k < kKernCount; k++) {
      launches_[k] = 0;
      total_ms_[k] = 0.0;
    }
  }

 private:
  struct Pending {
    int kid;
    cudaEvent_t a, b;
  };
  bool take(cudaEvent_t& e) {
    if (!free_.empty()) {
      e = free_.back();
      free_.pop_back();
      return true;
    }
    return cudaEventCreate(&e) == cudaSuccess;
  }
  std::atomic<bool> on_{false};
  std::mutex mu_;
  std::vector<Pending> pending_;
  std::vector<cudaEvent_t> free_;
  long long launches_[kKernCount] = {};
  double total_ms_[kKernCount] = {};
};

// RAII bracket around one launch.
struct TimedLaunch {
  int slot = -1;
  cudaStream_t st;
  bool ok = true;
  TimedLaunch(int kid, cudaStream_t s) : st(s) { ok = Timing::get().begin(kid, s, slot); }
  bool finish() { return Timing::get().end(slot, st) && ok; }
};

}  // namespace dsa3d
