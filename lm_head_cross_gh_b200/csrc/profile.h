// Kernel timing and launch counting for libgh (host side).
//
// While timing is enabled (gh_profile_enable), each ProfileScope records a
// pair of CUDA events on the launching stream around one kernel; the pairs
// are kept per kernel kind and summed by gh_profile_read.  note_launch counts
// every kernel the library launches (gh_launch_count).
#pragma once

#include <atomic>
#include <mutex>
#include <vector>

#include <cuda_runtime.h>

#include "../../include/gh.h"

namespace gh {

struct ProfileState {
  std::mutex mu;
  bool enabled = false;
  struct Rec {
    int kind;
    cudaEvent_t start, stop;
  };
  std::vector<Rec> recs;
  std::vector<cudaEvent_t> pool;

  cudaEvent_t take() {
    if (!pool.empty()) {
      cudaEvent_t e = pool.back();
      pool.pop_back();
      return e;
    }
    cudaEvent_t e = nullptr;
    if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
    return e;
  }
};

inline ProfileState& profile_state() {
  static ProfileState s;
  return s;
}

inline std::atomic<long long>& launch_counter() {
  static std::atomic<long long> c{0};
  return c;
}

inline void note_launch(int n = 1) { launch_counter().fetch_add(n, std::memory_order_relaxed); }

// Failure-path test knobs (gh_debug_set): each names one copy that the next
// launch of its kernel leaves out, so that a consumer's bounded wait runs
// out.  -1 (the default) leaves nothing out; a launch takes the value and
// resets it.
inline std::atomic<long long>& debug_ring_piece() {
  static std::atomic<long long> v{-1};
  return v;
}
inline std::atomic<long long>& debug_gemm_stage() {
  static std::atomic<long long> v{-1};
  return v;
}

class ProfileScope {
 public:
  ProfileScope(int kind, cudaStream_t stream) : stream_(stream) {
    ProfileState& s = profile_state();
    std::lock_guard<std::mutex> g(s.mu);
    if (!s.enabled) return;
    rec_.kind = kind;
    rec_.start = s.take();
    rec_.stop = s.take();
    if (!rec_.start || !rec_.stop) return;
    active_ = cudaEventRecord(rec_.start, stream_) == cudaSuccess;
  }
  ~ProfileScope() {
    if (!active_) return;
    ProfileState& s = profile_state();
    std::lock_guard<std::mutex> g(s.mu);
    if (cudaEventRecord(rec_.stop, stream_) == cudaSuccess) s.recs.push_back(rec_);
  }
  ProfileScope(const ProfileScope&) = delete;
  ProfileScope& operator=(const ProfileScope&) = delete;

 private:
  cudaStream_t stream_;
  ProfileState::Rec rec_{};
  bool active_ = false;
};

}  // namespace gh
