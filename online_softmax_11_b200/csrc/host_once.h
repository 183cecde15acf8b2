// host_once.h -- per-device set-up that is remembered only once it has succeeded.
//
// The library does some work once per device (device checks, kernel attributes, the
// address of a __device__ array).  std::call_once would also remember a failure, so a
// transient error on the first call (for example a call made while a stream is being
// captured, or before a context is usable) would poison that device for the life of the
// process.  OnceOnSuccess runs the set-up again on the next call until it succeeds;
// after that the fast path is a single acquire load.  Host code only, no CUDA types.
#pragma once

#include <atomic>
#include <mutex>

namespace fa {

struct OnceOnSuccess {
  std::atomic<bool> done{false};
  std::mutex mu;

  // Runs `init` (returning 0 on success, an error code otherwise) unless an earlier
  // call succeeded.  Concurrent first calls are serialised; a failed attempt leaves the
  // state untouched, so the next call tries again.
  template <typename F>
  int run(F&& init) {
    if (done.load(std::memory_order_acquire)) return 0;
    std::lock_guard<std::mutex> lock(mu);
    if (done.load(std::memory_order_relaxed)) return 0;
    const int rc = init();
    if (rc == 0) done.store(true, std::memory_order_release);
    return rc;
  }
};

}  // namespace fa
