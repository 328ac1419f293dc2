// launch_stats.cuh -- host-side launch counting and optional per-kernel
// CUDA-event timing (measurement support for the benchmark; the scan itself
// does not depend on it).
#pragma once

#include <cuda_runtime.h>

#include <atomic>
#include <mutex>
#include <string>
#include <utility>
#include <vector>

namespace gdn {

struct LaunchStats {
    std::atomic<unsigned long long> launches{0};
    std::atomic<bool> timing{false};
    std::mutex mu;
    // per kernel name: event pairs recorded since the last read
    std::vector<std::pair<std::string, std::vector<std::pair<cudaEvent_t, cudaEvent_t>>>> events;

    static LaunchStats &get() {
        static LaunchStats s;
        return s;
    }
};

// Brackets one kernel launch: counts it and, when timing is on, records a
// start event before and an end event after it on the launch stream.
class LaunchScope {
  public:
    LaunchScope(const char *name, cudaStream_t stream) : name_(name), stream_(stream) {
        LaunchStats &st = LaunchStats::get();
        st.launches.fetch_add(1, std::memory_order_relaxed);
        if (!st.timing.load(std::memory_order_relaxed)) return;
        if (cudaEventCreate(&start_) != cudaSuccess) { start_ = nullptr; return; }
        if (cudaEventCreate(&end_) != cudaSuccess) { end_ = nullptr; release(); return; }
        active_ = cudaEventRecord(start_, stream_) == cudaSuccess;
        if (!active_) release();
    }
    ~LaunchScope() {
        if (!active_) return;
        if (cudaEventRecord(end_, stream_) != cudaSuccess) { release(); return; }
        LaunchStats &st = LaunchStats::get();
        std::lock_guard<std::mutex> g(st.mu);
        for (auto &e : st.events)
            if (e.first == name_) { e.second.emplace_back(start_, end_); return; }
        st.events.emplace_back(name_, std::vector<std::pair<cudaEvent_t, cudaEvent_t>>{{start_, end_}});
    }

  private:
    void release() {
        if (start_) cudaEventDestroy(start_);
        if (end_) cudaEventDestroy(end_);
        start_ = end_ = nullptr;
    }
    const char *name_;
    cudaStream_t stream_;
    cudaEvent_t start_ = nullptr, end_ = nullptr;
    bool active_ = false;
};

}  // namespace gdn
