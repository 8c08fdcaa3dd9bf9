// la_runtime.cuh — host-side launch accounting: a launch counter and an
// optional per-launch CUDA-event timer (la_profile_* in include/la_api.h).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>
#include <string.h>

#include <atomic>
#include <mutex>
#include <string>
#include <vector>

namespace la {

struct ProfRecord {
    const char* name;
    cudaEvent_t start, stop;
};

struct Profiler {
    std::atomic<uint64_t> launches{0};
    std::atomic<bool> on{false};
    std::mutex mu;
    std::vector<ProfRecord> records;
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

inline Profiler& profiler() {
    static Profiler p;
    return p;
}

// Brackets one kernel launch: counts it, and records start/stop events on the
// launch stream while profiling is enabled.
class LaunchScope {
   public:
    LaunchScope(const char* name, cudaStream_t st) : name_(name), st_(st) {
        Profiler& p = profiler();
        p.launches.fetch_add(1, std::memory_order_relaxed);
        if (p.on.load(std::memory_order_relaxed)) {
            std::lock_guard<std::mutex> g(p.mu);
            start_ = p.take();
            stop_ = p.take();
            if (start_) cudaEventRecord(start_, st_);
        }
    }
    ~LaunchScope() {
        if (!start_) return;
        Profiler& p = profiler();
        std::lock_guard<std::mutex> g(p.mu);
        if (stop_) {
            cudaEventRecord(stop_, st_);
            p.records.push_back({name_, start_, stop_});
        }
    }

   private:
    const char* name_;
    cudaStream_t st_;
    cudaEvent_t start_ = nullptr, stop_ = nullptr;
};

}  // namespace la
