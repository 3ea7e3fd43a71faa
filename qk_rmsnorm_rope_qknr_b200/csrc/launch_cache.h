// Launch facts that stay fixed for a (kernel, device) pair, looked up once
// instead of on every call: the device's SM count, the dynamic shared memory
// a kernel has been granted, and how many of its CTAs fit on an SM for a given
// block and dynamic shared memory size. The driver queries behind them cost
// microseconds, which matters for launches of a few microseconds of work.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>
#include <unordered_map>

namespace qknr {

namespace launch_cache_detail {

struct Key {
    const void* kern;
    int device, block, smem;
    bool operator==(const Key& o) const {
        return kern == o.kern && device == o.device && block == o.block && smem == o.smem;
    }
};

struct KeyHash {
    size_t operator()(const Key& k) const {
        uint64_t h = reinterpret_cast<uintptr_t>(k.kern);
        h = h * 1000003u ^ (uint64_t)(uint32_t)k.device;
        h = h * 1000003u ^ (uint64_t)(uint32_t)k.block;
        h = h * 1000003u ^ (uint64_t)(uint32_t)k.smem;
        return (size_t)h;
    }
};

struct State {
    std::mutex mu;
    std::unordered_map<int, int> sms;                  // device -> SM count
    std::unordered_map<Key, int, KeyHash> granted;     // (kernel, device) -> smem granted
    std::unordered_map<Key, int, KeyHash> occupancy;   // (kernel, device, block, smem) -> CTAs/SM
};

inline State& state() {
    static State s;
    return s;
}

}  // namespace launch_cache_detail

// SM count of the current device.
inline cudaError_t cached_sm_count(int* out) {
    using namespace launch_cache_detail;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    State& s = state();
    std::lock_guard<std::mutex> lock(s.mu);
    auto it = s.sms.find(dev);
    if (it != s.sms.end()) {
        *out = it->second;
        return cudaSuccess;
    }
    int n = 0;
    e = cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    s.sms.emplace(dev, n);
    *out = n;
    return cudaSuccess;
}

// Lets `kern` use `smem` bytes of dynamic shared memory on the current device
// (a no-op once it has been granted as much or more), and returns how many of
// its CTAs of `block` threads fit on one SM with that much (0 if none).
inline cudaError_t cached_smem_and_occupancy(const void* kern, int block, int smem,
                                             int* ctas_per_sm) {
    using namespace launch_cache_detail;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    State& s = state();
    std::lock_guard<std::mutex> lock(s.mu);
    const Key gk{kern, dev, 0, 0};
    auto g = s.granted.find(gk);
    if (smem > 48 * 1024 && (g == s.granted.end() || g->second < smem)) {
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e != cudaSuccess) return e;
        s.granted[gk] = smem;
    }
    const Key ok{kern, dev, block, smem};
    auto o = s.occupancy.find(ok);
    if (o != s.occupancy.end()) {
        *ctas_per_sm = o->second;
        return cudaSuccess;
    }
    int n = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kern, block, smem);
    if (e != cudaSuccess) return e;
    s.occupancy.emplace(ok, n);
    *ctas_per_sm = n;
    return cudaSuccess;
}

// Drops what is known about `kern`: a reset of the device's context takes
// back the shared memory it was granted, so a launch that fails is retried
// once after forgetting.
inline void forget_kernel(const void* kern) {
    using namespace launch_cache_detail;
    State& s = state();
    std::lock_guard<std::mutex> lock(s.mu);
    for (auto* m : {&s.granted, &s.occupancy}) {
        for (auto it = m->begin(); it != m->end();) {
            if (it->first.kern == kern) {
                it = m->erase(it);
            } else {
                ++it;
            }
        }
    }
}

}  // namespace qknr
