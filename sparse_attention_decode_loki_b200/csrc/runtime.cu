// Per-device launch-shape cache: SM count, opt-in shared memory and the
// resident-CTA count of each kernel instantiation. Grids are sized as
// (SM count x resident CTAs per SM) so every CTA of a persistent split runs in
// a single wave.
#include <mutex>
#include <set>
#include <unordered_map>
#include <utility>

#include "launch.h"

namespace loki {

// Set by a kernel whose bounded wait on an asynchronous copy gave up (see
// tma.cuh); read and cleared through loki_device_error().
__device__ int g_device_error;

namespace {
constexpr int kMaxDevices = 64;
int* g_err_ptr[kMaxDevices] = {};
std::mutex g_mu;
DevInfo g_dev[kMaxDevices];
bool g_dev_ok[kMaxDevices] = {};

struct OccKey {
    const void* f;
    int dev, threads;
    size_t smem;
    bool operator==(const OccKey& o) const {
        return f == o.f && dev == o.dev && threads == o.threads && smem == o.smem;
    }
};
struct OccHash {
    size_t operator()(const OccKey& k) const {
        return std::hash<const void*>()(k.f) ^ (size_t(k.dev) << 1) ^ (size_t(k.threads) << 7) ^
               (k.smem << 17);
    }
};
std::unordered_map<OccKey, int, OccHash> g_occ;
std::set<std::pair<int, const void*>> g_carveout_set;
}  // namespace

cudaError_t prefer_carveout(const void* func, int carveout) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    std::lock_guard<std::mutex> lk(g_mu);
    if (g_carveout_set.count({dev, func})) return cudaSuccess;
    e = cudaFuncSetAttribute(func, cudaFuncAttributePreferredSharedMemoryCarveout, carveout);
    if (e != cudaSuccess) return e;
    g_carveout_set.insert({dev, func});
    return cudaSuccess;
}

cudaError_t dev_info(DevInfo* out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lk(g_mu);
    if (!g_dev_ok[dev]) {
        DevInfo d{dev, 0, 0};
        e = cudaDeviceGetAttribute(&d.sm_count, cudaDevAttrMultiProcessorCount, dev);
        if (e != cudaSuccess) return e;
        e = cudaDeviceGetAttribute(&d.smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
        if (e != cudaSuccess) return e;
        g_dev[dev] = d;
        g_dev_ok[dev] = true;
    }
    *out = g_dev[dev];
    return cudaSuccess;
}

int* device_error_word() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    std::lock_guard<std::mutex> lk(g_mu);
    if (g_err_ptr[dev] == nullptr) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_device_error) != cudaSuccess) return nullptr;
        g_err_ptr[dev] = static_cast<int*>(p);
    }
    return g_err_ptr[dev];
}

int occupancy(const void* func, int threads, size_t smem) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 1;
    OccKey key{func, dev, threads, smem};
    {
        std::lock_guard<std::mutex> lk(g_mu);
        auto it = g_occ.find(key);
        if (it != g_occ.end()) return it->second;
    }
    int n = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, func, threads, smem) != cudaSuccess ||
        n < 1)
        n = 1;
    std::lock_guard<std::mutex> lk(g_mu);
    g_occ[key] = n;
    return n;
}

}  // namespace loki
