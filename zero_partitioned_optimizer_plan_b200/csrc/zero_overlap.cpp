// Regions of mutually independent calls on one stream (zero_overlap_begin / zero_overlap_end).
//
// The bulk-copy kernels are launched with programmatic stream serialization allowed. Outside a
// region each of them waits, before its first global-memory access, for the kernel before it
// to complete ("ordered"). Inside a region the first such launch is ordered and every later one
// is "chained": it may run alongside the kernels before it and waits for its predecessor only
// before exiting (the device side is pdl_enter / pdl_leave in zero_device.cuh). The state here
// is one entry per stream with an open region; the calls enqueue nothing, so they work the same
// while a CUDA graph is being captured.
//
// The launch path reads the table without a lock: a count of open regions (zero on the common
// path outside any region) and, inside one, a scan of a fixed table of kMaxRegions entries.
// Opening and closing regions, which are rare, serialise on a mutex.
#include <atomic>
#include <mutex>

#include <cuda_runtime.h>

#include "../../include/libzero.h"
#include "zero_internal.h"

namespace {

constexpr int kMaxRegions = 64;

struct Region {
    std::atomic<int> open{0};
    std::atomic<cudaStream_t> stream{nullptr};
    std::atomic<int> launched{0};   // a bulk-copy launch has been made in the region
};

Region g_regions[kMaxRegions];
std::atomic<int> g_open{0};
std::mutex g_change_mu;

Region* find(cudaStream_t s) {
    for (Region& r : g_regions)
        if (r.open.load(std::memory_order_acquire) && r.stream.load(std::memory_order_relaxed) == s)
            return &r;
    return nullptr;
}

}  // namespace

namespace zk {

bool overlap_next(cudaStream_t stream) {
    if (g_open.load(std::memory_order_acquire) == 0) return false;
    Region* r = find(stream);
    if (!r) return false;
    // the region's first launch is ordered after everything before it; later ones chain
    return r->launched.exchange(1, std::memory_order_relaxed) != 0;
}

}  // namespace zk

extern "C" {

zero_status zero_overlap_begin(zero_stream_t stream) {
    std::lock_guard<std::mutex> lk(g_change_mu);
    const cudaStream_t s = (cudaStream_t)stream;
    if (find(s)) return ZERO_EINVAL;
    for (Region& r : g_regions) {
        if (r.open.load(std::memory_order_relaxed)) continue;
        r.stream.store(s, std::memory_order_relaxed);
        r.launched.store(0, std::memory_order_relaxed);
        r.open.store(1, std::memory_order_release);
        g_open.fetch_add(1, std::memory_order_release);
        return ZERO_OK;
    }
    return ZERO_ENOMEM;   // kMaxRegions regions are open
}

zero_status zero_overlap_end(zero_stream_t stream) {
    std::lock_guard<std::mutex> lk(g_change_mu);
    Region* r = find((cudaStream_t)stream);
    if (!r) return ZERO_EINVAL;
    r->open.store(0, std::memory_order_release);
    g_open.fetch_sub(1, std::memory_order_release);
    return ZERO_OK;
}

}  // extern "C"
