// Regions of mutually independent calls on one stream (zero_overlap_begin / zero_overlap_end).
//
// The bulk-copy kernels are launched with programmatic stream serialization allowed. Outside a
// region each of them waits, before its first global-memory access, for the kernel before it
// to complete ("ordered"). Inside a region the first such launch is ordered and every later one
// is "chained": it may run alongside the kernels before it and waits for its predecessor only
// before exiting (the device side is pdl_enter / pdl_leave in zero_device.cuh). The state here
// is one flag per stream with an open region; the calls enqueue nothing, so they work the same
// while a CUDA graph is being captured.
#include <map>
#include <mutex>

#include <cuda_runtime.h>

#include "../../include/libzero.h"
#include "zero_internal.h"

namespace {

std::mutex g_overlap_mu;
std::map<cudaStream_t, bool> g_open;   // stream -> a bulk-copy launch has been made in the region

}  // namespace

namespace zk {

bool overlap_next(cudaStream_t stream) {
    std::lock_guard<std::mutex> lk(g_overlap_mu);
    auto it = g_open.find(stream);
    if (it == g_open.end()) return false;
    if (!it->second) {   // the region's first launch: ordered after everything before it
        it->second = true;
        return false;
    }
    return true;
}

}  // namespace zk

extern "C" {

zero_status zero_overlap_begin(zero_stream_t stream) {
    std::lock_guard<std::mutex> lk(g_overlap_mu);
    const cudaStream_t s = (cudaStream_t)stream;
    if (g_open.find(s) != g_open.end()) return ZERO_EINVAL;
    g_open[s] = false;
    return ZERO_OK;
}

zero_status zero_overlap_end(zero_stream_t stream) {
    std::lock_guard<std::mutex> lk(g_overlap_mu);
    auto it = g_open.find((cudaStream_t)stream);
    if (it == g_open.end()) return ZERO_EINVAL;
    g_open.erase(it);
    return ZERO_OK;
}

}  // extern "C"
