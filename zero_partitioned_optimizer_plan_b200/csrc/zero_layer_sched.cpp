// Just-in-time layer scheduler for ZeRO stage 3.
//
// "ZeRO" (lastdictionary.com), main definition: with the parameters partitioned too, each
// layer's parameters are gathered just in time for its computation and discarded afterwards.
// "ZeRO: particionar estados do treino entre GPUs" (upskillscore.com), "Como funciona": a
// process that needs a parameter partition it does not own receives it from the owner; a step
// moves one parameter all-gather in the forward pass and another in the backward pass.
//
// The scheduler owns nothing on the device but CUDA events. The caller gives it a pool of layer
// buffers (device memory) and a gather stream. acquire(l) makes sure layer l sits gathered in
// one of the buffers -- gathering it on the gather stream if it is not already there from a
// prefetch -- and makes the caller's compute stream wait for that gather; it can also start
// the gather of the layer the pass needs next, so that it runs during layer l's computation.
// release(l) marks the point on the compute stream after which layer l's buffer may be
// overwritten: a later gather into it waits for that point. A released layer is discarded; the
// backward pass gathers it again. All ordering is carried by events; the host never blocks.
#include <cstdint>
#include <cstring>
#include <new>
#include <vector>

#include <cuda_runtime.h>

#include "../../include/libzero.h"
#include "zero_internal.h"

struct zero_layer_sched {
    const zero_plan* plan = nullptr;
    int nd = 0;
    uint64_t shard = 0;
    std::vector<uint64_t> bounds;         // n_layers + 1 flat offsets
    const uint16_t* shards[ZERO_MAX_RANKS] = {};
    uint16_t* buf_mem = nullptr;
    uint64_t buf_stride = 0;             // fp16 elements per buffer (16-byte multiple)
    int n_bufs = 0;
    cudaStream_t gs = nullptr;            // the gather stream
    uint32_t* status = nullptr;
    std::vector<cudaEvent_t> gathered;    // per buffer: the last gather into it
    std::vector<cudaEvent_t> released;    // per buffer: its last user's release point
    std::vector<uint64_t> rel_seq;        // per buffer: number of its last release (0: none)
    std::vector<cudaStream_t> rel_stream; // per buffer: the stream of its last release
    uint64_t n_releases = 0;              // releases so far (numbers them)
    // The gather stream has waited for every release on covered_stream numbered up to
    // covered_seq (releases on one stream are ordered, so one wait covers the earlier ones).
    cudaStream_t covered_stream = nullptr;
    uint64_t covered_seq = 0;
    std::vector<int> layer_of_buf;        // per buffer: the layer it holds (-1: none)
    std::vector<int> buf_of_layer;        // per layer: the buffer holding it (-1: none)
    std::vector<int> held;                // per layer: acquired and not yet released
    std::vector<uint64_t> stamp;          // per buffer: when it was last filled or released
    uint64_t clock = 0;
    cudaEvent_t step_ev = nullptr;
    uint64_t gathers = 0;
};

namespace {

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

bool overlap(const void* a, uint64_t na, const void* b, uint64_t nb) {
    if (na == 0 || nb == 0) return false;
    const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
    return x < y + nb && y < x + na;
}

uint64_t round8(uint64_t x) { return (x + 7) & ~(uint64_t)7; }

// Layer bounds: 0 = b[0] < b[1] < ... < b[n], b[n] in [psi, psi_p]. Longest layer into *longest.
bool bounds_ok(const zero_plan* plan, int n_layers, const uint64_t* b, uint64_t* longest) {
    uint64_t psi = 0, psi_p = 0;
    if (!plan || !b || n_layers < 1 || zero_plan_info(plan, &psi, &psi_p, nullptr, nullptr))
        return false;
    if (b[0] != 0 || b[n_layers] < psi || b[n_layers] > psi_p) return false;
    uint64_t m = 0;
    for (int l = 0; l < n_layers; ++l) {
        if (b[l + 1] <= b[l]) return false;
        if (b[l + 1] - b[l] > m) m = b[l + 1] - b[l];
    }
    if (longest) *longest = m;
    return true;
}

void destroy_events(zero_layer_sched* s) {
    for (cudaEvent_t e : s->gathered)
        if (e) cudaEventDestroy(e);
    for (cudaEvent_t e : s->released)
        if (e) cudaEventDestroy(e);
    if (s->step_ev) cudaEventDestroy(s->step_ev);
    s->gathered.clear();
    s->released.clear();
    s->step_ev = nullptr;
}

uint16_t* buffer(const zero_layer_sched* s, int b) {
    return s->buf_mem + (size_t)b * s->buf_stride;
}

// A buffer for a new gather: one holding no layer, else the least recently used one that holds
// a prefetched layer nobody has acquired (never a held layer). -1 if none.
int free_buffer(const zero_layer_sched* s) {
    int best = -1;
    for (int b = 0; b < s->n_bufs; ++b) {
        const int l = s->layer_of_buf[(size_t)b];
        if (l >= 0 && s->held[(size_t)l]) continue;
        const bool empty = l < 0;
        if (best < 0) {
            best = b;
            continue;
        }
        const bool best_empty = s->layer_of_buf[(size_t)best] < 0;
        if ((empty && !best_empty) ||
            (empty == best_empty && s->stamp[(size_t)b] < s->stamp[(size_t)best]))
            best = b;
    }
    return best;
}

// Make the gather stream wait for buffer b's last release, unless an earlier wait already
// covers it. The wait is on the latest release recorded on that stream (covering every buffer
// released there so far), so that consecutive gathers are not each separated by a wait: a wait
// between two kernels on the gather stream ends the programmatic overlap of the second one's
// launch with the first one's tail.
cudaError_t wait_release(zero_layer_sched* s, int b) {
    const uint64_t need = s->rel_seq[(size_t)b];
    const cudaStream_t st = s->rel_stream[(size_t)b];
    if (need == 0 || (st == s->covered_stream && need <= s->covered_seq)) return cudaSuccess;
    int latest = b;
    for (int i = 0; i < s->n_bufs; ++i)
        if (s->rel_stream[(size_t)i] == st && s->rel_seq[(size_t)i] > s->rel_seq[(size_t)latest])
            latest = i;
    const cudaError_t e = cudaStreamWaitEvent(s->gs, s->released[(size_t)latest], 0);
    if (e == cudaSuccess) {
        s->covered_stream = st;
        s->covered_seq = s->rel_seq[(size_t)latest];
    }
    return e;
}

// Gather layer l into buffer b on the gather stream, after the buffer's last release.
zero_status gather_into(zero_layer_sched* s, int l, int b) {
    const int old = s->layer_of_buf[(size_t)b];
    if (old >= 0) s->buf_of_layer[(size_t)old] = -1;   // an unused prefetch, dropped
    s->layer_of_buf[(size_t)b] = -1;
    if (wait_release(s, b) != cudaSuccess) return zk::from_cuda(cudaGetLastError());
    const uint64_t lo = s->bounds[(size_t)l], len = s->bounds[(size_t)l + 1] - lo;
    cudaError_t e = zk::launch_gather(lo, len, s->shard, s->nd, s->shards, buffer(s, b),
                                      s->status, s->gs);
    if (e == cudaSuccess) e = cudaEventRecord(s->gathered[(size_t)b], s->gs);
    if (e != cudaSuccess) return zk::from_cuda(e);
    ++s->gathers;
    s->layer_of_buf[(size_t)b] = l;
    s->buf_of_layer[(size_t)l] = b;
    s->stamp[(size_t)b] = ++s->clock;
    return ZERO_OK;
}

}  // namespace

extern "C" {

zero_status zero_layer_sched_buf_elems(const zero_plan* plan, int n_layers,
                                       const uint64_t* layer_bounds, int n_bufs,
                                       uint64_t* elems) {
    uint64_t longest = 0;
    if (!elems || n_bufs < 1 || !bounds_ok(plan, n_layers, layer_bounds, &longest))
        return ZERO_EINVAL;
    *elems = (uint64_t)n_bufs * round8(longest);
    return ZERO_OK;
}

zero_status zero_layer_sched_create(const zero_plan* plan, int n_layers,
                                    const uint64_t* layer_bounds,
                                    const uint16_t* const* param_shards, uint16_t* buf_mem,
                                    uint64_t buf_mem_elems, int n_bufs,
                                    zero_stream_t gather_stream, zero_layer_sched** out) {
    if (!out) return ZERO_EINVAL;
    *out = nullptr;
    int nd = 0;
    uint64_t psi_p = 0, S = 0, longest = 0;
    if (!zk::plan_geometry(plan, &nd, &psi_p, &S) || n_bufs < 1 || !param_shards || !buf_mem ||
        !bounds_ok(plan, n_layers, layer_bounds, &longest))
        return ZERO_EINVAL;
    if (!aligned(buf_mem, 16)) return ZERO_EALIGN;
    uint64_t need = 0;
    zero_layer_sched_buf_elems(plan, n_layers, layer_bounds, n_bufs, &need);
    if (buf_mem_elems < need) return ZERO_ENOMEM;
    for (int q = 0; q < nd; ++q) {
        if (!param_shards[q]) return ZERO_EINVAL;
        if (!aligned(param_shards[q], 2)) return ZERO_EALIGN;
        if (overlap(buf_mem, need * 2, param_shards[q], S * 2)) return ZERO_EINVAL;
    }
    zero_layer_sched* s = new (std::nothrow) zero_layer_sched();
    if (!s) return ZERO_ENOMEM;
    s->plan = plan;
    s->nd = nd;
    s->shard = S;
    for (int q = 0; q < nd; ++q) s->shards[q] = param_shards[q];
    s->buf_mem = buf_mem;
    s->buf_stride = round8(longest);
    s->n_bufs = n_bufs;
    s->gs = (cudaStream_t)gather_stream;
    try {
        s->bounds.assign(layer_bounds, layer_bounds + n_layers + 1);
        s->gathered.assign((size_t)n_bufs, nullptr);
        s->released.assign((size_t)n_bufs, nullptr);
        s->rel_seq.assign((size_t)n_bufs, 0);
        s->rel_stream.assign((size_t)n_bufs, nullptr);
        s->layer_of_buf.assign((size_t)n_bufs, -1);
        s->stamp.assign((size_t)n_bufs, 0);
        s->buf_of_layer.assign((size_t)n_layers, -1);
        s->held.assign((size_t)n_layers, 0);
    } catch (...) {
        delete s;
        return ZERO_ENOMEM;
    }
    bool ok = cudaEventCreateWithFlags(&s->step_ev, cudaEventDisableTiming) == cudaSuccess;
    for (int b = 0; ok && b < n_bufs; ++b)
        ok = cudaEventCreateWithFlags(&s->gathered[(size_t)b], cudaEventDisableTiming) ==
                 cudaSuccess &&
             cudaEventCreateWithFlags(&s->released[(size_t)b], cudaEventDisableTiming) ==
                 cudaSuccess;
    if (!ok) {
        const zero_status st = zk::from_cuda(cudaGetLastError());
        destroy_events(s);
        delete s;
        return st == ZERO_OK ? ZERO_ECUDA : st;
    }
    *out = s;
    return ZERO_OK;
}

zero_status zero_layer_sched_begin_step(zero_layer_sched* s, uint32_t* d_status,
                                        zero_stream_t stream) {
    if (!s || !d_status) return ZERO_EINVAL;
    if (!aligned(d_status, 4)) return ZERO_EALIGN;
    for (int h : s->held)
        if (h) return ZERO_EINVAL;   // a layer of the last step was never released
    for (int q = 0; q < s->nd; ++q)
        if (overlap(d_status, 4, s->shards[q], s->shard * 2)) return ZERO_EINVAL;
    if (overlap(d_status, 4, s->buf_mem, (uint64_t)s->n_bufs * s->buf_stride * 2))
        return ZERO_EINVAL;
    // what was gathered before now is stale: the partitions have been updated since
    for (int b = 0; b < s->n_bufs; ++b) s->layer_of_buf[(size_t)b] = -1;
    for (int& l : s->buf_of_layer) l = -1;
    s->status = d_status;
    cudaError_t e = cudaEventRecord(s->step_ev, (cudaStream_t)stream);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(s->gs, s->step_ev, 0);
    if (e != cudaSuccess) return zk::from_cuda(e);
    s->covered_stream = (cudaStream_t)stream;   // every release on `stream` so far is covered
    s->covered_seq = s->n_releases;
    return ZERO_OK;
}

zero_status zero_layer_sched_acquire(zero_layer_sched* s, int layer, int prefetch,
                                     zero_stream_t compute, uint16_t** layer_params) {
    if (!s || !layer_params || !s->status) return ZERO_EINVAL;
    const int L = (int)s->held.size();
    if (layer < 0 || layer >= L || s->held[(size_t)layer]) return ZERO_EINVAL;
    if (prefetch >= L || prefetch == layer) prefetch = -1;
    int b = s->buf_of_layer[(size_t)layer];
    if (b < 0) {
        b = free_buffer(s);
        if (b < 0) return ZERO_ENOMEM;   // every buffer holds an acquired layer
        const zero_status st = gather_into(s, layer, b);
        if (st != ZERO_OK) return st;
    }
    if (cudaStreamWaitEvent((cudaStream_t)compute, s->gathered[(size_t)b], 0) != cudaSuccess)
        return zk::from_cuda(cudaGetLastError());
    s->held[(size_t)layer] = 1;
    *layer_params = buffer(s, b);
    if (prefetch >= 0 && !s->held[(size_t)prefetch] && s->buf_of_layer[(size_t)prefetch] < 0) {
        const int pb = free_buffer(s);
        if (pb >= 0) return gather_into(s, prefetch, pb);   // no free buffer: no prefetch
    }
    return ZERO_OK;
}

zero_status zero_layer_sched_release(zero_layer_sched* s, int layer, zero_stream_t compute) {
    if (!s || layer < 0 || layer >= (int)s->held.size() || !s->held[(size_t)layer])
        return ZERO_EINVAL;
    const int b = s->buf_of_layer[(size_t)layer];
    if (b < 0) return ZERO_EINVAL;
    const cudaError_t e = cudaEventRecord(s->released[(size_t)b], (cudaStream_t)compute);
    if (e != cudaSuccess) return zk::from_cuda(e);
    s->rel_seq[(size_t)b] = ++s->n_releases;
    s->rel_stream[(size_t)b] = (cudaStream_t)compute;
    s->held[(size_t)layer] = 0;
    s->buf_of_layer[(size_t)layer] = -1;   // discarded
    s->layer_of_buf[(size_t)b] = -1;
    s->stamp[(size_t)b] = ++s->clock;
    return ZERO_OK;
}

zero_status zero_layer_sched_gathers(const zero_layer_sched* s, uint64_t* count) {
    if (!s || !count) return ZERO_EINVAL;
    *count = s->gathers;
    return ZERO_OK;
}

void zero_layer_sched_destroy(zero_layer_sched* s) {
    if (!s) return;
    destroy_events(s);
    delete s;
}

}  // extern "C"
