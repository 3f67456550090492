// Stream-ordered bucket scheduler for ZeRO stage 2.
//
// "ZeRO-2" card (llm-engineer.pages.dev), section "Gradient 생명주기": during the backward pass
// each layer's (bucket's) local gradient is reduce-scattered as soon as it exists; the GPU keeps
// only its own reduced shard and releases the rest of the local gradient; this repeats for
// every bucket. Diagram: buckets B2, B1, B0 are produced and reduce-scattered in that order.
//
// Here the local gradients of a bucket (all Nd simulated ranks) live in a staging slot. The
// producer (the backward pass, or whatever stands for it) fills the slot on its own stream; the
// reduce-scatter runs on the scheduler's stream after a CUDA event says the fill is done; when
// the reduce-scatter has read the slot, another event releases the slot, and the producer's
// stream waits on that event before it fills the slot with a later bucket. The host never
// blocks: all ordering is carried by events, so the fill of bucket k+1 overlaps the
// reduce-scatter of bucket k whenever more than one slot exists.
//
// In the fused mode (zero_sched_create_fused) the kernel launched for a bucket is the fused
// step over the bucket's range -- reduce, unscale, Adam, fp16 cast and write-back -- so the
// reduced gradient never reaches memory; the caller commits the step after the last bucket.
// The int8 mode (zero_sched_create_fused_q8) does the same with each rank's bucket arriving as
// int8 records with their scales ("ZeRO" (lastdictionary.com): ZeRO++ compresses the
// communication), reduced by the int8 fused step.
#include <cstdint>
#include <cstring>
#include <new>
#include <vector>

#include <cuda_runtime.h>

#include "../../include/libzero.h"
#include "zero_internal.h"

struct zero_sched {
    const zero_plan* plan = nullptr;
    int nd = 0;
    int n_slots = 0;
    uint64_t stride = 0;                 // fp16 elements per rank region of a slot
    uint16_t* slot_mem = nullptr;
    float* shards[ZERO_MAX_RANKS] = {};
    uint32_t* status = nullptr;
    cudaStream_t rs = nullptr;
    std::vector<cudaEvent_t> produced;   // per slot: the producer finished filling it
    std::vector<cudaEvent_t> released;   // per slot: its last reduce-scatter finished
    std::vector<int> filled;             // per slot: released[] has been recorded once
    std::vector<int> bucket_of_slot;     // per slot: the bucket begun in it (-1: none)
    cudaEvent_t tail = nullptr;          // scratch event for zero_sched_wait
    uint64_t launches = 0;
    // fused mode: the step's state (flat, psi_p elements each) and constants
    bool fused = false;
    const float* w_in = nullptr;
    const float* m_in = nullptr;
    const float* v_in = nullptr;
    float* w_out = nullptr;
    float* m_out = nullptr;
    float* v_out = nullptr;
    uint16_t* param_out = nullptr;
    const zero_adam_consts* consts = nullptr;
    // int8 mode (fused only): the slots hold each rank's int8 records of a bucket, in
    // region_bytes-byte regions of slot_bytes (slot_mem is unused)
    bool q8 = false;
    uint8_t* slot_bytes = nullptr;
    uint64_t region_bytes = 0;
};

namespace {

uint64_t round8(uint64_t x) { return (x + 7) & ~(uint64_t)7; }

uint64_t round16(uint64_t x) { return (x + 15) & ~(uint64_t)15; }

// Bytes of one rank's region in an int8 slot: the longest bucket's records, 16-byte multiple.
uint64_t q8_region(const zero_plan* plan) {
    return round16(ZERO_Q8_PAYLOAD_BYTES(zk::plan_max_bucket(plan)));
}

void destroy_events(zero_sched* s) {
    for (cudaEvent_t e : s->produced)
        if (e) cudaEventDestroy(e);
    for (cudaEvent_t e : s->released)
        if (e) cudaEventDestroy(e);
    if (s->tail) cudaEventDestroy(s->tail);
    s->produced.clear();
    s->released.clear();
    s->tail = nullptr;
}

}  // namespace

extern "C" {

zero_status zero_sched_slot_elems(const zero_plan* plan, int n_slots, uint64_t* elems) {
    int nd = 0;
    uint64_t psi_p = 0, S = 0;
    if (!elems || n_slots < 1 || !zk::plan_geometry(plan, &nd, &psi_p, &S)) return ZERO_EINVAL;
    *elems = (uint64_t)n_slots * (uint64_t)nd * round8(zk::plan_max_bucket(plan));
    return ZERO_OK;
}

zero_status zero_sched_slot_bytes_q8(const zero_plan* plan, int n_slots, uint64_t* bytes) {
    int nd = 0;
    uint64_t psi_p = 0, S = 0;
    if (!bytes || n_slots < 1 || !zk::plan_geometry(plan, &nd, &psi_p, &S)) return ZERO_EINVAL;
    *bytes = (uint64_t)n_slots * (uint64_t)nd * q8_region(plan);
    return ZERO_OK;
}

}  // extern "C"

namespace {

// Validation and set-up shared by every mode (everything but what the bucket kernel writes).
// slot_mem: fp16 slots of slot_size elements, or (q8) int8-record slots of slot_size bytes.
zero_status create_common(const zero_plan* plan, void* slot_mem, uint64_t slot_size, bool q8,
                          int n_slots, uint32_t* d_status, cudaStream_t stream, zero_sched** out) {
    if (!out) return ZERO_EINVAL;
    *out = nullptr;
    int nd = 0;
    uint64_t psi_p = 0, S = 0;
    if (!zk::plan_geometry(plan, &nd, &psi_p, &S) || n_slots < 1 || !slot_mem || !d_status)
        return ZERO_EINVAL;
    if ((reinterpret_cast<uintptr_t>(slot_mem) & 15u) || (reinterpret_cast<uintptr_t>(d_status) & 3u))
        return ZERO_EALIGN;
    uint64_t need = 0;
    if (q8)
        zero_sched_slot_bytes_q8(plan, n_slots, &need);
    else
        zero_sched_slot_elems(plan, n_slots, &need);
    if (slot_size < need) return ZERO_ENOMEM;
    zero_sched* s = new (std::nothrow) zero_sched();
    if (!s) return ZERO_ENOMEM;
    s->plan = plan;
    s->nd = nd;
    s->n_slots = n_slots;
    s->q8 = q8;
    if (q8) {
        s->slot_bytes = static_cast<uint8_t*>(slot_mem);
        s->region_bytes = q8_region(plan);
    } else {
        s->stride = round8(zk::plan_max_bucket(plan));
        s->slot_mem = static_cast<uint16_t*>(slot_mem);
    }
    s->status = d_status;
    s->rs = stream;
    try {
        s->produced.assign((size_t)n_slots, nullptr);
        s->released.assign((size_t)n_slots, nullptr);
        s->filled.assign((size_t)n_slots, 0);
        s->bucket_of_slot.assign((size_t)n_slots, -1);
    } catch (...) {
        delete s;
        return ZERO_ENOMEM;
    }
    bool ok = cudaEventCreateWithFlags(&s->tail, cudaEventDisableTiming) == cudaSuccess;
    for (int i = 0; ok && i < n_slots; ++i) {
        ok = cudaEventCreateWithFlags(&s->produced[(size_t)i], cudaEventDisableTiming) == cudaSuccess &&
             cudaEventCreateWithFlags(&s->released[(size_t)i], cudaEventDisableTiming) == cudaSuccess;
    }
    if (!ok) {
        const zero_status st = zk::from_cuda(cudaGetLastError());
        destroy_events(s);
        delete s;
        return st == ZERO_OK ? ZERO_ECUDA : st;
    }
    *out = s;
    return ZERO_OK;
}

bool overlaps(const void* a, uint64_t na, const void* b, uint64_t nb) {
    const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
    return na && nb && x < y + nb && y < x + na;
}

// The staging slots' memory as bytes (either mode), for the overlap checks.
void slot_span(const zero_sched* s, const void** base, uint64_t* bytes) {
    if (s->q8) {
        *base = s->slot_bytes;
        *bytes = (uint64_t)s->n_slots * (uint64_t)s->nd * s->region_bytes;
    } else {
        *base = s->slot_mem;
        *bytes = (uint64_t)s->n_slots * (uint64_t)s->nd * s->stride * 2;
    }
}

// Outputs and the status word against the slots (the bucket kernels read the slots).
bool state_overlaps_slots(const void* slots, uint64_t slot_bytes, uint64_t psi_p,
                          const float* master_out, const float* m_out, const float* v_out,
                          const uint16_t* param_out, const uint32_t* d_status) {
    const void* outs[4] = {master_out, m_out, v_out, param_out};
    const uint64_t olen[4] = {psi_p * 4, psi_p * 4, psi_p * 4, psi_p * 2};
    for (int i = 0; i < 4; ++i)
        if (overlaps(outs[i], olen[i], slots, slot_bytes)) return true;
    return overlaps(d_status, 4, slots, slot_bytes);
}

// The slot of bucket k: make `producer` wait for its release and mark it begun.
zero_status begin_slot(zero_sched* s, int k, zero_stream_t producer, int* slot_out) {
    uint64_t lo = 0, len = 0;
    if (!zk::plan_bucket_range(s->plan, k, &lo, &len)) return ZERO_EINVAL;
    const int slot = k % s->n_slots;
    // the slot still holds a bucket that was begun and not ended: its fill would be lost
    if (s->bucket_of_slot[(size_t)slot] != -1) return ZERO_EINVAL;
    if (s->filled[(size_t)slot]) {
        // the slot still holds an earlier bucket until its kernel has finished
        if (cudaError_t e = cudaStreamWaitEvent((cudaStream_t)producer, s->released[(size_t)slot], 0); e != cudaSuccess)
            return zk::from_cuda(e);
    }
    s->bucket_of_slot[(size_t)slot] = k;
    *slot_out = slot;
    return ZERO_OK;
}

}  // namespace

extern "C" {

zero_status zero_sched_create(const zero_plan* plan, uint16_t* slot_mem, uint64_t slot_mem_elems,
                              int n_slots, float* const* owner_grad_shards, uint32_t* d_status,
                              zero_stream_t rs_stream, zero_sched** out) {
    int nd = 0;
    uint64_t psi_p = 0, S = 0;
    if (!out) return ZERO_EINVAL;
    *out = nullptr;
    if (!zk::plan_geometry(plan, &nd, &psi_p, &S) || !owner_grad_shards) return ZERO_EINVAL;
    for (int r = 0; r < nd; ++r) {
        if (!owner_grad_shards[r]) return ZERO_EINVAL;
        if (reinterpret_cast<uintptr_t>(owner_grad_shards[r]) & 3u) return ZERO_EALIGN;
    }
    zero_sched* s = nullptr;
    const zero_status st = create_common(plan, slot_mem, slot_mem_elems, false, n_slots,
                                         d_status, (cudaStream_t)rs_stream, &s);
    if (st != ZERO_OK) return st;
    for (int r = 0; r < nd; ++r) s->shards[r] = owner_grad_shards[r];
    *out = s;
    return ZERO_OK;
}

zero_status zero_sched_create_fused(const zero_plan* plan, uint16_t* slot_mem,
                                    uint64_t slot_mem_elems, int n_slots, const float* master_in,
                                    const float* m_in, const float* v_in, float* master_out,
                                    float* m_out, float* v_out, uint16_t* param_out,
                                    const zero_adam_consts* d_consts, uint32_t* d_status,
                                    zero_stream_t stream, zero_sched** out) {
    int nd = 0;
    uint64_t psi_p = 0, S = 0;
    if (!out) return ZERO_EINVAL;
    *out = nullptr;
    if (!zk::plan_geometry(plan, &nd, &psi_p, &S) || !d_consts) return ZERO_EINVAL;
    if (reinterpret_cast<uintptr_t>(d_consts) & 3u) return ZERO_EALIGN;
    zero_status st = zk::check_fused_state(psi_p, master_in, m_in, v_in, master_out, m_out, v_out,
                                           param_out, d_status);
    if (st != ZERO_OK) return st;
    // the staging slots are read by the bucket kernels: no output may overlap them
    uint64_t need = 0;
    zero_sched_slot_elems(plan, n_slots < 1 ? 1 : n_slots, &need);
    const void* outs[4] = {master_out, m_out, v_out, param_out};
    const uint64_t olen[4] = {psi_p * 4, psi_p * 4, psi_p * 4, psi_p * 2};
    for (int i = 0; i < 4; ++i)
        if (overlaps(outs[i], olen[i], slot_mem, need * 2)) return ZERO_EINVAL;
    if (overlaps(d_status, 4, slot_mem, need * 2)) return ZERO_EINVAL;
    zero_sched* s = nullptr;
    st = create_common(plan, slot_mem, slot_mem_elems, false, n_slots, d_status,
                       (cudaStream_t)stream, &s);
    if (st != ZERO_OK) return st;
    s->fused = true;
    s->w_in = master_in;
    s->m_in = m_in;
    s->v_in = v_in;
    s->w_out = master_out;
    s->m_out = m_out;
    s->v_out = v_out;
    s->param_out = param_out;
    s->consts = d_consts;
    *out = s;
    return ZERO_OK;
}

zero_status zero_sched_create_fused_q8(const zero_plan* plan, uint8_t* slot_mem,
                                       uint64_t slot_mem_bytes, int n_slots,
                                       const float* master_in, const float* m_in,
                                       const float* v_in, float* master_out, float* m_out,
                                       float* v_out, uint16_t* param_out,
                                       const zero_adam_consts* d_consts, uint32_t* d_status,
                                       zero_stream_t stream, zero_sched** out) {
    int nd = 0;
    uint64_t psi_p = 0, S = 0;
    if (!out) return ZERO_EINVAL;
    *out = nullptr;
    if (!zk::plan_geometry(plan, &nd, &psi_p, &S) || !d_consts) return ZERO_EINVAL;
    if (reinterpret_cast<uintptr_t>(d_consts) & 3u) return ZERO_EALIGN;
    zero_status st = zk::check_fused_state(psi_p, master_in, m_in, v_in, master_out, m_out, v_out,
                                           param_out, d_status);
    if (st != ZERO_OK) return st;
    uint64_t need = 0;
    zero_sched_slot_bytes_q8(plan, n_slots < 1 ? 1 : n_slots, &need);
    if (state_overlaps_slots(slot_mem, need, psi_p, master_out, m_out, v_out, param_out,
                             d_status))
        return ZERO_EINVAL;
    zero_sched* s = nullptr;
    st = create_common(plan, slot_mem, slot_mem_bytes, true, n_slots, d_status,
                       (cudaStream_t)stream, &s);
    if (st != ZERO_OK) return st;
    s->fused = true;
    s->w_in = master_in;
    s->m_in = m_in;
    s->v_in = v_in;
    s->w_out = master_out;
    s->m_out = m_out;
    s->v_out = v_out;
    s->param_out = param_out;
    s->consts = d_consts;
    *out = s;
    return ZERO_OK;
}

zero_status zero_sched_rebind_fused(zero_sched* s, const float* master_in, const float* m_in,
                                    const float* v_in, float* master_out, float* m_out,
                                    float* v_out, uint16_t* param_out, uint32_t* d_status) {
    if (!s || !s->fused) return ZERO_EINVAL;
    for (int b : s->bucket_of_slot)
        if (b != -1) return ZERO_EINVAL;   // a bucket is between begin and end
    int nd = 0;
    uint64_t psi_p = 0, S = 0;
    zk::plan_geometry(s->plan, &nd, &psi_p, &S);
    zero_status st = zk::check_fused_state(psi_p, master_in, m_in, v_in, master_out, m_out, v_out,
                                           param_out, d_status);
    if (st != ZERO_OK) return st;
    const void* slots = nullptr;
    uint64_t slot_bytes = 0;
    slot_span(s, &slots, &slot_bytes);
    if (state_overlaps_slots(slots, slot_bytes, psi_p, master_out, m_out, v_out, param_out,
                             d_status))
        return ZERO_EINVAL;
    s->w_in = master_in;
    s->m_in = m_in;
    s->v_in = v_in;
    s->w_out = master_out;
    s->m_out = m_out;
    s->v_out = v_out;
    s->param_out = param_out;
    s->status = d_status;
    return ZERO_OK;
}

zero_status zero_sched_rebind_status(zero_sched* s, uint32_t* d_status) {
    if (!s || !d_status) return ZERO_EINVAL;
    if (reinterpret_cast<uintptr_t>(d_status) & 3u) return ZERO_EALIGN;
    for (int b : s->bucket_of_slot)
        if (b != -1) return ZERO_EINVAL;
    const void* slots = nullptr;
    uint64_t slot_bytes = 0;
    slot_span(s, &slots, &slot_bytes);
    if (overlaps(d_status, 4, slots, slot_bytes)) return ZERO_EINVAL;
    if (!s->fused) {
        int nd = 0;
        uint64_t psi_p = 0, S = 0;
        zk::plan_geometry(s->plan, &nd, &psi_p, &S);
        for (int r = 0; r < nd; ++r)
            if (overlaps(d_status, 4, s->shards[r], S * 4)) return ZERO_EINVAL;
    } else {
        int nd = 0;
        uint64_t psi_p = 0, S = 0;
        zk::plan_geometry(s->plan, &nd, &psi_p, &S);
        const void* arr[7] = {s->w_in, s->m_in, s->v_in, s->w_out, s->m_out, s->v_out,
                              s->param_out};
        for (int i = 0; i < 7; ++i)
            if (overlaps(d_status, 4, arr[i], psi_p * (i == 6 ? 2 : 4))) return ZERO_EINVAL;
    }
    s->status = d_status;
    return ZERO_OK;
}

zero_status zero_sched_begin_bucket(zero_sched* s, int k, zero_stream_t producer,
                                    uint16_t** rank_ptrs) {
    if (!s || !rank_ptrs || s->q8) return ZERO_EINVAL;
    int slot = 0;
    const zero_status st = begin_slot(s, k, producer, &slot);
    if (st != ZERO_OK) return st;
    for (int r = 0; r < s->nd; ++r)
        rank_ptrs[r] = s->slot_mem + ((uint64_t)slot * (uint64_t)s->nd + (uint64_t)r) * s->stride;
    return ZERO_OK;
}

zero_status zero_sched_begin_bucket_q8(zero_sched* s, int k, zero_stream_t producer,
                                       uint8_t** rank_ptrs) {
    if (!s || !rank_ptrs || !s->q8) return ZERO_EINVAL;
    int slot = 0;
    const zero_status st = begin_slot(s, k, producer, &slot);
    if (st != ZERO_OK) return st;
    for (int r = 0; r < s->nd; ++r)
        rank_ptrs[r] = s->slot_bytes + ((uint64_t)slot * (uint64_t)s->nd + (uint64_t)r) *
                                           s->region_bytes;
    return ZERO_OK;
}

zero_status zero_sched_end_bucket(zero_sched* s, int k, zero_stream_t producer) {
    uint64_t lo = 0, len = 0;
    if (!s || !zk::plan_bucket_range(s->plan, k, &lo, &len)) return ZERO_EINVAL;
    const int slot = k % s->n_slots;
    if (s->bucket_of_slot[(size_t)slot] != k) return ZERO_EINVAL;   // not begun
    const uint16_t* ptrs[ZERO_MAX_RANKS];
    const uint8_t* ptrs8[ZERO_MAX_RANKS];
    for (int r = 0; r < s->nd; ++r) {
        const uint64_t region = (uint64_t)slot * (uint64_t)s->nd + (uint64_t)r;
        if (s->q8)
            ptrs8[r] = s->slot_bytes + region * s->region_bytes;
        else
            ptrs[r] = s->slot_mem + region * s->stride;
    }
    cudaEvent_t prod = s->produced[(size_t)slot];
    if (cudaError_t e = cudaEventRecord(prod, (cudaStream_t)producer); e != cudaSuccess) return zk::from_cuda(e);
    if (cudaError_t e = cudaStreamWaitEvent(s->rs, prod, 0); e != cudaSuccess) return zk::from_cuda(e);
    cudaError_t e = cudaSuccess;
    if (s->q8) {
        zero_adam_consts unused;
        memset(&unused, 0, sizeof(unused));
        e = zk::launch_fused_q8(len, s->nd, ptrs8, s->w_in + lo, s->m_in + lo, s->v_in + lo,
                                s->w_out + lo, s->m_out + lo, s->v_out + lo, s->param_out + lo,
                                unused, s->consts, zk::make_mean(s->nd), s->status, s->rs);
    } else if (s->fused) {
        zero_adam_consts unused;
        memset(&unused, 0, sizeof(unused));
        e = zk::launch_fused(len, s->nd, ptrs, s->w_in + lo, s->m_in + lo, s->v_in + lo,
                             s->w_out + lo, s->m_out + lo, s->v_out + lo, s->param_out + lo, unused,
                             s->consts, zk::make_mean(s->nd), s->status, s->rs);
    } else {
        e = zk::rs_bucket_launch(s->plan, k, ptrs, s->shards, s->status, s->rs);
    }
    if (e != cudaSuccess) return zk::from_cuda(e);
    ++s->launches;
    // release: the slot may be refilled once this reduce-scatter is done with it
    if (cudaError_t e = cudaEventRecord(s->released[(size_t)slot], s->rs); e != cudaSuccess) return zk::from_cuda(e);
    s->filled[(size_t)slot] = 1;
    s->bucket_of_slot[(size_t)slot] = -1;
    return ZERO_OK;
}

zero_status zero_sched_wait(zero_sched* s, zero_stream_t stream) {
    if (!s) return ZERO_EINVAL;
    if (cudaError_t e = cudaEventRecord(s->tail, s->rs); e != cudaSuccess) return zk::from_cuda(e);
    if (cudaError_t e = cudaStreamWaitEvent((cudaStream_t)stream, s->tail, 0); e != cudaSuccess) return zk::from_cuda(e);
    return ZERO_OK;
}

zero_status zero_sched_launches(const zero_sched* s, uint64_t* count) {
    if (!s || !count) return ZERO_EINVAL;
    *count = s->launches;
    return ZERO_OK;
}

void zero_sched_destroy(zero_sched* s) {
    if (!s) return;
    destroy_events(s);
    delete s;
}

}  // extern "C"
