// Partition planner and model-state accounting of libzero (host only, no CUDA).
//
// Plan: "ZeRO: particionar estados do treino entre GPUs", section "Como funciona" (model states
// divided into Nd parts, each process updates its own); "ZeRO-2" card, sections
// "ZeRO-1에서 남은 낭비" (per-GPU local gradient [g_A, g_B, g_C]) and "Gradient 생명주기"
// (buckets handed over in backward order, each reduce-scattered at once).
// Accounting: "Como funciona" (2 + 2 + K bytes per parameter, K = 12; 4psi + 12psi/Nd for Pos,
// about 2psi for Pos+g, 16psi/Nd for Pos+g+p; 2psi vs 3psi of communication) and "ZeRO"
// (lastdictionary.com), main definition.
#include <cstdint>
#include <new>
#include <vector>

#include "../../include/libzero.h"
#include "zero_internal.h"

struct zero_plan {
    int nd = 0;
    int stage = 0;
    uint64_t psi = 0;        // parameters in the flat list
    uint64_t psi_p = 0;      // padded to a multiple of nd
    uint64_t shard = 0;      // psi_p / nd
    uint64_t bucket = 0;     // bucket length (psi_p when the caller asked for one bucket)
    uint64_t n_buckets = 0;
    std::vector<uint64_t> offsets;
};

namespace zk {

bool plan_geometry(const zero_plan* p, int* nd, uint64_t* psi_p, uint64_t* shard) {
    if (!p) return false;
    *nd = p->nd;
    *psi_p = p->psi_p;
    *shard = p->shard;
    return true;
}

// Bucket k counts down from the end of the flat buffer: [max(0, psi_p-(k+1)B), psi_p-kB).
bool plan_bucket_range(const zero_plan* p, int k, uint64_t* lo, uint64_t* len) {
    if (!p || k < 0 || (uint64_t)k >= p->n_buckets) return false;
    uint64_t top = p->psi_p - (uint64_t)k * p->bucket;
    uint64_t bottom = top > p->bucket ? top - p->bucket : 0;
    *lo = bottom;
    *len = top - bottom;
    return true;
}

uint64_t plan_max_bucket(const zero_plan* p) { return p ? (p->psi_p < p->bucket ? p->psi_p : p->bucket) : 0; }

uint64_t plan_n_buckets(const zero_plan* p) { return p ? p->n_buckets : 0; }

}  // namespace zk

extern "C" {

zero_status zero_plan_create(const uint64_t* numels, int n_tensors, int nd, int stage,
                             uint64_t bucket_elems, zero_plan** out) {
    if (!out) return ZERO_EINVAL;
    *out = nullptr;
    if (n_tensors < 0 || (n_tensors > 0 && !numels)) return ZERO_EINVAL;
    if (nd < 1 || nd > ZERO_MAX_RANKS) return ZERO_EINVAL;
    if (stage < 1 || stage > 3) return ZERO_EINVAL;
    zero_plan* p = new (std::nothrow) zero_plan();
    if (!p) return ZERO_ENOMEM;
    try {
        p->offsets.resize((size_t)n_tensors);
    } catch (...) {
        delete p;
        return ZERO_ENOMEM;
    }
    uint64_t run = 0;
    for (int i = 0; i < n_tensors; ++i) {
        p->offsets[(size_t)i] = run;
        if (numels[i] > UINT64_MAX / 4 - run) {  // keep every byte count below 2^64
            delete p;
            return ZERO_EINVAL;
        }
        run += numels[i];
    }
    if (run == 0) {
        delete p;
        return ZERO_EINVAL;
    }
    const uint64_t d = (uint64_t)nd;
    p->nd = nd;
    p->stage = stage;
    p->psi = run;
    p->shard = run / d + (run % d ? 1 : 0);
    p->psi_p = p->shard * d;
    p->bucket = (bucket_elems == 0 || bucket_elems > p->psi_p) ? p->psi_p : bucket_elems;
    p->n_buckets = p->psi_p / p->bucket + (p->psi_p % p->bucket ? 1 : 0);
    if (p->n_buckets > (uint64_t)INT32_MAX) {
        delete p;
        return ZERO_EINVAL;
    }
    *out = p;
    return ZERO_OK;
}

void zero_plan_destroy(zero_plan* plan) { delete plan; }

zero_status zero_plan_info(const zero_plan* plan, uint64_t* psi, uint64_t* psi_padded,
                           uint64_t* shard_elems, int* n_buckets) {
    if (!plan) return ZERO_EINVAL;
    if (psi) *psi = plan->psi;
    if (psi_padded) *psi_padded = plan->psi_p;
    if (shard_elems) *shard_elems = plan->shard;
    if (n_buckets) *n_buckets = (int)plan->n_buckets;
    return ZERO_OK;
}

zero_status zero_plan_tensor_offsets(const zero_plan* plan, uint64_t* out) {
    if (!plan || (!out && !plan->offsets.empty())) return ZERO_EINVAL;
    for (size_t i = 0; i < plan->offsets.size(); ++i) out[i] = plan->offsets[i];
    return ZERO_OK;
}

zero_status zero_plan_bucket(const zero_plan* plan, int k, uint64_t* flat_lo, uint64_t* len,
                             int* owner_lo, int* owner_hi) {
    uint64_t lo, ln;
    if (!zk::plan_bucket_range(plan, k, &lo, &ln)) return ZERO_EINVAL;
    if (flat_lo) *flat_lo = lo;
    if (len) *len = ln;
    if (owner_lo) *owner_lo = (int)(lo / plan->shard);
    if (owner_hi) *owner_hi = (int)((lo + ln - 1) / plan->shard);
    return ZERO_OK;
}

zero_status zero_state_bytes(uint64_t psi, int nd, int K, zero_state_report* out) {
    if (!out || nd < 1 || K < 0) return ZERO_EINVAL;
    const uint64_t k = (uint64_t)K;
    if (psi > UINT64_MAX / (k + 6)) return ZERO_EINVAL;   // every byte count fits in 64 bits
    const uint64_t part = psi / (uint64_t)nd + (psi % (uint64_t)nd ? 1 : 0);
    // {params, grads, optimizer} per stage: which of the three is partitioned
    const bool split[4][3] = {
        {false, false, false},   // plain DP: full replica
        {false, false, true},    // Pos
        {false, true, true},     // Pos+g
        {true, true, true},      // Pos+g+p
    };
    const uint64_t per_elem[3] = {2, 2, k};
    for (int s = 0; s < 4; ++s) {
        uint64_t b[3];
        for (int q = 0; q < 3; ++q) b[q] = per_elem[q] * (split[s][q] ? part : psi);
        out->stage[s].params = b[0];
        out->stage[s].grads = b[1];
        out->stage[s].optim = b[2];
        out->stage[s].total = b[0] + b[1] + b[2];
        // reduce-scatter + all-gather of psi each; Pos+g+p gathers parameters twice
        out->comm_elems[s] = (s == 3 ? 3 : 2) * psi;
        out->comm_bytes_fp16[s] = 2 * out->comm_elems[s];
    }
    return ZERO_OK;
}

}  // extern "C"
