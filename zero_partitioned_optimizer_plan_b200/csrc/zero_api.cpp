// C ABI of the libzero data path: argument checks, the host-side Adam constants, and the
// launches. Every function returns a zero_status and never throws.
#include <cmath>
#include <cstdint>
#include <cstdio>
#include <cstring>

#include <cuda_runtime.h>

#include "../../include/libzero.h"
#include "zero_internal.h"

namespace zk {

namespace {

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// Do the byte ranges [a, a+na) and [b, b+nb) intersect?
bool overlap(const void* a, uint64_t na, const void* b, uint64_t nb) {
    if (na == 0 || nb == 0) return false;
    const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
    return x < y + nb && y < x + na;
}

bool finite(double x) { return std::isfinite(x); }

// 2^k with 1/2^k a normal binary32 number: then x * (1/2^k) rounds exactly like x / 2^k.
bool pow2_with_normal_reciprocal(double x, float* inv) {
    if (!(x > 0.0) || !finite(x)) return false;
    int e = 0;
    const double mant = std::frexp(x, &e);   // x = mant * 2^e, mant in [0.5, 1)
    if (mant != 0.5) return false;
    const int k = e - 1;                     // x = 2^k
    if (k < -126 || k > 126) return false;
    *inv = (float)std::ldexp(1.0, -k);
    return true;
}

bool hparams_ok(const zero_adam_hparams* hp) {
    return hp && finite(hp->lr) && hp->beta1 >= 0.0 && hp->beta1 < 1.0 && hp->beta2 >= 0.0 &&
           hp->beta2 < 1.0 && finite(hp->eps) && hp->eps >= 0.0 && finite(hp->loss_scale) &&
           hp->loss_scale > 0.0;
}

// The fp32 constants of step t: computed in double, each rounded once to binary32.
AdamConsts make_adam(const zero_adam_hparams* hp, int64_t t) {
    AdamConsts a;
    const double c1 = 1.0 - std::pow(hp->beta1, (double)t);
    const double c2 = 1.0 - std::pow(hp->beta2, (double)t);
    a.beta1 = (float)hp->beta1;
    a.one_minus_beta1 = (float)(1.0 - hp->beta1);
    a.beta2 = (float)hp->beta2;
    a.one_minus_beta2 = (float)(1.0 - hp->beta2);
    a.step_size = (float)(hp->lr / c1);
    a.bias2_sqrt = (float)std::sqrt(c2);
    a.eps = (float)hp->eps;
    a.loss_scale = (float)hp->loss_scale;
    a.inv_loss_scale = 0.0f;
    a.loss_scale_pow2 =
        pow2_with_normal_reciprocal((double)a.loss_scale, &a.inv_loss_scale) ? 1 : 0;
    return a;
}

}  // namespace

// The last CUDA failure seen by a libzero call on this host thread.
thread_local char g_last_error[256] = "";

zero_status from_cuda(cudaError_t e) {
    if (e == cudaSuccess) return ZERO_OK;
    snprintf(g_last_error, sizeof(g_last_error), "%s: %s", cudaGetErrorName(e),
             cudaGetErrorString(e));
    return ZERO_ECUDA;
}

MeanConsts make_mean(int nd) {
    MeanConsts mc;
    mc.fnd = (float)nd;
    mc.nd_pow2 = (nd & (nd - 1)) == 0 ? 1 : 0;
    mc.inv_nd = 1.0f / (float)nd;   // exact when nd is a power of two
    return mc;
}

cudaError_t rs_bucket_launch(const zero_plan* plan, int k, const uint16_t* const* rank_grads,
                             float* const* shards, uint32_t* status, cudaStream_t stream) {
    int nd = 0;
    uint64_t psi_p = 0, S = 0, lo = 0, len = 0;
    plan_geometry(plan, &nd, &psi_p, &S);
    plan_bucket_range(plan, k, &lo, &len);
    return launch_reduce_scatter(len, nd, rank_grads, shards, lo, S, make_mean(nd), status, stream);
}

zero_status check_fused_state(uint64_t n, const float* master_in, const float* m_in,
                              const float* v_in, float* master_out, float* m_out,
                              float* v_out, uint16_t* param_out, uint32_t* d_status) {
    if (!master_in || !m_in || !v_in || !master_out || !m_out || !v_out || !param_out ||
        !d_status)
        return ZERO_EINVAL;
    if (n > (UINT64_MAX / 8)) return ZERO_EINVAL;
    if (!zk::aligned(master_in, 4) || !zk::aligned(m_in, 4) || !zk::aligned(v_in, 4) ||
        !zk::aligned(master_out, 4) || !zk::aligned(m_out, 4) || !zk::aligned(v_out, 4) ||
        !zk::aligned(param_out, 2) || !zk::aligned(d_status, 4))
        return ZERO_EALIGN;
    const void* outs[5] = {master_out, m_out, v_out, param_out, d_status};
    const uint64_t olen[5] = {n * 4, n * 4, n * 4, n * 2, 4};
    const void* ins[3] = {master_in, m_in, v_in};
    for (int i = 0; i < 5; ++i) {
        for (int j = 0; j < 3; ++j)
            if (zk::overlap(outs[i], olen[i], ins[j], n * 4)) return ZERO_EINVAL;
        for (int j = i + 1; j < 5; ++j)
            if (zk::overlap(outs[i], olen[i], outs[j], olen[j])) return ZERO_EINVAL;
    }
    return ZERO_OK;
}

}  // namespace zk

extern "C" {

const char* zero_status_string(zero_status s) {
    switch (s) {
        case ZERO_OK: return "ZERO_OK";
        case ZERO_EINVAL: return "ZERO_EINVAL: invalid argument";
        case ZERO_EALIGN: return "ZERO_EALIGN: pointer not aligned to its element size";
        case ZERO_ECUDA: return "ZERO_ECUDA: CUDA error";
        case ZERO_ENOMEM: return "ZERO_ENOMEM: out of memory or buffer too small";
        case ZERO_STEP_SKIPPED: return "ZERO_STEP_SKIPPED: step skipped on gradient overflow";
    }
    return "unknown zero_status";
}

uint64_t zero_kernel_launches(void) { return zk::launches(); }

const char* zero_last_error(void) { return zk::g_last_error; }

zero_status zero_selftest_timeout(uint32_t* d_status, zero_stream_t stream) {
    if (!d_status) return ZERO_EINVAL;
    if (!zk::aligned(d_status, 4)) return ZERO_EALIGN;
    return zk::from_cuda(zk::launch_selftest_timeout(d_status, (cudaStream_t)stream));
}

zero_status zero_reduce_scatter_bucket(const zero_plan* plan, int k,
                                       const uint16_t* const* rank_grads,
                                       float* const* owner_grad_shards, uint32_t* d_status,
                                       zero_stream_t stream) {
    int nd = 0;
    uint64_t psi_p = 0, S = 0, lo = 0, len = 0;
    if (!zk::plan_geometry(plan, &nd, &psi_p, &S)) return ZERO_EINVAL;
    if (!zk::plan_bucket_range(plan, k, &lo, &len)) return ZERO_EINVAL;
    if (!rank_grads || !owner_grad_shards || !d_status) return ZERO_EINVAL;
    if (!zk::aligned(d_status, 4)) return ZERO_EALIGN;
    for (int r = 0; r < nd; ++r) {
        if (!rank_grads[r] || !owner_grad_shards[r]) return ZERO_EINVAL;
        if (!zk::aligned(rank_grads[r], 2) || !zk::aligned(owner_grad_shards[r], 4))
            return ZERO_EALIGN;
    }
    // outputs may not overlap inputs, each other or the status word
    for (int o = 0; o < nd; ++o) {
        if (zk::overlap(owner_grad_shards[o], S * 4, d_status, 4)) return ZERO_EINVAL;
        for (int r = 0; r < nd; ++r) {
            if (zk::overlap(owner_grad_shards[o], S * 4, rank_grads[r], len * 2)) return ZERO_EINVAL;
            if (r != o && zk::overlap(owner_grad_shards[o], S * 4, owner_grad_shards[r], S * 4))
                return ZERO_EINVAL;
        }
    }
    return zk::from_cuda(zk::rs_bucket_launch(plan, k, rank_grads, owner_grad_shards, d_status,
                                              (cudaStream_t)stream));
}

static zero_status check_adam(uint64_t n, const float* grad, float* master, float* m, float* v,
                              uint16_t* param_out, uint32_t* d_status) {
    if (!d_status) return ZERO_EINVAL;
    if (n == 0) return ZERO_OK;
    if (!grad || !master || !m || !v || !param_out) return ZERO_EINVAL;
    if (n > (UINT64_MAX / 8)) return ZERO_EINVAL;
    if (!zk::aligned(grad, 4) || !zk::aligned(master, 4) || !zk::aligned(m, 4) ||
        !zk::aligned(v, 4) || !zk::aligned(param_out, 2) || !zk::aligned(d_status, 4))
        return ZERO_EALIGN;
    const void* arr[6] = {grad, master, m, v, param_out, d_status};
    const uint64_t len[6] = {n * 4, n * 4, n * 4, n * 4, n * 2, 4};
    for (int i = 0; i < 6; ++i)
        for (int j = i + 1; j < 6; ++j)
            if (zk::overlap(arr[i], len[i], arr[j], len[j])) return ZERO_EINVAL;
    return ZERO_OK;
}

zero_status zero_adam_consts_for_step(const zero_adam_hparams* hp, int64_t step,
                                      zero_adam_consts* out) {
    if (!zk::hparams_ok(hp) || step < 1 || !out) return ZERO_EINVAL;
    *out = zk::make_adam(hp, step);
    return ZERO_OK;
}

zero_status zero_adam_consts_table(const zero_adam_hparams* hp, int64_t first_step, int64_t count,
                                   zero_adam_consts* out) {
    if (!zk::hparams_ok(hp) || first_step < 1 || count < 0 || (count > 0 && !out))
        return ZERO_EINVAL;
    if (count > 0 && first_step > INT64_MAX - count) return ZERO_EINVAL;
    for (int64_t i = 0; i < count; ++i) out[i] = zk::make_adam(hp, first_step + i);
    return ZERO_OK;
}

zero_status zero_scaler_prepare(const zero_scaler_state* d_state, const zero_adam_consts* d_table,
                                int64_t table_len, zero_adam_consts* d_consts, uint32_t* d_status,
                                zero_stream_t stream) {
    if (!d_state || !d_table || !d_consts || !d_status || table_len < 1) return ZERO_EINVAL;
    if (!zk::aligned(d_state, 8) || !zk::aligned(d_table, 4) || !zk::aligned(d_consts, 4) ||
        !zk::aligned(d_status, 4))
        return ZERO_EALIGN;
    if (zk::overlap(d_consts, sizeof(zero_adam_consts), d_table,
                    (uint64_t)table_len * sizeof(zero_adam_consts)) ||
        zk::overlap(d_consts, sizeof(zero_adam_consts), d_status, 4) ||
        zk::overlap(d_consts, sizeof(zero_adam_consts), d_state, sizeof(zero_scaler_state)))
        return ZERO_EINVAL;
    return zk::from_cuda(zk::launch_scaler_prepare(d_state, d_table, table_len, d_consts,
                                                   d_status, (cudaStream_t)stream));
}

zero_status zero_scaler_update(zero_scaler_state* d_state, const zero_scaler_params* params,
                               const uint32_t* d_status, zero_stream_t stream) {
    if (!d_state || !params || !d_status || params->growth_interval < 1) return ZERO_EINVAL;
    if (!zk::finite(params->growth_factor) || !(params->growth_factor > 0.0f) ||
        !zk::finite(params->backoff_factor) || !(params->backoff_factor > 0.0f))
        return ZERO_EINVAL;
    if (!zk::aligned(d_state, 8) || !zk::aligned(d_status, 4)) return ZERO_EALIGN;
    return zk::from_cuda(zk::launch_scaler_update(d_state, *params, d_status,
                                                  (cudaStream_t)stream));
}

zero_status zero_adam_shard(uint64_t n, const float* grad, float* master, float* m, float* v,
                            uint16_t* param_out, const zero_adam_hparams* hp, int64_t step,
                            uint32_t* d_status, zero_stream_t stream) {
    if (!zk::hparams_ok(hp) || step < 1) return ZERO_EINVAL;
    const zero_status st = check_adam(n, grad, master, m, v, param_out, d_status);
    if (st != ZERO_OK || n == 0) return st;
    return zk::from_cuda(zk::launch_adam(n, grad, master, m, v, param_out,
                                         zk::make_adam(hp, step), nullptr, d_status,
                                         (cudaStream_t)stream));
}

zero_status zero_adam_shard_dc(uint64_t n, const float* grad, float* master, float* m, float* v,
                               uint16_t* param_out, const zero_adam_consts* d_consts,
                               uint32_t* d_status, zero_stream_t stream) {
    if (!d_consts) return ZERO_EINVAL;
    if (!zk::aligned(d_consts, 4)) return ZERO_EALIGN;
    const zero_status st = check_adam(n, grad, master, m, v, param_out, d_status);
    if (st != ZERO_OK || n == 0) return st;
    zero_adam_consts unused;
    memset(&unused, 0, sizeof(unused));
    return zk::from_cuda(zk::launch_adam(n, grad, master, m, v, param_out, unused, d_consts,
                                         d_status, (cudaStream_t)stream));
}


static zero_status check_fused(uint64_t n, int nd, const uint16_t* const* rank_grads,
                               const float* master_in, const float* m_in, const float* v_in,
                               float* master_out, float* m_out, float* v_out,
                               uint16_t* param_out, uint32_t* d_status) {
    if (nd < 1 || nd > ZERO_MAX_RANKS || !d_status) return ZERO_EINVAL;
    if (n == 0) return ZERO_OK;
    if (!rank_grads) return ZERO_EINVAL;
    zero_status st = zk::check_fused_state(n, master_in, m_in, v_in, master_out, m_out, v_out,
                                           param_out, d_status);
    if (st != ZERO_OK) return st;
    const void* outs[5] = {master_out, m_out, v_out, param_out, d_status};
    const uint64_t olen[5] = {n * 4, n * 4, n * 4, n * 2, 4};
    for (int r = 0; r < nd; ++r) {
        if (!rank_grads[r]) return ZERO_EINVAL;
        if (!zk::aligned(rank_grads[r], 2)) return ZERO_EALIGN;
        for (int i = 0; i < 5; ++i)
            if (zk::overlap(outs[i], olen[i], rank_grads[r], n * 2)) return ZERO_EINVAL;
    }
    return ZERO_OK;
}

// The replica list of the epilogue all-gather: 1..ZERO_MAX_RANKS distinct ranges, each
// checked like a param_out against the step's other buffers (rank_grads may be null: commit).
static zero_status check_replicas(uint64_t n, int nd, const uint16_t* const* rank_grads,
                                  const float* master_in, const float* m_in, const float* v_in,
                                  float* master_out, float* m_out, float* v_out, int n_replicas,
                                  uint16_t* const* replicas, uint32_t* d_status) {
    if (n_replicas < 1 || n_replicas > ZERO_MAX_RANKS || !replicas || !d_status)
        return ZERO_EINVAL;
    if (n == 0) return ZERO_OK;
    for (int d = 0; d < n_replicas; ++d) {
        const zero_status st =
            rank_grads ? check_fused(n, nd, rank_grads, master_in, m_in, v_in, master_out, m_out,
                                     v_out, replicas[d], d_status)
                       : zk::check_fused_state(n, master_in, m_in, v_in, master_out, m_out,
                                               v_out, replicas[d], d_status);
        if (st != ZERO_OK) return st;
        for (int e = 0; e < d; ++e)
            if (zk::overlap(replicas[e], n * 2, replicas[d], n * 2)) return ZERO_EINVAL;
    }
    return ZERO_OK;
}

zero_status zero_step_fused_replicas(uint64_t n, int nd, const uint16_t* const* rank_grads,
                                     const float* master_in, const float* m_in, const float* v_in,
                                     float* master_out, float* m_out, float* v_out,
                                     int n_replicas, uint16_t* const* param_replicas,
                                     const zero_adam_hparams* hp, int64_t step,
                                     uint32_t* d_status, zero_stream_t stream) {
    if (!zk::hparams_ok(hp) || step < 1 || nd < 1 || nd > ZERO_MAX_RANKS) return ZERO_EINVAL;
    if (n > 0 && !rank_grads) return ZERO_EINVAL;
    const zero_status st = check_replicas(n, nd, rank_grads, master_in, m_in, v_in,
                                          master_out, m_out, v_out, n_replicas, param_replicas,
                                          d_status);
    if (st != ZERO_OK || n == 0) return st;
    return zk::from_cuda(zk::launch_fused(n, nd, rank_grads, master_in, m_in, v_in, master_out,
                                          m_out, v_out, param_replicas[0],
                                          zk::make_adam(hp, step), nullptr, zk::make_mean(nd),
                                          d_status, (cudaStream_t)stream, n_replicas,
                                          param_replicas));
}

zero_status zero_step_commit_replicas(uint64_t n, const float* master_in, const float* m_in,
                                      const float* v_in, float* master_out, float* m_out,
                                      float* v_out, int n_replicas,
                                      uint16_t* const* param_replicas, uint32_t* d_status,
                                      zero_stream_t stream) {
    const zero_status st = check_replicas(n, 1, nullptr, master_in, m_in, v_in, master_out, m_out,
                                          v_out, n_replicas, param_replicas, d_status);
    if (st != ZERO_OK || n == 0) return st;
    return zk::from_cuda(zk::launch_commit(n, master_in, m_in, v_in, master_out, m_out, v_out,
                                           param_replicas[0], d_status, (cudaStream_t)stream,
                                           n_replicas, param_replicas));
}

zero_status zero_step_fused(uint64_t n, int nd, const uint16_t* const* rank_grads,
                            const float* master_in, const float* m_in, const float* v_in,
                            float* master_out, float* m_out, float* v_out, uint16_t* param_out,
                            const zero_adam_hparams* hp, int64_t step, uint32_t* d_status,
                            zero_stream_t stream) {
    if (!zk::hparams_ok(hp) || step < 1) return ZERO_EINVAL;
    const zero_status st = check_fused(n, nd, rank_grads, master_in, m_in, v_in, master_out,
                                       m_out, v_out, param_out, d_status);
    if (st != ZERO_OK || n == 0) return st;
    return zk::from_cuda(zk::launch_fused(n, nd, rank_grads, master_in, m_in, v_in, master_out,
                                          m_out, v_out, param_out, zk::make_adam(hp, step),
                                          nullptr, zk::make_mean(nd), d_status,
                                          (cudaStream_t)stream));
}

zero_status zero_step_fused_ranges(int nd, int count, const zero_fused_range* ranges,
                                   const zero_adam_hparams* hp, int64_t step, uint32_t* d_status,
                                   int overlap, zero_stream_t stream) {
    if (!zk::hparams_ok(hp) || step < 1 || count < 0 || (count > 0 && !ranges)) return ZERO_EINVAL;
    for (int i = 0; i < count; ++i) {
        const zero_fused_range& r = ranges[i];
        const zero_status st = check_fused(r.n, nd, r.rank_grads, r.master_in, r.m_in, r.v_in,
                                           r.master_out, r.m_out, r.v_out, r.param_out, d_status);
        if (st != ZERO_OK) return st;
    }
    if (!d_status) return ZERO_EINVAL;
    const zk::AdamConsts a = zk::make_adam(hp, step);
    const zk::MeanConsts mc = zk::make_mean(nd);
    const cudaStream_t s = (cudaStream_t)stream;
    // a region already open on the stream (the caller's) chains these calls as well
    const bool opened = overlap && zero_overlap_begin(stream) == ZERO_OK;
    cudaError_t e = cudaSuccess;
    for (int i = 0; i < count && e == cudaSuccess; ++i) {
        const zero_fused_range& r = ranges[i];
        if (r.n == 0) continue;
        e = zk::launch_fused(r.n, nd, r.rank_grads, r.master_in, r.m_in, r.v_in, r.master_out,
                             r.m_out, r.v_out, r.param_out, a, nullptr, mc, d_status, s);
    }
    if (opened) zero_overlap_end(stream);
    return zk::from_cuda(e);
}

zero_status zero_step_fused_dc(uint64_t n, int nd, const uint16_t* const* rank_grads,
                               const float* master_in, const float* m_in, const float* v_in,
                               float* master_out, float* m_out, float* v_out,
                               uint16_t* param_out, const zero_adam_consts* d_consts,
                               uint32_t* d_status, zero_stream_t stream) {
    if (!d_consts) return ZERO_EINVAL;
    if (!zk::aligned(d_consts, 4)) return ZERO_EALIGN;
    const zero_status st = check_fused(n, nd, rank_grads, master_in, m_in, v_in, master_out,
                                       m_out, v_out, param_out, d_status);
    if (st != ZERO_OK || n == 0) return st;
    zero_adam_consts unused;
    memset(&unused, 0, sizeof(unused));
    return zk::from_cuda(zk::launch_fused(n, nd, rank_grads, master_in, m_in, v_in, master_out,
                                          m_out, v_out, param_out, unused, d_consts,
                                          zk::make_mean(nd), d_status, (cudaStream_t)stream));
}

zero_status zero_quantize_q8(uint64_t n, const uint16_t* grad, uint8_t* payload,
                             zero_stream_t stream) {
    if (n == 0) return ZERO_OK;
    if (!grad || !payload || n > (UINT64_MAX / 8)) return ZERO_EINVAL;
    if (!zk::aligned(grad, 2) || !zk::aligned(payload, 4)) return ZERO_EALIGN;
    if (zk::overlap(payload, ZERO_Q8_PAYLOAD_BYTES(n), grad, n * 2)) return ZERO_EINVAL;
    return zk::from_cuda(zk::launch_quant_q8(n, grad, payload, (cudaStream_t)stream));
}

static zero_status check_fused_q8(uint64_t n, int nd, const uint8_t* const* rank_payload,
                                  const float* master_in, const float* m_in, const float* v_in,
                                  float* master_out, float* m_out, float* v_out,
                                  uint16_t* param_out, uint32_t* d_status) {
    if (nd < 1 || nd > ZERO_MAX_RANKS || !d_status) return ZERO_EINVAL;
    if (n == 0) return ZERO_OK;
    if (!rank_payload) return ZERO_EINVAL;
    zero_status st = zk::check_fused_state(n, master_in, m_in, v_in, master_out, m_out, v_out,
                                           param_out, d_status);
    if (st != ZERO_OK) return st;
    const uint64_t pb = ZERO_Q8_PAYLOAD_BYTES(n);
    const void* outs[5] = {master_out, m_out, v_out, param_out, d_status};
    const uint64_t olen[5] = {n * 4, n * 4, n * 4, n * 2, 4};
    for (int r = 0; r < nd; ++r) {
        if (!rank_payload[r]) return ZERO_EINVAL;
        if (!zk::aligned(rank_payload[r], 4)) return ZERO_EALIGN;
        for (int i = 0; i < 5; ++i)
            if (zk::overlap(outs[i], olen[i], rank_payload[r], pb)) return ZERO_EINVAL;
    }
    return ZERO_OK;
}

zero_status zero_step_fused_q8(uint64_t n, int nd, const uint8_t* const* rank_payload,
                               const float* master_in, const float* m_in, const float* v_in,
                               float* master_out, float* m_out, float* v_out,
                               uint16_t* param_out, const zero_adam_hparams* hp, int64_t step,
                               uint32_t* d_status, zero_stream_t stream) {
    if (!zk::hparams_ok(hp) || step < 1) return ZERO_EINVAL;
    const zero_status st = check_fused_q8(n, nd, rank_payload, master_in, m_in, v_in, master_out,
                                          m_out, v_out, param_out, d_status);
    if (st != ZERO_OK || n == 0) return st;
    return zk::from_cuda(zk::launch_fused_q8(n, nd, rank_payload, master_in, m_in, v_in,
                                             master_out, m_out, v_out, param_out,
                                             zk::make_adam(hp, step), nullptr, zk::make_mean(nd),
                                             d_status, (cudaStream_t)stream));
}

zero_status zero_step_fused_q8_ranges(int nd, int count, const zero_fused_q8_range* ranges,
                                      const zero_adam_hparams* hp, int64_t step,
                                      uint32_t* d_status, int overlap, zero_stream_t stream) {
    if (!zk::hparams_ok(hp) || step < 1 || count < 0 || (count > 0 && !ranges)) return ZERO_EINVAL;
    for (int i = 0; i < count; ++i) {
        const zero_fused_q8_range& r = ranges[i];
        const zero_status st = check_fused_q8(r.n, nd, r.rank_payload, r.master_in, r.m_in,
                                              r.v_in, r.master_out, r.m_out, r.v_out,
                                              r.param_out, d_status);
        if (st != ZERO_OK) return st;
    }
    if (!d_status) return ZERO_EINVAL;
    const zk::AdamConsts a = zk::make_adam(hp, step);
    const zk::MeanConsts mc = zk::make_mean(nd);
    const cudaStream_t s = (cudaStream_t)stream;
    // a region already open on the stream (the caller's) chains these calls as well
    const bool opened = overlap && zero_overlap_begin(stream) == ZERO_OK;
    cudaError_t e = cudaSuccess;
    for (int i = 0; i < count && e == cudaSuccess; ++i) {
        const zero_fused_q8_range& r = ranges[i];
        if (r.n == 0) continue;
        e = zk::launch_fused_q8(r.n, nd, r.rank_payload, r.master_in, r.m_in, r.v_in,
                                r.master_out, r.m_out, r.v_out, r.param_out, a, nullptr, mc,
                                d_status, s);
    }
    if (opened) zero_overlap_end(stream);
    return zk::from_cuda(e);
}

zero_status zero_step_fused_q8_dc(uint64_t n, int nd, const uint8_t* const* rank_payload,
                                  const float* master_in, const float* m_in, const float* v_in,
                                  float* master_out, float* m_out, float* v_out,
                                  uint16_t* param_out, const zero_adam_consts* d_consts,
                                  uint32_t* d_status, zero_stream_t stream) {
    if (!d_consts) return ZERO_EINVAL;
    if (!zk::aligned(d_consts, 4)) return ZERO_EALIGN;
    const zero_status st = check_fused_q8(n, nd, rank_payload, master_in, m_in, v_in, master_out,
                                          m_out, v_out, param_out, d_status);
    if (st != ZERO_OK || n == 0) return st;
    zero_adam_consts unused;
    memset(&unused, 0, sizeof(unused));
    return zk::from_cuda(zk::launch_fused_q8(n, nd, rank_payload, master_in, m_in, v_in,
                                             master_out, m_out, v_out, param_out, unused,
                                             d_consts, zk::make_mean(nd), d_status,
                                             (cudaStream_t)stream));
}

zero_status zero_step_commit(uint64_t n, const float* master_in, const float* m_in,
                             const float* v_in, float* master_out, float* m_out, float* v_out,
                             uint16_t* param_out, uint32_t* d_status, zero_stream_t stream) {
    if (!d_status) return ZERO_EINVAL;
    if (n == 0) return ZERO_OK;
    zero_status st = zk::check_fused_state(n, master_in, m_in, v_in, master_out, m_out, v_out,
                                           param_out, d_status);
    if (st != ZERO_OK) return st;
    return zk::from_cuda(zk::launch_commit(n, master_in, m_in, v_in, master_out, m_out, v_out,
                                           param_out, d_status, (cudaStream_t)stream));
}

// ---------------------------------------------------------------------------------------------
// stage 3: parameters partitioned, gathered per layer
// ---------------------------------------------------------------------------------------------
// The owners whose partitions meet [flat_lo, flat_lo + len), and that range against the plan.
static zero_status stage3_range(const zero_plan* plan, uint64_t flat_lo, uint64_t len, int* nd,
                                uint64_t* psi_p, uint64_t* S, uint64_t* q_lo, uint64_t* q_hi) {
    if (!zk::plan_geometry(plan, nd, psi_p, S)) return ZERO_EINVAL;
    if (flat_lo > *psi_p || len > *psi_p - flat_lo) return ZERO_EINVAL;
    if (len) {
        *q_lo = flat_lo / *S;
        *q_hi = (flat_lo + len - 1) / *S;
    }
    return ZERO_OK;
}

zero_status zero_gather_params(const zero_plan* plan, uint64_t flat_lo, uint64_t len,
                               const uint16_t* const* param_shards, uint16_t* out,
                               uint32_t* d_status, zero_stream_t stream) {
    int nd = 0;
    uint64_t psi_p = 0, S = 0, q_lo = 0, q_hi = 0;
    zero_status st = stage3_range(plan, flat_lo, len, &nd, &psi_p, &S, &q_lo, &q_hi);
    if (st != ZERO_OK) return st;
    if (!d_status) return ZERO_EINVAL;
    if (!zk::aligned(d_status, 4)) return ZERO_EALIGN;
    if (len == 0) return ZERO_OK;
    if (!param_shards || !out) return ZERO_EINVAL;
    if (!zk::aligned(out, 2)) return ZERO_EALIGN;
    if (zk::overlap(out, len * 2, d_status, 4)) return ZERO_EINVAL;
    for (uint64_t q = q_lo; q <= q_hi; ++q) {
        const uint16_t* sh = param_shards[q];
        if (!sh) return ZERO_EINVAL;
        if (!zk::aligned(sh, 2)) return ZERO_EALIGN;
        if (zk::overlap(out, len * 2, sh, S * 2) || zk::overlap(d_status, 4, sh, S * 2))
            return ZERO_EINVAL;
    }
    return zk::from_cuda(zk::launch_gather(flat_lo, len, S, nd, param_shards, out, d_status,
                                           (cudaStream_t)stream));
}

}  // extern "C"

namespace {

// The owners' update of a stage-3 range with the step's constants `a` (by value) or, when `ad`
// is not null, read from device memory; every part is checked before any is launched.
zero_status stage3_fused(const zero_plan* plan, uint64_t flat_lo, uint64_t len,
                         const uint16_t* const* rank_grads, const float* master_in,
                         const float* m_in, const float* v_in, float* master_out, float* m_out,
                         float* v_out, uint16_t* const* param_shards, const zk::AdamConsts& a,
                         const zk::AdamConsts* ad, uint32_t* d_status, cudaStream_t stream) {
    int nd = 0;
    uint64_t psi_p = 0, S = 0, q_lo = 0, q_hi = 0;
    zero_status st = stage3_range(plan, flat_lo, len, &nd, &psi_p, &S, &q_lo, &q_hi);
    if (st != ZERO_OK) return st;
    if (!d_status) return ZERO_EINVAL;
    if (len == 0) return ZERO_OK;
    if (!rank_grads || !param_shards || !master_in || !m_in || !v_in || !master_out || !m_out ||
        !v_out)
        return ZERO_EINVAL;
    const uint16_t* part_grads[ZERO_MAX_RANKS];
    for (int pass = 0; pass < 2; ++pass) {
        for (uint64_t q = q_lo; q <= q_hi; ++q) {
            const uint64_t lo = flat_lo > q * S ? flat_lo : q * S;
            const uint64_t hi = (q + 1) * S < flat_lo + len ? (q + 1) * S : flat_lo + len;
            const uint64_t off = lo - flat_lo, n = hi - lo;
            for (int r = 0; r < nd; ++r) part_grads[r] = rank_grads[r] ? rank_grads[r] + off : nullptr;
            uint16_t* pout = param_shards[q] ? param_shards[q] + (lo - q * S) : nullptr;
            if (pass == 0) {
                st = check_fused(n, nd, part_grads, master_in + off, m_in + off, v_in + off,
                                 master_out + off, m_out + off, v_out + off, pout, d_status);
                if (st != ZERO_OK) return st;
                for (uint64_t o = q_lo; o < q; ++o)   // partitions are distinct buffers
                    if (param_shards[o] &&
                        zk::overlap(param_shards[o], S * 2, param_shards[q], S * 2))
                        return ZERO_EINVAL;
            } else {
                const cudaError_t e = zk::launch_fused(
                    n, nd, part_grads, master_in + off, m_in + off, v_in + off, master_out + off,
                    m_out + off, v_out + off, pout, a, ad, zk::make_mean(nd), d_status, stream);
                if (e != cudaSuccess) return zk::from_cuda(e);
            }
        }
    }
    return ZERO_OK;
}

}  // namespace

extern "C" {

zero_status zero_stage3_step_fused(const zero_plan* plan, uint64_t flat_lo, uint64_t len,
                             const uint16_t* const* rank_grads, const float* master_in,
                             const float* m_in, const float* v_in, float* master_out,
                             float* m_out, float* v_out, uint16_t* const* param_shards,
                             const zero_adam_hparams* hp, int64_t step, uint32_t* d_status,
                             zero_stream_t stream) {
    if (!zk::hparams_ok(hp) || step < 1) return ZERO_EINVAL;
    return stage3_fused(plan, flat_lo, len, rank_grads, master_in, m_in, v_in, master_out, m_out,
                        v_out, param_shards, zk::make_adam(hp, step), nullptr, d_status,
                        (cudaStream_t)stream);
}

zero_status zero_stage3_step_fused_dc(const zero_plan* plan, uint64_t flat_lo, uint64_t len,
                                      const uint16_t* const* rank_grads, const float* master_in,
                                      const float* m_in, const float* v_in, float* master_out,
                                      float* m_out, float* v_out, uint16_t* const* param_shards,
                                      const zero_adam_consts* d_consts, uint32_t* d_status,
                                      zero_stream_t stream) {
    if (!d_consts) return ZERO_EINVAL;
    if (!zk::aligned(d_consts, 4)) return ZERO_EALIGN;
    zero_adam_consts unused;
    memset(&unused, 0, sizeof(unused));
    return stage3_fused(plan, flat_lo, len, rank_grads, master_in, m_in, v_in, master_out, m_out,
                        v_out, param_shards, unused, d_consts, d_status, (cudaStream_t)stream);
}

// The int8 payload of a stage-3 range: one segment per owner part of the range, the part's
// records counted from its first element, each segment rounded up to 16 bytes.
static uint64_t q8_segment_bytes(uint64_t n) {
    return (ZERO_Q8_PAYLOAD_BYTES(n) + 15) & ~(uint64_t)15;
}

zero_status zero_stage3_payload_bytes_q8(const zero_plan* plan, uint64_t flat_lo, uint64_t len,
                                         uint64_t* bytes) {
    int nd = 0;
    uint64_t psi_p = 0, S = 0, q_lo = 0, q_hi = 0;
    if (!bytes) return ZERO_EINVAL;
    const zero_status st = stage3_range(plan, flat_lo, len, &nd, &psi_p, &S, &q_lo, &q_hi);
    if (st != ZERO_OK) return st;
    uint64_t total = 0;
    for (uint64_t q = q_lo; len > 0 && q <= q_hi; ++q) {
        const uint64_t lo = flat_lo > q * S ? flat_lo : q * S;
        const uint64_t hi = (q + 1) * S < flat_lo + len ? (q + 1) * S : flat_lo + len;
        total += q8_segment_bytes(hi - lo);
    }
    *bytes = total;
    return ZERO_OK;
}

zero_status zero_stage3_quantize_q8(const zero_plan* plan, uint64_t flat_lo, uint64_t len,
                                    const uint16_t* grad, uint8_t* payload,
                                    zero_stream_t stream) {
    int nd = 0;
    uint64_t psi_p = 0, S = 0, q_lo = 0, q_hi = 0;
    zero_status st = stage3_range(plan, flat_lo, len, &nd, &psi_p, &S, &q_lo, &q_hi);
    if (st != ZERO_OK) return st;
    if (len == 0) return ZERO_OK;
    if (!grad || !payload) return ZERO_EINVAL;
    if (!zk::aligned(grad, 2) || !zk::aligned(payload, 16)) return ZERO_EALIGN;
    uint64_t bytes = 0;
    zero_stage3_payload_bytes_q8(plan, flat_lo, len, &bytes);
    if (zk::overlap(payload, bytes, grad, len * 2)) return ZERO_EINVAL;
    uint64_t seg = 0;
    for (uint64_t q = q_lo; q <= q_hi; ++q) {
        const uint64_t lo = flat_lo > q * S ? flat_lo : q * S;
        const uint64_t hi = (q + 1) * S < flat_lo + len ? (q + 1) * S : flat_lo + len;
        const cudaError_t e = zk::launch_quant_q8(hi - lo, grad + (lo - flat_lo), payload + seg,
                                                  (cudaStream_t)stream);
        if (e != cudaSuccess) return zk::from_cuda(e);
        seg += q8_segment_bytes(hi - lo);
    }
    return ZERO_OK;
}

// The owners' int8 update of a stage-3 range with the constants `a` or, when `ad` is not
// null, from device memory; every part is checked before any is launched.
static zero_status stage3_fused_q8(const zero_plan* plan, uint64_t flat_lo, uint64_t len,
                                   const uint8_t* const* rank_payload, const float* master_in,
                                   const float* m_in, const float* v_in, float* master_out,
                                   float* m_out, float* v_out, uint16_t* const* param_shards,
                                   const zk::AdamConsts& a, const zk::AdamConsts* ad,
                                   uint32_t* d_status, cudaStream_t stream) {
    int nd = 0;
    uint64_t psi_p = 0, S = 0, q_lo = 0, q_hi = 0;
    zero_status st = stage3_range(plan, flat_lo, len, &nd, &psi_p, &S, &q_lo, &q_hi);
    if (st != ZERO_OK) return st;
    if (!d_status) return ZERO_EINVAL;
    if (len == 0) return ZERO_OK;
    if (!rank_payload || !param_shards || !master_in || !m_in || !v_in || !master_out ||
        !m_out || !v_out)
        return ZERO_EINVAL;
    for (int r = 0; r < nd; ++r)
        if (!rank_payload[r]) return ZERO_EINVAL;
    const uint8_t* part_pay[ZERO_MAX_RANKS];
    for (int pass = 0; pass < 2; ++pass) {
        uint64_t seg = 0;
        for (uint64_t q = q_lo; q <= q_hi; ++q) {
            const uint64_t lo = flat_lo > q * S ? flat_lo : q * S;
            const uint64_t hi = (q + 1) * S < flat_lo + len ? (q + 1) * S : flat_lo + len;
            const uint64_t off = lo - flat_lo, n = hi - lo;
            for (int r = 0; r < nd; ++r) part_pay[r] = rank_payload[r] + seg;
            uint16_t* pout = param_shards[q] ? param_shards[q] + (lo - q * S) : nullptr;
            if (pass == 0) {
                st = check_fused_q8(n, nd, part_pay, master_in + off, m_in + off, v_in + off,
                                    master_out + off, m_out + off, v_out + off, pout, d_status);
                if (st != ZERO_OK) return st;
                for (uint64_t o = q_lo; o < q; ++o)   // partitions are distinct buffers
                    if (param_shards[o] &&
                        zk::overlap(param_shards[o], S * 2, param_shards[q], S * 2))
                        return ZERO_EINVAL;
            } else {
                const cudaError_t e = zk::launch_fused_q8(
                    n, nd, part_pay, master_in + off, m_in + off, v_in + off, master_out + off,
                    m_out + off, v_out + off, pout, a, ad, zk::make_mean(nd), d_status, stream);
                if (e != cudaSuccess) return zk::from_cuda(e);
            }
            seg += q8_segment_bytes(n);
        }
    }
    return ZERO_OK;
}

zero_status zero_stage3_step_fused_q8(const zero_plan* plan, uint64_t flat_lo, uint64_t len,
                                      const uint8_t* const* rank_payload, const float* master_in,
                                      const float* m_in, const float* v_in, float* master_out,
                                      float* m_out, float* v_out, uint16_t* const* param_shards,
                                      const zero_adam_hparams* hp, int64_t step,
                                      uint32_t* d_status, zero_stream_t stream) {
    if (!zk::hparams_ok(hp) || step < 1) return ZERO_EINVAL;
    return stage3_fused_q8(plan, flat_lo, len, rank_payload, master_in, m_in, v_in, master_out,
                           m_out, v_out, param_shards, zk::make_adam(hp, step), nullptr,
                           d_status, (cudaStream_t)stream);
}

zero_status zero_stage3_step_fused_q8_dc(const zero_plan* plan, uint64_t flat_lo, uint64_t len,
                                         const uint8_t* const* rank_payload,
                                         const float* master_in, const float* m_in,
                                         const float* v_in, float* master_out, float* m_out,
                                         float* v_out, uint16_t* const* param_shards,
                                         const zero_adam_consts* d_consts, uint32_t* d_status,
                                         zero_stream_t stream) {
    if (!d_consts) return ZERO_EINVAL;
    if (!zk::aligned(d_consts, 4)) return ZERO_EALIGN;
    zero_adam_consts unused;
    memset(&unused, 0, sizeof(unused));
    return stage3_fused_q8(plan, flat_lo, len, rank_payload, master_in, m_in, v_in, master_out,
                           m_out, v_out, param_shards, unused, d_consts, d_status,
                           (cudaStream_t)stream);
}

zero_status zero_stage3_step_commit(const zero_plan* plan, const float* master_in, const float* m_in,
                              const float* v_in, float* master_out, float* m_out, float* v_out,
                              uint16_t* const* param_shards, uint32_t* d_status,
                              zero_stream_t stream) {
    int nd = 0;
    uint64_t psi_p = 0, S = 0;
    if (!zk::plan_geometry(plan, &nd, &psi_p, &S)) return ZERO_EINVAL;
    if (!d_status || !param_shards || !master_in || !m_in || !v_in || !master_out || !m_out ||
        !v_out)
        return ZERO_EINVAL;
    for (int q = 0; q < nd; ++q) {
        const uint64_t off = (uint64_t)q * S;
        const zero_status st = zk::check_fused_state(
            S, master_in + off, m_in + off, v_in + off, master_out + off, m_out + off,
            v_out + off, param_shards[q], d_status);
        if (st != ZERO_OK) return st;
        for (int o = 0; o < q; ++o)
            if (zk::overlap(param_shards[o], S * 2, param_shards[q], S * 2)) return ZERO_EINVAL;
    }
    if (S == 0) return ZERO_OK;
    return zk::from_cuda(zk::launch_stage3_commit(S, nd, master_in, m_in, v_in, master_out,
                                                  m_out, v_out, param_shards, d_status,
                                                  (cudaStream_t)stream));
}

zero_status zero_step_status(const uint32_t* d_status, zero_stream_t stream, uint32_t* flags_out) {
    if (!d_status) return ZERO_EINVAL;
    if (!zk::aligned(d_status, 4)) return ZERO_EALIGN;
    uint32_t flags = 0;
    cudaError_t e = cudaMemcpyAsync(&flags, d_status, sizeof(flags), cudaMemcpyDeviceToHost,
                                    (cudaStream_t)stream);
    if (e == cudaSuccess) e = cudaStreamSynchronize((cudaStream_t)stream);
    if (e != cudaSuccess) return zk::from_cuda(e);
    if (flags_out) *flags_out = flags;
    if (flags & (ZERO_FLAG_TIMEOUT | ZERO_FLAG_BOUNDS)) return ZERO_ECUDA;
    if (flags & ZERO_FLAG_SKIPPED) return ZERO_STEP_SKIPPED;
    return ZERO_OK;
}

}  // extern "C"
