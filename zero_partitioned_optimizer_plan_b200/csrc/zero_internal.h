// Internal declarations shared by the libzero translation units (not part of the C ABI).
#pragma once

#include <cstdint>

#include <cuda_runtime.h>

#include "../../include/libzero.h"

namespace zk {

// fp32 constants of one Adam step, computed on the host (zero_api.cpp), in the public layout.
using AdamConsts = zero_adam_consts;

// The division of the rank sum by nd.
struct MeanConsts {
    float fnd;
    float inv_nd;      // 1/nd when nd is a power of two (then x*inv_nd == x/nd exactly)
    int nd_pow2;
};

// Plan accessors used by the data path and the scheduler (zero_plan.cpp).
bool plan_geometry(const zero_plan* p, int* nd, uint64_t* psi_p, uint64_t* shard);
bool plan_bucket_range(const zero_plan* p, int k, uint64_t* lo, uint64_t* len);
uint64_t plan_max_bucket(const zero_plan* p);
uint64_t plan_n_buckets(const zero_plan* p);

// Launchers (zero_kernels.cu). They validate nothing: the C ABI layer has done that.
// `ad` (device memory) overrides `a` when it is not null.
cudaError_t launch_fused(uint64_t n, int nd, const uint16_t* const* grads, const float* master_in,
                         const float* m_in, const float* v_in, float* master_out, float* m_out,
                         float* v_out, uint16_t* param_out, const AdamConsts& a,
                         const AdamConsts* ad, const MeanConsts& mc, uint32_t* status,
                         cudaStream_t stream, int n_replicas = 0,
                         uint16_t* const* replicas = nullptr);
// n_replicas > 0: the fp16 write-back (and the commit's repair) goes to every replicas[d]
// instead of param_out (the all-gather in the epilogue).
cudaError_t launch_commit(uint64_t n, const float* master_in, const float* m_in,
                          const float* v_in, float* master_out, float* m_out, float* v_out,
                          uint16_t* param_out, uint32_t* status, cudaStream_t stream,
                          int n_replicas = 0, uint16_t* const* replicas = nullptr);
cudaError_t launch_reduce_scatter(uint64_t n, int nd, const uint16_t* const* grads,
                                  float* const* shards, uint64_t flat_lo, uint64_t shard,
                                  const MeanConsts& mc, uint32_t* status, cudaStream_t stream);
cudaError_t launch_adam(uint64_t n, const float* grad, float* master, float* m, float* v,
                        uint16_t* param_out, const AdamConsts& a, const AdamConsts* ad,
                        uint32_t* status, cudaStream_t stream);

cudaError_t launch_selftest_timeout(uint32_t* status, cudaStream_t stream);
// Stage 3 (zero_stage3.cu): copy the flat range [flat_lo, flat_lo + len) out of the owners'
// fp16 partitions (shards[q]: S values) into out.
cudaError_t launch_gather(uint64_t flat_lo, uint64_t len, uint64_t shard, int nd,
                          const uint16_t* const* shards, uint16_t* out, uint32_t* status,
                          cudaStream_t stream);
// The commit of a stage-3 step over every owner in one launch (state flat, nd partitions).
cudaError_t launch_stage3_commit(uint64_t shard, int nd, const float* master_in,
                                 const float* m_in, const float* v_in, float* master_out,
                                 float* m_out, float* v_out, uint16_t* const* shards,
                                 uint32_t* status, cudaStream_t stream);
cudaError_t launch_quant_q8(uint64_t n, const uint16_t* grad, uint8_t* payload,
                            cudaStream_t stream);
cudaError_t launch_fused_q8(uint64_t n, int nd, const uint8_t* const* payload,
                            const float* master_in, const float* m_in, const float* v_in,
                            float* master_out, float* m_out, float* v_out, uint16_t* param_out,
                            const AdamConsts& a, const AdamConsts* ad, const MeanConsts& mc,
                            uint32_t* status, cudaStream_t stream);
cudaError_t launch_scaler_prepare(const zero_scaler_state* st, const AdamConsts* table,
                                  int64_t table_len, AdamConsts* out, uint32_t* status,
                                  cudaStream_t stream);
cudaError_t launch_scaler_update(zero_scaler_state* st, const zero_scaler_params& prm,
                                 const uint32_t* status, cudaStream_t stream);

// Whether the pipeline launch about to be made on `stream` may be chained to the previous one
// (a later call inside a zero_overlap_begin/end region); the first call of a region, and every
// call outside one, is ordered (zero_api.cpp).
bool overlap_next(cudaStream_t stream);

// Count of kernels this library has launched in this process.
void count_launch();
uint64_t launches();

// Launch the reduce-scatter of bucket k of a plan (arguments already validated).
cudaError_t rs_bucket_launch(const zero_plan* plan, int k, const uint16_t* const* rank_grads,
                             float* const* shards, uint32_t* status, cudaStream_t stream);

MeanConsts make_mean(int nd);

// Argument checks of a fused update over n elements (null, alignment, outputs overlapping
// inputs or each other); zero_api.cpp.
zero_status check_fused_state(uint64_t n, const float* master_in, const float* m_in,
                              const float* v_in, float* master_out, float* m_out, float* v_out,
                              uint16_t* param_out, uint32_t* d_status);

// Map a CUDA error to a zero_status, remembering its text for zero_last_error().
zero_status from_cuda(cudaError_t e);

}  // namespace zk
