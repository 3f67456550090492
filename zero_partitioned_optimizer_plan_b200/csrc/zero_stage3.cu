// ZeRO stage 3 (Pos+g+p) on one B200: the fp16 parameters are partitioned like the optimizer
// state, and each layer's parameters are gathered from the owners' partitions just in time.
//
// "ZeRO: particionar estados do treino entre GPUs" (upskillscore.com), "Como funciona": in the
// third stage the parameters are split among the Nd processes too, a process that needs a
// partition it does not own receives it from its owner, and a step moves 3 psi (a parameter
// all-gather in the forward pass, another in the backward pass, and the gradient
// reduce-scatter). "ZeRO" (lastdictionary.com), main definition: each layer's parameters are
// gathered just in time for its computation and discarded afterwards.
//
// With the Nd ranks simulated in one GPU's memory, the gather of a layer is a copy of the
// layer's flat range [flat_lo, flat_lo + len) out of the owners' partitions (separate
// buffers of S fp16 values) into one layer buffer that stands for every rank's gathered copy.
// It is a pure streaming copy: 2 bytes read and 2 bytes written per element, bound by HBM.
//
// Kernel shape. The output is cut into 16-byte chunks (8 fp16 values) aligned to the output
// buffer; the first elements up to that alignment and the last partial chunk are copied one
// by one. The range splits into per-owner segments (consecutive in the output); the host
// computes each segment's source pointer and the widest load its alignment allows for every
// chunk of the segment (chunk starts differ by 16 bytes, so the alignment class is the same
// for all of them): one 16-byte load, four 4-byte loads or eight 2-byte loads, never reading a
// byte outside the segment. A chunk that straddles two owners is copied one element at a
// time. Threads walk their chunks in increasing order, so each one finds a chunk's segment by
// moving forward through the segment table (at most Nd steps in all), with no division.
// Every thread keeps U chunks' loads in flight before it stores.
//
// The update of stage 3 is the fused step of zero_kernels.cu applied to each owner's part of
// a layer's range, its fp16 output written into that owner's partition; the commit of a step is
// one launch over every owner (commit3_kernel below).
#include <cuda_runtime.h>

#include <cstdint>
#include <cstring>

#include "zero_device.cuh"
#include "zero_internal.h"

namespace zk {
namespace {

constexpr int kGatherThreads = 256;
constexpr int kGatherUnroll = 4;   // 16-byte chunks in flight per thread

struct GatherArgs {
    const uint16_t* seg_src[kMaxRanks];   // the segment's first element in its owner's shard
    uint64_t seg_end[kMaxRanks];          // exclusive end of the segment in output elements
    uint8_t seg_vec[kMaxRanks];           // load width (bytes) of the segment's chunks
    uint16_t* out;
    uint32_t* status;
    uint64_t len;
    uint64_t head;       // elements before out + head is 16-byte aligned (<= len)
    uint64_t nchunks;    // whole 16-byte chunks after the head
    int nseg;
};

// Segment holding output element j, searching forward from `seg`; nseg if none (a bug).
__device__ __forceinline__ int seg_of(const GatherArgs& p, uint64_t j, int seg) {
    while (seg < p.nseg && j >= p.seg_end[seg]) ++seg;
    return seg;
}

__device__ __forceinline__ uint64_t seg_begin(const GatherArgs& p, int seg) {
    return seg == 0 ? 0 : p.seg_end[seg - 1];
}

__device__ __forceinline__ void copy_one(const GatherArgs& p, uint64_t j, int& seg) {
    seg = seg_of(p, j, seg);
    if (seg >= p.nseg || j >= p.len) {   // self-check: never taken when the table is right
        atomicOr(p.status, ZERO_FLAG_BOUNDS);
        return;
    }
    p.out[j] = p.seg_src[seg][j - seg_begin(p, seg)];
}

__device__ __forceinline__ uint4 load_chunk(const uint16_t* src, int vec) {
    uint4 v;
    if (vec == 16) {
        v = __ldcs(reinterpret_cast<const uint4*>(src));
    } else if (vec == 4) {
        const uint32_t* s = reinterpret_cast<const uint32_t*>(src);
        v.x = __ldg(s);
        v.y = __ldg(s + 1);
        v.z = __ldg(s + 2);
        v.w = __ldg(s + 3);
    } else {
        uint32_t h[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) h[i] = __ldg(reinterpret_cast<const unsigned short*>(src + i));
        v.x = h[0] | (h[1] << 16);
        v.y = h[2] | (h[3] << 16);
        v.z = h[4] | (h[5] << 16);
        v.w = h[6] | (h[7] << 16);
    }
    return v;
}

__global__ void __launch_bounds__(kGatherThreads) gather_kernel(const __grid_constant__ GatherArgs p) {
    // launched with programmatic stream serialization: the grid may be resident before the
    // previous kernel on the stream ends; it waits for that kernel here, before any access
    pdl_enter(0);
    const uint64_t tid = (uint64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const uint64_t stride = (uint64_t)gridDim.x * blockDim.x;
    int seg = 0;
    for (uint64_t c0 = tid; c0 < p.nchunks; c0 += stride * kGatherUnroll) {
        uint4 v[kGatherUnroll];
        uint8_t kind[kGatherUnroll];   // 0: none, 1: whole chunk loaded, 2: straddles owners
#pragma unroll
        for (int u = 0; u < kGatherUnroll; ++u) {
            const uint64_t c = c0 + (uint64_t)u * stride;
            kind[u] = 0;
            if (c >= p.nchunks) continue;
            const uint64_t j = p.head + 8 * c;
            seg = seg_of(p, j, seg);
            if (seg >= p.nseg) {
                atomicOr(p.status, ZERO_FLAG_BOUNDS);
                continue;
            }
            if (j + 8 > p.seg_end[seg]) {
                kind[u] = 2;
                continue;
            }
            v[u] = load_chunk(p.seg_src[seg] + (j - seg_begin(p, seg)), p.seg_vec[seg]);
            kind[u] = 1;
        }
#pragma unroll
        for (int u = 0; u < kGatherUnroll; ++u) {
            const uint64_t j = p.head + 8 * (c0 + (uint64_t)u * stride);
            if (kind[u] == 1) {
                *reinterpret_cast<uint4*>(p.out + j) = v[u];
            } else if (kind[u] == 2) {
                int s = 0;
                for (int e = 0; e < 8; ++e) copy_one(p, j + e, s);
            }
        }
    }
    // the head (before the first aligned chunk) and the tail (after the last whole chunk)
    if (blockIdx.x == 0) {
        const uint64_t tail0 = p.head + 8 * p.nchunks;
        const uint64_t extra = p.head + (p.len - tail0);   // < 16
        if (threadIdx.x < extra) {
            const uint64_t j = threadIdx.x < p.head ? threadIdx.x : tail0 + (threadIdx.x - p.head);
            int s = 0;
            copy_one(p, j, s);
        }
    }
}

// The commit of a stage-3 step in one launch: when the step is void, every owner's state is
// restored over the flat range and its fp16 partition rewritten from the restored master.
struct Commit3Args {
    const float* master_in;
    const float* m_in;
    const float* v_in;
    float* master_out;
    float* m_out;
    float* v_out;
    uint16_t* shards[kMaxRanks];
    uint32_t* status;
    uint64_t shard;
    int nd;
};

__global__ void __launch_bounds__(256) commit3_kernel(const __grid_constant__ Commit3Args p) {
    pdl_enter(0);
    if (!(*reinterpret_cast<volatile uint32_t*>(p.status) & kStepVoid)) return;
    if (blockIdx.x == 0 && threadIdx.x == 0) atomicOr(p.status, ZERO_FLAG_SKIPPED);
    const uint64_t n = p.shard * (uint64_t)p.nd;
    const uint64_t stride = (uint64_t)gridDim.x * blockDim.x;
    for (uint64_t i = (uint64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += stride) {
        const uint64_t q = i / p.shard;
        const float w = p.master_in[i];
        p.master_out[i] = w;
        p.m_out[i] = p.m_in[i];
        p.v_out[i] = p.v_in[i];
        p.shards[q][i - q * p.shard] = f2h(w);
    }
}

int load_width(const void* p) {
    const uintptr_t a = reinterpret_cast<uintptr_t>(p);
    return (a & 15u) == 0 ? 16 : (a & 3u) == 0 ? 4 : 2;
}

}  // namespace

cudaError_t launch_gather(uint64_t flat_lo, uint64_t len, uint64_t shard, int nd,
                          const uint16_t* const* shards, uint16_t* out, uint32_t* status,
                          cudaStream_t stream) {
    GatherArgs p;
    memset(&p, 0, sizeof(p));
    const uint64_t q_lo = flat_lo / shard, q_hi = (flat_lo + len - 1) / shard;
    if (q_hi >= (uint64_t)nd || q_hi - q_lo + 1 > (uint64_t)kMaxRanks) return cudaErrorInvalidValue;
    p.out = out;
    p.status = status;
    p.len = len;
    const uintptr_t oa = reinterpret_cast<uintptr_t>(out);
    uint64_t head = ((16u - (oa & 15u)) & 15u) / 2u;   // out is 2-byte aligned
    if (head > len) head = len;
    p.head = head;
    p.nchunks = (len - head) / 8;
    p.nseg = (int)(q_hi - q_lo + 1);
    for (uint64_t q = q_lo; q <= q_hi; ++q) {
        const int s = (int)(q - q_lo);
        const uint64_t a = flat_lo > q * shard ? flat_lo : q * shard;
        const uint64_t b = (q + 1) * shard < flat_lo + len ? (q + 1) * shard : flat_lo + len;
        p.seg_src[s] = shards[q] + (a - q * shard);
        p.seg_end[s] = b - flat_lo;
        // every whole chunk's output index j satisfies j = head (mod 8); its source address is
        // seg_src + 2*(j - seg_begin), so one alignment class holds for the whole segment
        const uint64_t seg_beg = a - flat_lo;
        const int64_t rel = ((int64_t)head - (int64_t)seg_beg) % 8;
        const uint16_t* first = p.seg_src[s] + (rel < 0 ? rel + 8 : rel);
        p.seg_vec[s] = (uint8_t)load_width(first);
    }
    DevInfo di;
    cudaError_t e = dev_info(&di);
    if (e != cudaSuccess) return e;
    const uint64_t per_block = (uint64_t)kGatherThreads * kGatherUnroll;
    uint64_t blocks = (p.nchunks + per_block - 1) / per_block;
    const uint64_t cap = (uint64_t)di.sms * 8;
    if (blocks > cap) blocks = cap;
    if (blocks < 1) blocks = 1;
    return launch_ordered(gather_kernel, p, (unsigned)blocks, kGatherThreads, stream);
}

cudaError_t launch_stage3_commit(uint64_t shard, int nd, const float* master_in,
                                 const float* m_in, const float* v_in, float* master_out,
                                 float* m_out, float* v_out, uint16_t* const* shards,
                                 uint32_t* status, cudaStream_t stream) {
    Commit3Args p;
    memset(&p, 0, sizeof(p));
    p.master_in = master_in;
    p.m_in = m_in;
    p.v_in = v_in;
    p.master_out = master_out;
    p.m_out = m_out;
    p.v_out = v_out;
    for (int q = 0; q < nd; ++q) p.shards[q] = shards[q];
    p.status = status;
    p.shard = shard;
    p.nd = nd;
    DevInfo di;
    const cudaError_t e = dev_info(&di);
    if (e != cudaSuccess) return e;
    return launch_ordered(commit3_kernel, p, plain_grid(shard * (uint64_t)nd, di.sms), 256,
                          stream);
}

}  // namespace zk
