// libzero kernels for sm_100a (B200).
//
// The path is a streaming reduction plus an elementwise update: per parameter it reads Nd fp16
// gradients (2*Nd bytes), 12 bytes of fp32 optimizer state and writes 12 + 2 bytes back, at
// about one flop per byte. Nothing is a dense contraction, so no tensor cores; the bound is
// HBM bandwidth, and the design is about keeping enough bytes in flight:
//
//   * persistent grid, one CTA per SM, tiles of T elements taken round-robin;
//   * one producer warp per CTA streams each tile's Nd gradient rows and three state rows into
//     a ring of shared-memory stages with 1-D bulk async copies (cp.async.bulk ...
//     mbarrier::complete_tx, no multicast), so 100-200 KB per SM are in flight without
//     spending registers on it;
//   * 16-24 consumer warps (by Nd) sum the Nd rows in rank order in fp32, release the stage,
//     then run Adam and store fp32 state and fp16 parameters straight from registers;
//   * a warp vote collects the overflow (inf/NaN) check, one atomicOr per warp at the end;
//   * programmatic dependent launch lets the next call's CTAs start while this one drains
//     (ordered by default; overlapped inside a zero_overlap_begin/end region).
//
// Every wait on an mbarrier is bounded (1 s); on expiry the kernel sets ZERO_FLAG_TIMEOUT,
// lets its own copies in flight land, and returns.
//
// Arithmetic (identical in every kernel here; see include/libzero.h):
//   red = (sum_{r=0..nd-1} fp32(g_r)) / nd, the sum strictly in rank order;
//   g = red / loss_scale; m = b1*m + (1-b1)*g; v = b2*v + (1-b2)*(g*g);
//   w = w - step_size * (m / (sqrt(v)/bc2s + eps)); p = fp16_rn(w)
// with every operation a separately rounded IEEE fp32 operation (no FMA contraction; this file
// is also compiled with -fmad=false). A division by a power of two is done as the product with
// its exact reciprocal, which is the same correctly rounded real number.
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cstdint>
#include <cstring>

#include "zero_device.cuh"
#include "zero_internal.h"

namespace zk {

namespace {

struct FusedArgs {
    const uint16_t* grads[kMaxRanks];
    const float* master_in;
    const float* m_in;
    const float* v_in;
    float* master_out;
    float* m_out;
    float* v_out;
    uint16_t* param_out;
    uint32_t* status;
    uint64_t n;          // elements of the range
    uint64_t n_tiled;    // elements covered by tiles (multiple of 8); [n_tiled, n) is the tail
    uint64_t num_tiles;
    Geom g;
    int nd;
    int param_vec;       // widest param store the pointer's alignment allows: 16, 8, 4, 2
    AdamConsts a;
    const AdamConsts* ad;  // when not null: the constants, read from device memory at run time
    MeanConsts mc;
    int selftest_no_copies;  // self-test only: the producer issues nothing (waits must expire)
    int chained;         // programmatic launch chained to the previous call (see pdl_enter)
};

// The fused step with the all-gather in its epilogue: the fp16 values go to every replica's
// buffer (replicas[d], possibly a peer's address) instead of param_out. A separate argument
// type, so that the one-buffer kernels keep their parameter block and code unchanged.
struct FusedRepArgs : FusedArgs {
    int n_replicas;
    uint16_t* replicas[kMaxRanks];
};

// The fp16 write-back of one value, or of a thread's E values.
__device__ __forceinline__ void store_param(const FusedArgs& p, uint64_t i, float w) {
    p.param_out[i] = f2h(w);
}

__device__ __forceinline__ void store_param(const FusedRepArgs& p, uint64_t i, float w) {
    const uint16_t h = f2h(w);
    for (int d = 0; d < p.n_replicas; ++d) p.replicas[d][i] = h;
}

template <int E>
__device__ __forceinline__ void store_params(const FusedArgs& p, uint64_t g0,
                                             const float (&w)[E]) {
    stg_f16<E>(p.param_out + g0, w, p.param_vec);
}

template <int E>
__device__ __forceinline__ void store_params(const FusedRepArgs& p, uint64_t g0,
                                             const float (&w)[E]) {
    for (int d = 0; d < p.n_replicas; ++d) stg_f16<E>(p.replicas[d] + g0, w, p.param_vec);
}

struct RsArgs {
    const uint16_t* grads[kMaxRanks];
    float* shards[kMaxRanks];
    uint32_t* status;
    uint64_t n;
    uint64_t n_tiled;
    uint64_t num_tiles;
    uint64_t flat_lo;    // flat index of element 0 of the bucket
    uint64_t shard;      // S
    double inv_shard;    // 1/S, for the owner estimate
    Geom g;
    int nd;
    MeanConsts mc;
    int chained;         // programmatic launch chained to the previous call (see pdl_enter)
};

struct CommitArgs {
    const float* master_in;
    const float* m_in;
    const float* v_in;
    float* master_out;
    float* m_out;
    float* v_out;
    uint16_t* param_out;
    uint32_t* status;
    uint64_t n;
    int n_replicas;                  // > 0: restore every replica's range instead of param_out
    uint16_t* replicas[kMaxRanks];
};

struct AdamArgs {
    const float* grad;
    float* master;
    float* m;
    float* v;
    uint16_t* param_out;
    uint32_t* status;
    uint64_t n;
    int vec;             // 1: every fp32 pointer 16-byte aligned (float4 path)
    int param_vec;       // 8, 4 or 2
    AdamConsts a;
    const AdamConsts* ad;  // when not null: the constants, read from device memory at run time
};

// ---------------------------------------------------------------------------------------------
// the pipeline
//
// A tile is T consecutive elements. Its Nd gradient rows are split into chunks of at most
// `rc` ranks; chunk c of a tile fills one shared-memory stage with rows c*rc .. c*rc+nr-1 (and,
// for the last chunk of a fused tile, the three fp32 state rows). The CTA walks its tiles
// round-robin and, within a tile, its chunks in rank order, so the same consumer thread adds
// rank 0, 1, ..., Nd-1 of each of its elements into one accumulator: the order of the sum does
// not depend on the chunking. Stage s of iteration `it` is it % stages, its use it / stages.
// ---------------------------------------------------------------------------------------------
__device__ __forceinline__ const float* state_row(const FusedArgs& p, uint32_t k) {
    return k == 0 ? p.master_in : (k == 1 ? p.m_in : p.v_in);
}

__device__ __forceinline__ const float* state_row(const RsArgs&, uint32_t) { return nullptr; }

// Producer: the whole warp; lane 0 posts each stage's byte count and all lanes issue copies.
template <bool kState, typename Args>
__device__ void produce(const Args& p, uint64_t* full, uint64_t* empty, uint8_t* data) {
    const Geom& g = p.g;
    const uint32_t T = g.tile;
    const int lane = threadIdx.x & 31;
    uint32_t it = 0;
    bool ok = true;
    for (uint64_t tile = blockIdx.x; ok && tile < p.num_tiles; tile += gridDim.x) {
        const TileSpan ts = tile_span(tile, T, p.n_tiled);
        for (uint32_t c = 0; c < g.nchunks; ++c, ++it) {
            const uint32_t s = it % g.stages;
            const uint32_t use = it / g.stages;
            if (use > 0) {
                // the stage's previous fill must have been read by every consumer warp
                bool w = true;
                if (lane == 0) w = mbar_wait(&empty[s], (use - 1) & 1u);
                if (!__shfl_sync(0xffffffffu, w, 0)) {
                    ok = false;
                    break;
                }
            }
            const uint32_t r0 = c * g.rc;
            const uint32_t nr = min(g.rc, (uint32_t)p.nd - r0);
            const bool with_state = kState && c + 1 == g.nchunks;
            const uint32_t gb = ts.cnt * 2u, fb = ts.cnt * 4u;
            uint8_t* st = data + (size_t)s * g.stage_bytes;
            const bool sane = ts.base < p.n_tiled && (ts.cnt & 7u) == 0 && ts.cnt > 0 &&
                              r0 < (uint32_t)p.nd && nr <= g.rc && s < (uint32_t)g.stages;
            if (lane == 0) {
                if (!sane) atomicOr(p.status, ZERO_FLAG_BOUNDS);
                mbar_arrive_expect_tx(&full[s], sane ? nr * gb + (with_state ? 3u * fb : 0u) : 0u);
            }
            __syncwarp();
            if (!sane) continue;   // consumers are released without data; stores are checked
            const uint32_t ncopy = nr + (with_state ? 3u : 0u);
            for (uint32_t j = (uint32_t)lane; j < ncopy; j += 32u) {
                if (j < nr) {
                    bulk_g2s(st + (size_t)j * T * 2u, p.grads[r0 + j] + ts.base, gb, &full[s]);
                } else {
                    const uint32_t k = j - nr;
                    bulk_g2s(st + g.state_off + (size_t)k * T * 4u, state_row(p, k) + ts.base, fb,
                             &full[s]);
                }
            }
        }
    }
    if (!ok && lane == 0) {
        atomicOr(p.status, ZERO_FLAG_TIMEOUT);
        // let every copy this warp started land before the CTA can exit
        for (uint32_t s = 0; s < (uint32_t)g.stages && s < it; ++s) {
            const uint32_t last = s + ((it - 1u - s) / (uint32_t)g.stages) * (uint32_t)g.stages;
            (void)mbar_wait(&full[s], (last / (uint32_t)g.stages) & 1u);
        }
    }
}

// ---------------------------------------------------------------------------------------------
// fused step: reduce-scatter + unscale + Adam + fp16 cast + write-back, TMA-pipelined
// ---------------------------------------------------------------------------------------------
template <typename Args>
__device__ __forceinline__ void fused_element(const Args& p, const AdamConsts& a, uint64_t i,
                                              bool& bad) {
    if (i >= p.n) {   // self-check: never taken when the launch arithmetic is right
        atomicOr(p.status, ZERO_FLAG_BOUNDS);
        return;
    }
    float s = 0.0f;
    for (int r = 0; r < p.nd; ++r) s = __fadd_rn(s, h2f(p.grads[r][i]));
    const float red = mean_of(s, p.mc);
    bad |= non_finite(red);
    float w = p.master_in[i], m = p.m_in[i], v = p.v_in[i];
    adam_elem(red, w, m, v, a);
    p.master_out[i] = w;
    p.m_out[i] = m;
    p.v_out[i] = v;
    store_param(p, i, w);
}

template <int E, int W, bool kDC, typename Args = FusedArgs>
__global__ void __launch_bounds__(Warps<W>::kThreads, Warps<W>::kMinBlocks)
    fused_tma_kernel(const __grid_constant__ Args p) {
    extern __shared__ __align__(128) uint8_t smem[];
    uint64_t* full = reinterpret_cast<uint64_t*>(smem);
    uint64_t* empty = full + kMaxStages;
    uint8_t* data = smem + kDataOffset;
    init_barriers(full, empty, p.g.stages, W);
    pdl_enter(p.chained);

    if ((threadIdx.x >> 5) == W) {
        if (!p.selftest_no_copies) produce<true>(p, full, empty, data);
        pdl_leave(p.chained);
        return;
    }

    // consumers: thread t owns elements [t*E, t*E + E) of every tile
    ZK_STEP_CONSTS(p, a);
    bool bad = false;
    const uint32_t T = p.g.tile;
    const uint32_t e0 = (uint32_t)threadIdx.x * E;
    uint32_t it = 0;
    bool ok = p.g.tile == 32u * W * E;   // self-check of the launch's shape
    if (!ok && threadIdx.x == 0) atomicOr(p.status, ZERO_FLAG_BOUNDS);
    for (uint64_t tile = blockIdx.x; ok && tile < p.num_tiles; tile += gridDim.x) {
        const TileSpan ts = tile_span(tile, T, p.n_tiled);
        const bool active = e0 < ts.cnt;   // cnt is a multiple of 8, E divides 8
        float acc[E], w[E], m[E], v[E];
#pragma unroll
        for (int j = 0; j < E; ++j) acc[j] = 0.0f;
        for (uint32_t c = 0; c < p.g.nchunks; ++c, ++it) {
            if (!consume_stage<E, true, 32u * W * E>(
                    p.g, p.nd, full, empty, data, it, c, e0, active, acc, w,
                                        m, v)) {
                if ((threadIdx.x & 31) == 0) atomicOr(p.status, ZERO_FLAG_TIMEOUT);
                ok = false;
                break;
            }
        }
        if (!ok || !active) continue;
        const uint64_t g0 = ts.base + e0;
        if (g0 + E > p.n_tiled) {
            atomicOr(p.status, ZERO_FLAG_BOUNDS);
            continue;
        }
#pragma unroll
        for (int j = 0; j < E; ++j) {
            const float red = mean_of(acc[j], p.mc);
            bad |= non_finite(red);
            adam_elem(red, w[j], m[j], v[j], a);
        }
        stg_f32<E>(p.master_out + g0, w);
        stg_f32<E>(p.m_out + g0, m);
        stg_f32<E>(p.v_out + g0, v);
        store_params<E>(p, g0, w);
    }
    // the < 8 elements past the last tile
    if (blockIdx.x == 0 && (uint64_t)threadIdx.x < p.n - p.n_tiled)
        fused_element(p, a, p.n_tiled + threadIdx.x, bad);
    flag_overflow(bad, p.status);
    pdl_leave(p.chained);
}

// plain-load variant for ranges whose pointers are not 16-byte aligned (or tiny ranges)
template <bool kDC, typename Args = FusedArgs>
__global__ void __launch_bounds__(256) fused_plain_kernel(const __grid_constant__ Args p) {
    ZK_STEP_CONSTS(p, a);
    bool bad = false;
    const uint64_t stride = (uint64_t)gridDim.x * blockDim.x;
    for (uint64_t i = (uint64_t)blockIdx.x * blockDim.x + threadIdx.x; i < p.n; i += stride)
        fused_element(p, a, i, bad);
    flag_overflow(bad, p.status);
}

// ---------------------------------------------------------------------------------------------
// bucketed reduce-scatter: red -> owner shard, TMA-pipelined
// ---------------------------------------------------------------------------------------------
__device__ __forceinline__ uint32_t owner_of(uint64_t f, const RsArgs& p) {
    uint64_t o = (uint64_t)((double)f * p.inv_shard);
    while (o > 0 && o * p.shard > f) --o;
    while ((o + 1) * p.shard <= f) ++o;
    return (uint32_t)o;
}

__device__ __forceinline__ void rs_store_one(const RsArgs& p, uint64_t local, float red) {
    const uint64_t f = p.flat_lo + local;
    const uint32_t o = owner_of(f, p);
    if (o >= (uint32_t)p.nd) {
        atomicOr(p.status, ZERO_FLAG_BOUNDS);
        return;
    }
    __stcs(p.shards[o] + (f - (uint64_t)o * p.shard), red);
}

__device__ __forceinline__ void rs_element(const RsArgs& p, uint64_t i, bool& bad) {
    if (i >= p.n) {
        atomicOr(p.status, ZERO_FLAG_BOUNDS);
        return;
    }
    float s = 0.0f;
    for (int r = 0; r < p.nd; ++r) s = __fadd_rn(s, h2f(p.grads[r][i]));
    const float red = mean_of(s, p.mc);
    bad |= non_finite(red);
    rs_store_one(p, i, red);
}

template <int E, int W>
__global__ void __launch_bounds__(Warps<W>::kThreads, Warps<W>::kMinBlocks)
    rs_tma_kernel(const __grid_constant__ RsArgs p) {
    extern __shared__ __align__(128) uint8_t smem[];
    uint64_t* full = reinterpret_cast<uint64_t*>(smem);
    uint64_t* empty = full + kMaxStages;
    uint8_t* data = smem + kDataOffset;
    init_barriers(full, empty, p.g.stages, W);
    pdl_enter(p.chained);

    if ((threadIdx.x >> 5) == W) {
        produce<false>(p, full, empty, data);
        pdl_leave(p.chained);
        return;
    }

    bool bad = false;
    const uint32_t T = p.g.tile;
    const uint32_t e0 = (uint32_t)threadIdx.x * E;
    uint32_t it = 0;
    bool ok = p.g.tile == 32u * W * E;   // self-check of the launch's shape
    if (!ok && threadIdx.x == 0) atomicOr(p.status, ZERO_FLAG_BOUNDS);
    for (uint64_t tile = blockIdx.x; ok && tile < p.num_tiles; tile += gridDim.x) {
        const TileSpan ts = tile_span(tile, T, p.n_tiled);
        const bool active = e0 < ts.cnt;
        float acc[E], unused[E];
#pragma unroll
        for (int j = 0; j < E; ++j) acc[j] = 0.0f;
        for (uint32_t c = 0; c < p.g.nchunks; ++c, ++it) {
            if (!consume_stage<E, false, 32u * W * E>(
                    p.g, p.nd, full, empty, data, it, c, e0, active, acc,
                                         unused, unused, unused)) {
                if ((threadIdx.x & 31) == 0) atomicOr(p.status, ZERO_FLAG_TIMEOUT);
                ok = false;
                break;
            }
        }
        if (!ok || !active) continue;
#pragma unroll
        for (int j = 0; j < E; ++j) {
            acc[j] = mean_of(acc[j], p.mc);
            bad |= non_finite(acc[j]);
        }
        const uint64_t l0 = ts.base + e0;
        const uint64_t f0 = p.flat_lo + l0;
        const uint32_t o0 = owner_of(f0, p);
        const uint32_t o1 = owner_of(f0 + E - 1, p);
        if (l0 + E > p.n_tiled || o1 >= (uint32_t)p.nd) {
            atomicOr(p.status, ZERO_FLAG_BOUNDS);
            continue;
        }
        if (o0 == o1) {
            stg_f32_any<E>(p.shards[o0] + (f0 - (uint64_t)o0 * p.shard), acc);
        } else {
#pragma unroll
            for (int j = 0; j < E; ++j) rs_store_one(p, l0 + j, acc[j]);
        }
    }
    if (blockIdx.x == 0 && (uint64_t)threadIdx.x < p.n - p.n_tiled)
        rs_element(p, p.n_tiled + threadIdx.x, bad);
    flag_overflow(bad, p.status);
    pdl_leave(p.chained);
}

__global__ void __launch_bounds__(256) rs_plain_kernel(const __grid_constant__ RsArgs p) {
    bool bad = false;
    const uint64_t stride = (uint64_t)gridDim.x * blockDim.x;
    for (uint64_t i = (uint64_t)blockIdx.x * blockDim.x + threadIdx.x; i < p.n; i += stride)
        rs_element(p, i, bad);
    flag_overflow(bad, p.status);
}

// ---------------------------------------------------------------------------------------------
// owner update of a shard from its reduced gradient (unfused path), in place.
// 30 bytes per parameter, half of them written back to the addresses just read; plain
// 128-bit loads with two groups in flight per thread measured faster on B200 (6.18 TB/s) than
// a bulk-copy pipeline like the fused kernel's (5.2-6.0 TB/s for 8-24 consumer warps).
// ---------------------------------------------------------------------------------------------
template <bool kDC>
__global__ void __launch_bounds__(256) adam_kernel(const __grid_constant__ AdamArgs p) {
    pdl_enter(0);   // ordered after the reduce-scatters (see launch_ordered)
    // skip the whole step if any reduce-scatter of it saw inf/NaN, or if one of them failed
    // (its reduced shard is then incomplete)
    if (*reinterpret_cast<volatile uint32_t*>(p.status) & kStepVoid) {
        if (blockIdx.x == 0 && threadIdx.x == 0) atomicOr(p.status, ZERO_FLAG_SKIPPED);
        return;
    }
    ZK_STEP_CONSTS(p, a);
    const uint64_t tid = (uint64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const uint64_t stride = (uint64_t)gridDim.x * blockDim.x;
    uint64_t done = 0;
    if (p.vec) {
        // U float4 groups per thread and iteration: all their loads are issued before any
        // arithmetic, so U*64 bytes per thread are in flight
        constexpr int U = ZK_ADAM_UNROLL;
        const uint64_t n4 = p.n / 4;
        for (uint64_t q0 = tid; q0 < n4; q0 += stride * U) {
            float4 g[U], w[U], m[U], v[U];
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const uint64_t q = q0 + (uint64_t)u * stride;
                if (q < n4) {
                    g[u] = __ldcs(reinterpret_cast<const float4*>(p.grad) + q);
                    w[u] = __ldcs(reinterpret_cast<const float4*>(p.master) + q);
                    m[u] = __ldcs(reinterpret_cast<const float4*>(p.m) + q);
                    v[u] = __ldcs(reinterpret_cast<const float4*>(p.v) + q);
                }
            }
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const uint64_t q = q0 + (uint64_t)u * stride;
                if (q >= n4) break;
                adam_elem(g[u].x, w[u].x, m[u].x, v[u].x, a);
                adam_elem(g[u].y, w[u].y, m[u].y, v[u].y, a);
                adam_elem(g[u].z, w[u].z, m[u].z, v[u].z, a);
                adam_elem(g[u].w, w[u].w, m[u].w, v[u].w, a);
                __stcs(reinterpret_cast<float4*>(p.master) + q, w[u]);
                __stcs(reinterpret_cast<float4*>(p.m) + q, m[u]);
                __stcs(reinterpret_cast<float4*>(p.v) + q, v[u]);
                const float x[4] = {w[u].x, w[u].y, w[u].z, w[u].w};
                stg_f16<4>(p.param_out + 4 * q, x, p.param_vec);
            }
        }
        done = n4 * 4;
    }
    for (uint64_t i = done + tid; i < p.n; i += stride) {
        float w = p.master[i], m = p.m[i], v = p.v[i];
        adam_elem(p.grad[i], w, m, v, a);
        p.master[i] = w;
        p.m[i] = m;
        p.v[i] = v;
        p.param_out[i] = f2h(w);
    }
}

// ---------------------------------------------------------------------------------------------
// commit / skip of a fused step
// ---------------------------------------------------------------------------------------------
// The step is void -- its inputs are restored over its outputs -- when a reduced gradient
// overflowed, and also when a kernel of the step gave up on a wait or failed its bounds
// self-check: those leave some tiles of the outputs unwritten.
__global__ void __launch_bounds__(256) commit_kernel(const __grid_constant__ CommitArgs p) {
    pdl_enter(0);   // ordered after the step's kernels (see launch_ordered)
    if (!(*reinterpret_cast<volatile uint32_t*>(p.status) & kStepVoid)) return;
    if (blockIdx.x == 0 && threadIdx.x == 0) atomicOr(p.status, ZERO_FLAG_SKIPPED);
    const uint64_t stride = (uint64_t)gridDim.x * blockDim.x;
    for (uint64_t i = (uint64_t)blockIdx.x * blockDim.x + threadIdx.x; i < p.n; i += stride) {
        const float w = p.master_in[i];
        p.master_out[i] = w;
        p.m_out[i] = p.m_in[i];
        p.v_out[i] = p.v_in[i];
        const uint16_t h = f2h(w);
        if (p.n_replicas == 0) {
            p.param_out[i] = h;
        } else {
            for (int d = 0; d < p.n_replicas; ++d) p.replicas[d][i] = h;
        }
    }
}

// ---------------------------------------------------------------------------------------------
// dynamic loss scaling: one thread each, before and after a step
// ---------------------------------------------------------------------------------------------
__global__ void scaler_prepare_kernel(const zero_scaler_state* st, const AdamConsts* table,
                                      int64_t table_len, AdamConsts* out, uint32_t* status) {
    if (threadIdx.x != 0 || blockIdx.x != 0) return;
    const int64_t t = st->next_step;
    if (t < 1 || t > table_len) {   // refuse the step: skipped by its kernels, scaler kept
        *status = ZERO_FLAG_OVERFLOW | ZERO_FLAG_BOUNDS;
        return;
    }
    *status = 0u;
    AdamConsts c = table[t - 1];
    const float s = st->scale;
    const uint32_t bits = __float_as_uint(s);
    const uint32_t e = (bits >> 23) & 0xffu;
    // a positive power of two 2^k whose reciprocal 2^-k is a normal number (1 <= e <= 253):
    // the unscale may multiply by the exact reciprocal instead of dividing
    const bool pow2 = (bits & 0x807fffffu) == 0u && e >= 1u && e <= 253u;
    c.loss_scale = s;
    c.inv_loss_scale = pow2 ? __uint_as_float((254u - e) << 23) : 0.0f;
    c.loss_scale_pow2 = pow2 ? 1 : 0;
    *out = c;
}

__global__ void scaler_update_kernel(zero_scaler_state* st, zero_scaler_params prm,
                                     const uint32_t* status) {
    if (threadIdx.x != 0 || blockIdx.x != 0) return;
    const uint32_t f = *status;
    if (f & (ZERO_FLAG_TIMEOUT | ZERO_FLAG_BOUNDS)) return;   // an error, not an overflow
    if (f & ZERO_FLAG_OVERFLOW) {
        st->scale = __fmul_rn(st->scale, prm.backoff_factor);
        st->good_steps = 0;
        st->skipped_steps += 1;
    } else {
        st->next_step += 1;
        st->good_steps += 1;
        if (st->good_steps >= prm.growth_interval) {
            st->scale = __fmul_rn(st->scale, prm.growth_factor);
            st->good_steps = 0;
        }
    }
}

// ---------------------------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------------------------
std::atomic<uint64_t> g_launches{0};


// Tile = 32 * warps * kElems elements; as many rank rows per stage as leave target_stages
// stages inside the shared-memory budget, the ranks split evenly into chunks.
PipeShape make_shape(int nd, bool with_state, int warps, int target_stages, size_t budget) {
    PipeShape sh;
    sh.warps = warps;
    sh.grid_per_sm = 0;
    Geom& g = sh.g;
    g.tile = (uint32_t)(32 * warps * kElems);
    const size_t row = (size_t)g.tile * 2u;
    const size_t state = with_state ? (size_t)g.tile * 12u : 0u;
    const size_t per_stage = budget / (size_t)target_stages;
    size_t rc_max = per_stage > state + row ? (per_stage - state) / row : 1;
    if (rc_max > (size_t)nd) rc_max = (size_t)nd;
    g.nchunks = (uint32_t)(((size_t)nd + rc_max - 1) / rc_max);
    g.rc = (uint32_t)(((size_t)nd + g.nchunks - 1) / g.nchunks);
    g.state_off = (uint32_t)(g.rc * row);
    g.stage_bytes = (uint32_t)(g.state_off + state);
    size_t st = budget / g.stage_bytes;
    if (st < 2) st = 2;
    if (st > kMaxStages) st = kMaxStages;
    g.stages = (int)st;
    sh.smem = (size_t)kDataOffset + st * g.stage_bytes;
    return sh;
}

// The shape of a call over n elements: the per-Nd table, or for a call too small to give
// every SM several tiles, the small shape (one CTA per SM, room for a second CTA of the next
// call on the same SM).
PipeShape pipe_shape(int nd, bool with_state, uint64_t n, int sms) {
    const Variant var = pick_variant(nd);
    const SmallVariant small = pick_small_variant(nd);
    const uint64_t big_tile = 32ull * (uint64_t)var.warps * kElems;
    const uint64_t tiles = (n + big_tile - 1) / big_tile;
    if (tiles < (uint64_t)small.max_tiles_per_sm * (uint64_t)sms) {
        PipeShape sh = make_shape(nd, with_state, small.warps, 2, ZK_SMALL_BUDGET);
        sh.grid_per_sm = 1;
        return sh;
    }
    return make_shape(nd, with_state, var.warps, var.target_stages, kSmemBudget);
}

// Launch a bulk-copy kernel template instantiated for the shape's number of consumer warps.
#define ZK_LAUNCH_BY_WARPS(KERNEL, ...)                                                    \
    switch (sh.warps) {                                                                    \
        case 8: return launch_pipe(KERNEL<kElems, 8 __VA_ARGS__>, p, sh, stream);          \
        case 12: return launch_pipe(KERNEL<kElems, 12 __VA_ARGS__>, p, sh, stream);        \
        case 16: return launch_pipe(KERNEL<kElems, 16 __VA_ARGS__>, p, sh, stream);        \
        case 20: return launch_pipe(KERNEL<kElems, 20 __VA_ARGS__>, p, sh, stream);        \
        case 24: return launch_pipe(KERNEL<kElems, 24 __VA_ARGS__>, p, sh, stream);        \
        case 28: return launch_pipe(KERNEL<kElems, 28 __VA_ARGS__>, p, sh, stream);        \
    }                                                                                      \
    return cudaErrorInvalidConfiguration

}  // namespace

void count_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }

// Launch the fused pipeline on one tile whose producer issues nothing: every consumer's bounded
// wait on the first stage expires, the kernel sets ZERO_FLAG_TIMEOUT and returns. No global
// memory is read or written except the status word.
cudaError_t launch_selftest_timeout(uint32_t* status, cudaStream_t stream) {
    FusedArgs p;
    memset(&p, 0, sizeof(p));
    p.status = status;
    p.nd = 1;
    p.n = 4096;
    p.n_tiled = 4096;
    p.selftest_no_copies = 1;
    p.mc = make_mean(1);
    DevInfo di;
    cudaError_t e = dev_info(&di);
    if (e != cudaSuccess) return e;
    const PipeShape sh = pipe_shape(1, true, p.n, di.sms);
    p.g = sh.g;
    p.num_tiles = 1;
    ZK_LAUNCH_BY_WARPS(fused_tma_kernel, , false);
}

uint64_t launches() { return g_launches.load(std::memory_order_relaxed); }

// The launch of either argument type: the one-buffer step, or the epilogue all-gather.
template <typename Args>
cudaError_t launch_fused_args(Args& p, bool all16, cudaStream_t stream) {
    DevInfo di;
    cudaError_t e = dev_info(&di);
    if (e != cudaSuccess) return e;
    if (!all16 || p.n < kMinTiledElems) {
        if (p.ad)
            fused_plain_kernel<true, Args><<<plain_grid(p.n, di.sms), 256, 0, stream>>>(p);
        else
            fused_plain_kernel<false, Args><<<plain_grid(p.n, di.sms), 256, 0, stream>>>(p);
        count_launch();
        return cudaGetLastError();
    }
    const PipeShape sh = pipe_shape(p.nd, true, p.n, di.sms);
    p.g = sh.g;
    p.n_tiled = p.n & ~(uint64_t)7;
    p.num_tiles = (p.n_tiled + sh.g.tile - 1) / sh.g.tile;
    p.chained = overlap_next(stream) ? 1 : 0;
    if (p.ad) {
        ZK_LAUNCH_BY_WARPS(fused_tma_kernel, , true, Args);
    }
    ZK_LAUNCH_BY_WARPS(fused_tma_kernel, , false, Args);
}

cudaError_t launch_fused(uint64_t n, int nd, const uint16_t* const* grads, const float* master_in,
                         const float* m_in, const float* v_in, float* master_out, float* m_out,
                         float* v_out, uint16_t* param_out, const AdamConsts& a,
                         const AdamConsts* ad, const MeanConsts& mc, uint32_t* status,
                         cudaStream_t stream, int n_replicas, uint16_t* const* replicas) {
    FusedArgs p;
    memset(&p, 0, sizeof(p));
    bool all16 = aligned16(master_in) && aligned16(m_in) && aligned16(v_in) &&
                 aligned16(master_out) && aligned16(m_out) && aligned16(v_out);
    for (int r = 0; r < nd; ++r) {
        p.grads[r] = grads[r];
        all16 = all16 && aligned16(grads[r]);
    }
    p.master_in = master_in;
    p.m_in = m_in;
    p.v_in = v_in;
    p.master_out = master_out;
    p.m_out = m_out;
    p.v_out = v_out;
    p.param_out = param_out;
    p.status = status;
    p.n = n;
    p.nd = nd;
    p.param_vec = store_vec(param_out);
    p.a = a;
    p.ad = ad;
    p.mc = mc;
    if (n_replicas == 0) return launch_fused_args(p, all16, stream);
    FusedRepArgs q;
    memset(&q, 0, sizeof(q));
    static_cast<FusedArgs&>(q) = p;
    q.n_replicas = n_replicas;
    for (int d = 0; d < n_replicas; ++d) {   // one store width that every replica allows
        q.replicas[d] = replicas[d];
        const int v = store_vec(replicas[d]);
        if (d == 0 || v < q.param_vec) q.param_vec = v;
    }
    return launch_fused_args(q, all16, stream);
}

cudaError_t launch_reduce_scatter(uint64_t n, int nd, const uint16_t* const* grads,
                                  float* const* shards, uint64_t flat_lo, uint64_t shard,
                                  const MeanConsts& mc, uint32_t* status, cudaStream_t stream) {
    RsArgs p;
    memset(&p, 0, sizeof(p));
    bool all16 = true;
    for (int r = 0; r < nd; ++r) {
        p.grads[r] = grads[r];
        p.shards[r] = shards[r];
        all16 = all16 && aligned16(grads[r]);
    }
    p.status = status;
    p.n = n;
    p.flat_lo = flat_lo;
    p.shard = shard;
    p.inv_shard = 1.0 / (double)shard;
    p.nd = nd;
    p.mc = mc;
    DevInfo di;
    cudaError_t e = dev_info(&di);
    if (e != cudaSuccess) return e;
    if (!all16 || n < kMinTiledElems) {
        rs_plain_kernel<<<plain_grid(n, di.sms), 256, 0, stream>>>(p);
        count_launch();
        return cudaGetLastError();
    }
    const PipeShape sh = pipe_shape(nd, false, n, di.sms);
    p.g = sh.g;
    p.n_tiled = n & ~(uint64_t)7;
    p.num_tiles = (p.n_tiled + sh.g.tile - 1) / sh.g.tile;
    p.chained = overlap_next(stream) ? 1 : 0;
    ZK_LAUNCH_BY_WARPS(rs_tma_kernel);
}

cudaError_t launch_adam(uint64_t n, const float* grad, float* master, float* m, float* v,
                        uint16_t* param_out, const AdamConsts& a, const AdamConsts* ad,
                        uint32_t* status, cudaStream_t stream) {
    AdamArgs p;
    memset(&p, 0, sizeof(p));
    p.grad = grad;
    p.master = master;
    p.m = m;
    p.v = v;
    p.param_out = param_out;
    p.status = status;
    p.n = n;
    p.vec = aligned16(grad) && aligned16(master) && aligned16(m) && aligned16(v);
    const int pv = store_vec(param_out);
    p.param_vec = pv > 8 ? 8 : pv;
    p.a = a;
    p.ad = ad;
    DevInfo di;
    cudaError_t e = dev_info(&di);
    if (e != cudaSuccess) return e;
    const uint64_t work = p.vec ? (n + 3) / 4 : n;
    return ad ? launch_ordered(adam_kernel<true>, p, plain_grid(work, di.sms), 256, stream)
              : launch_ordered(adam_kernel<false>, p, plain_grid(work, di.sms), 256, stream);
}

cudaError_t launch_scaler_prepare(const zero_scaler_state* st, const AdamConsts* table,
                                  int64_t table_len, AdamConsts* out, uint32_t* status,
                                  cudaStream_t stream) {
    scaler_prepare_kernel<<<1, 32, 0, stream>>>(st, table, table_len, out, status);
    count_launch();
    return cudaGetLastError();
}

cudaError_t launch_scaler_update(zero_scaler_state* st, const zero_scaler_params& prm,
                                 const uint32_t* status, cudaStream_t stream) {
    scaler_update_kernel<<<1, 32, 0, stream>>>(st, prm, status);
    count_launch();
    return cudaGetLastError();
}

cudaError_t launch_commit(uint64_t n, const float* master_in, const float* m_in,
                          const float* v_in, float* master_out, float* m_out, float* v_out,
                          uint16_t* param_out, uint32_t* status, cudaStream_t stream,
                          int n_replicas, uint16_t* const* replicas) {
    CommitArgs p;
    memset(&p, 0, sizeof(p));
    p.n_replicas = n_replicas;
    for (int d = 0; d < n_replicas; ++d) p.replicas[d] = replicas[d];
    p.master_in = master_in;
    p.m_in = m_in;
    p.v_in = v_in;
    p.master_out = master_out;
    p.m_out = m_out;
    p.v_out = v_out;
    p.param_out = param_out;
    p.status = status;
    p.n = n;
    DevInfo di;
    cudaError_t e = dev_info(&di);
    if (e != cudaSuccess) return e;
    return launch_ordered(commit_kernel, p, plain_grid(n, di.sms, ZK_COMMIT_BLOCKS_PER_SM), 256,
                          stream);
}

}  // namespace zk
