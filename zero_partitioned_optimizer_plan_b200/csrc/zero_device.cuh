// Device primitives and launch helpers shared by the libzero kernel files (internal).
//
// Everything here sits in an anonymous namespace: each translation unit that includes this
// header gets its own copy (its own caches of device attributes and kernel launch limits).
#pragma once

#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cstdint>
#include <cstring>

#include "zero_internal.h"

namespace zk {
namespace {

// Pipeline geometry. Per Nd the launcher picks the number of consumer warps W and how the
// shared-memory budget is split into stages from a table measured on B200 (pick_variant);
// the macros allow other geometries to be compiled and compared.
#ifndef ZK_SMEM_BUDGET
#define ZK_SMEM_BUDGET (220 * 1024)
#endif
#ifndef ZK_L2_EVICT_FIRST // streamed loads marked evict-first in L2
#define ZK_L2_EVICT_FIRST 0
#endif
#ifndef ZK_COMMIT_BLOCKS_PER_SM
#define ZK_COMMIT_BLOCKS_PER_SM 1
#endif
#ifndef ZK_ADAM_UNROLL     // float4 groups per thread and iteration of the plain owner update
#define ZK_ADAM_UNROLL 2
#endif
// Small calls take a shape with fewer consumer warps and ZK_SMALL_BUDGET bytes of stages,
// launched one CTA per SM, so that two CTAs fit on an SM and the next call's CTAs load while
// this call's finish (pick_small_variant).
#ifndef ZK_SMALL_BUDGET
#define ZK_SMALL_BUDGET (100 * 1024)
#endif


constexpr int kMaxRanks = ZERO_MAX_RANKS;
// Status bits under which a step is not applied (its commit restores the inputs).
constexpr uint32_t kStepVoid = ZERO_FLAG_OVERFLOW | ZERO_FLAG_TIMEOUT | ZERO_FLAG_BOUNDS;
constexpr int kElems = 4;                        // elements per consumer thread and tile
constexpr int kMaxStages = 8;
constexpr int kDataOffset = 128;                 // full[8] and empty[8] mbarriers first
constexpr size_t kSmemBudget = ZK_SMEM_BUDGET;   // pipeline stages per CTA
constexpr uint64_t kWaitLimitNs = 1000000000ull; // bounded waits: 1 s

template <int W>
struct Warps {
    static constexpr int kConsumerWarps = W;
    static constexpr int kConsumerThreads = W * 32;
    static constexpr int kThreads = W * 32 + 32;   // + one producer warp
    // up to 12 consumer warps (the small-call shapes), two CTAs must fit on an SM
    static constexpr int kMinBlocks = W <= 12 ? 2 : 1;
};

// Shape of the shared-memory pipeline of one launch (see "the pipeline" below).
struct Geom {
    uint32_t tile;         // T: elements per tile
    uint32_t rc;           // rank rows per stage
    uint32_t nchunks;      // stages per tile: ceil(nd / rc)
    uint32_t stage_bytes;
    uint32_t state_off;    // byte offset of the three fp32 state rows in a stage
    int stages;
};

// ---------------------------------------------------------------------------------------------
// element arithmetic
// ---------------------------------------------------------------------------------------------
__device__ __forceinline__ float h2f(uint16_t u) { return __half2float(__ushort_as_half(u)); }

__device__ __forceinline__ uint16_t f2h(float x) { return __half_as_ushort(__float2half_rn(x)); }

__device__ __forceinline__ float2 h2x2_to_f2(uint32_t u) {
    __half2 h;
    memcpy(&h, &u, 4);
    return __half22float2(h);
}

__device__ __forceinline__ float mean_of(float s, const MeanConsts& mc) {
    return mc.nd_pow2 ? __fmul_rn(s, mc.inv_nd) : __fdiv_rn(s, mc.fnd);
}

__device__ __forceinline__ bool non_finite(float x) {
    return (__float_as_uint(x) & 0x7f800000u) == 0x7f800000u;
}

// Adam on one element from its reduced (still loss-scaled) gradient; w, m, v updated in place.
__device__ __forceinline__ void adam_elem(float red, float& w, float& m, float& v,
                                          const AdamConsts& a) {
    const float g = a.loss_scale_pow2 ? __fmul_rn(red, a.inv_loss_scale)
                                      : __fdiv_rn(red, a.loss_scale);
    const float mt = __fadd_rn(__fmul_rn(a.beta1, m), __fmul_rn(a.one_minus_beta1, g));
    const float vt =
        __fadd_rn(__fmul_rn(a.beta2, v), __fmul_rn(a.one_minus_beta2, __fmul_rn(g, g)));
    const float denom = __fadd_rn(__fdiv_rn(__fsqrt_rn(vt), a.bias2_sqrt), a.eps);
    const float delta = __fmul_rn(a.step_size, __fdiv_rn(mt, denom));
    w = __fsub_rn(w, delta);
    m = mt;
    v = vt;
}

// The step's constants. kDC = false: straight from the kernel parameters (operands from the
// constant bank, no registers held); kDC = true: loaded once from device memory, for launches
// captured in a CUDA graph and replayed with other constants.
#define ZK_STEP_CONSTS(p, a)             \
    AdamConsts a##_dev;                  \
    if constexpr (kDC) a##_dev = *(p).ad; \
    const AdamConsts& a = kDC ? a##_dev : (p).a

// ---------------------------------------------------------------------------------------------
// mbarrier and bulk-copy primitives (PTX)
// ---------------------------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_addr(const void* p) {
    return (uint32_t)__cvta_generic_to_shared(p);
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count)
                 : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)),
                 "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(done)
        : "r"(smem_addr(bar)), "r"(parity)
        : "memory");
    return done != 0;
}

// ---------------------------------------------------------------------------------------------
// programmatic dependent launch
//
// The pipeline kernels are launched with programmatic stream serialization allowed, so that a
// kernel's CTAs can be scheduled while the kernel before it on the stream drains.
//   ordered (default): wait for the previous kernel to complete and its writes to be visible,
//     before the first global-memory access; then let the next kernel be scheduled. Stream
//     order is kept exactly.
//   chained (a later call of a zero_overlap_begin/end region, which the caller declares
//     independent of the region's other calls): let the next kernel be scheduled at once, run,
//     and wait for the previous kernel only before exiting. A kernel therefore completes only
//     after every kernel before it, and the first ordinary launch after the region sees all of
//     the region's writes.
// Without the launch attribute both instructions are no-ops.
// ---------------------------------------------------------------------------------------------
__device__ __forceinline__ void pdl_enter(int chained) {
    if (!chained) asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

__device__ __forceinline__ void pdl_leave(int chained) {
    if (chained) asm volatile("griddepcontrol.wait;" ::: "memory");
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// Wait for the phase with the given parity to complete; false after kWaitLimitNs.
__device__ __noinline__ bool mbar_wait(uint64_t* bar, uint32_t parity) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    for (uint32_t i = 1;; ++i) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((i & 63u) == 0 && globaltimer_ns() - t0 > kWaitLimitNs) return false;
    }
}

// 1-D bulk copy global -> this CTA's shared memory, completion counted on `bar` in bytes.
// Both addresses 16-byte aligned, bytes a multiple of 16.
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes,
                                         uint64_t* bar) {
#if ZK_L2_EVICT_FIRST
    uint64_t pol;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1], %2, [%3], %4;"
        ::"r"(smem_addr(dst)), "l"(src), "r"(bytes), "r"(smem_addr(bar)), "l"(pol)
        : "memory");
#else
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
        ::"r"(smem_addr(dst)), "l"(src), "r"(bytes), "r"(smem_addr(bar))
        : "memory");
#endif
}

// ---------------------------------------------------------------------------------------------
// vector helpers
// ---------------------------------------------------------------------------------------------
template <int E>
__device__ __forceinline__ void lds_f16(const uint8_t* p, float (&x)[E]) {
    if constexpr (E == 8) {
        const uint4 q = *reinterpret_cast<const uint4*>(p);
        float2 a = h2x2_to_f2(q.x), b = h2x2_to_f2(q.y), c = h2x2_to_f2(q.z), d = h2x2_to_f2(q.w);
        x[0] = a.x; x[1] = a.y; x[2] = b.x; x[3] = b.y;
        x[4] = c.x; x[5] = c.y; x[6] = d.x; x[7] = d.y;
    } else if constexpr (E == 4) {
        const uint2 q = *reinterpret_cast<const uint2*>(p);
        float2 a = h2x2_to_f2(q.x), b = h2x2_to_f2(q.y);
        x[0] = a.x; x[1] = a.y; x[2] = b.x; x[3] = b.y;
    } else {
        static_assert(E == 2, "E");
        const float2 a = h2x2_to_f2(*reinterpret_cast<const uint32_t*>(p));
        x[0] = a.x; x[1] = a.y;
    }
}

template <int E>
__device__ __forceinline__ void lds_f32(const uint8_t* p, float (&x)[E]) {
    if constexpr (E == 8) {
        const float4 a = reinterpret_cast<const float4*>(p)[0];
        const float4 b = reinterpret_cast<const float4*>(p)[1];
        x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w;
        x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
    } else if constexpr (E == 4) {
        const float4 a = *reinterpret_cast<const float4*>(p);
        x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w;
    } else {
        const float2 a = *reinterpret_cast<const float2*>(p);
        x[0] = a.x; x[1] = a.y;
    }
}

// Store E floats to global memory whose address is a multiple of 4*E bytes (E <= 4 needs
// 4*E-byte alignment, E == 8 needs 16). Streaming (evict-first) stores.
template <int E>
__device__ __forceinline__ void stg_f32(float* p, const float (&x)[E]) {
    if constexpr (E == 8) {
        __stcs(reinterpret_cast<float4*>(p), make_float4(x[0], x[1], x[2], x[3]));
        __stcs(reinterpret_cast<float4*>(p) + 1, make_float4(x[4], x[5], x[6], x[7]));
    } else if constexpr (E == 4) {
        __stcs(reinterpret_cast<float4*>(p), make_float4(x[0], x[1], x[2], x[3]));
    } else {
        __stcs(reinterpret_cast<float2*>(p), make_float2(x[0], x[1]));
    }
}

// Store E floats at any 4-byte aligned address, with the widest stores the address allows.
template <int E>
__device__ __forceinline__ void stg_f32_any(float* p, const float (&x)[E]) {
    const uintptr_t a = reinterpret_cast<uintptr_t>(p);
    if ((a & 15u) == 0 && (E % 4) == 0) {
#pragma unroll
        for (int j = 0; j < E; j += 4)
            __stcs(reinterpret_cast<float4*>(p + j), make_float4(x[j], x[j + 1], x[j + 2], x[j + 3]));
    } else if ((a & 7u) == 0) {
#pragma unroll
        for (int j = 0; j < E; j += 2) __stcs(reinterpret_cast<float2*>(p + j), make_float2(x[j], x[j + 1]));
    } else {
#pragma unroll
        for (int j = 0; j < E; ++j) __stcs(p + j, x[j]);
    }
}

// Store E fp16 values (given as floats, rounded here) with stores of at most `vec` bytes;
// `vec` is the widest store the destination's alignment allows.
template <int E>
__device__ __forceinline__ void stg_f16(uint16_t* p, const float (&x)[E], int vec) {
    constexpr int H = E / 2;
    uint32_t h[H];
#pragma unroll
    for (int j = 0; j < H; ++j)
        h[j] = (uint32_t)f2h(x[2 * j]) | ((uint32_t)f2h(x[2 * j + 1]) << 16);
    if constexpr (E == 8) {
        if (vec >= 16) {
            __stcs(reinterpret_cast<uint4*>(p), make_uint4(h[0], h[1], h[2], h[3]));
            return;
        }
    }
    if constexpr (E >= 4) {
        if (vec >= 8) {
#pragma unroll
            for (int j = 0; j < H; j += 2)
                __stcs(reinterpret_cast<uint2*>(p + 2 * j), make_uint2(h[j], h[j + 1]));
            return;
        }
    }
    if (vec >= 4) {
#pragma unroll
        for (int j = 0; j < H; ++j) __stcs(reinterpret_cast<unsigned int*>(p + 2 * j), h[j]);
        return;
    }
#pragma unroll
    for (int j = 0; j < H; ++j) {
        __stcs(reinterpret_cast<unsigned short*>(p + 2 * j), (unsigned short)(h[j] & 0xffffu));
        __stcs(reinterpret_cast<unsigned short*>(p + 2 * j + 1), (unsigned short)(h[j] >> 16));
    }
}

__device__ __forceinline__ void flag_overflow(bool bad, uint32_t* status) {
    const unsigned any = __ballot_sync(0xffffffffu, bad);
    if (any && (threadIdx.x & 31) == 0) atomicOr(status, ZERO_FLAG_OVERFLOW);
}

// ---------------------------------------------------------------------------------------------
// pipeline pieces shared by the bulk-copy kernels
// ---------------------------------------------------------------------------------------------
struct TileSpan {
    uint64_t base;   // first element of the tile
    uint32_t cnt;    // elements in the tile (a multiple of 8)
};

__device__ __forceinline__ TileSpan tile_span(uint64_t tile, uint32_t T, uint64_t n_tiled) {
    TileSpan t;
    t.base = tile * T;
    const uint64_t left = n_tiled - t.base;
    t.cnt = left < T ? (uint32_t)left : T;
    return t;
}

__device__ __forceinline__ void init_barriers(uint64_t* full, uint64_t* empty, int stages,
                                              int consumer_warps) {
    if (threadIdx.x == 0) {
        for (int s = 0; s < stages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], (uint32_t)consumer_warps);
        }
        fence_mbar_init();
    }
    __syncthreads();
}

// Consumer side of one stage: wait for it, add its rank rows into acc (rank order), optionally
// read the state rows, then release the stage. Returns false if the wait timed out. kTile is the
// tile length, known at compile time from the kernel's warps and values per thread (= g.tile):
// the rank rows sit at a constant stride, so the unrolled loads take immediate offsets
// (measured: Nd = 2 0.960 -> 0.980, Nd = 64 1.043 -> 1.061 of the peak against a runtime stride).
template <int E, bool kState, uint32_t kTile>
__device__ __forceinline__ bool consume_stage(const Geom& g, int nd, uint64_t* full,
                                              uint64_t* empty, const uint8_t* data, uint32_t it,
                                              uint32_t c, uint32_t e0, bool active,
                                              float (&acc)[E], float (&w)[E], float (&m)[E],
                                              float (&v)[E]) {
    const uint32_t s = it % g.stages;
    const uint32_t use = it / g.stages;
    if (!__all_sync(0xffffffffu, mbar_wait(&full[s], use & 1u))) return false;
    const uint8_t* st = data + (size_t)s * g.stage_bytes;
    static_assert(kTile > 0, "tile length");
    const uint32_t T = kTile;
    if (active) {
        const uint32_t nr = min(g.rc, (uint32_t)nd - c * g.rc);
        const uint8_t* row = st + (size_t)e0 * 2u;
#pragma unroll 4
        for (uint32_t r = 0; r < nr; ++r) {
            float x[E];
            lds_f16<E>(row + (size_t)r * T * 2u, x);
#pragma unroll
            for (int j = 0; j < E; ++j) acc[j] = __fadd_rn(acc[j], x[j]);
        }
        if (kState && c + 1 == g.nchunks) {
            const uint8_t* sf = st + g.state_off + (size_t)e0 * 4u;
            lds_f32<E>(sf, w);
            lds_f32<E>(sf + (size_t)T * 4u, m);
            lds_f32<E>(sf + (size_t)T * 8u, v);
        }
    }
    __syncwarp();
    if ((threadIdx.x & 31) == 0) mbar_arrive(&empty[s]);   // stage s may be refilled
    return true;
}

// ---------------------------------------------------------------------------------------------
// host side: device attributes, launch limits, grids
// ---------------------------------------------------------------------------------------------
// Nothing on the launch path takes a lock: the per-device attributes live in a fixed array of
// atomics (a racing first call on two threads computes the same value twice), and the
// occupancy of each (device, kernel, shared memory, threads) in a small per-thread table.
constexpr int kMaxDevices = 64;

struct DevInfo {
    int sms = 0;
    int dev = 0;
};

cudaError_t dev_info(DevInfo* out) {
    static std::atomic<int> sms_of[kMaxDevices];   // 0: not known yet
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    int sms = sms_of[dev].load(std::memory_order_relaxed);
    if (sms == 0) {
        e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        if (e != cudaSuccess) return e;
        sms_of[dev].store(sms, std::memory_order_relaxed);
    }
    out->sms = sms;
    out->dev = dev;
    return cudaSuccess;
}

// Resident CTAs per SM of a pipeline kernel with `smem` dynamic bytes and `threads` threads on
// device `dev`. The first time a host thread meets a (device, kernel) pair, the kernel's
// dynamic shared-memory limit is raised to the device's opt-in maximum (setting it again from
// another thread is harmless), so that every launch size (they differ with Nd) stays allowed.
template <typename K>
cudaError_t pipe_blocks_per_sm(K kernel, int dev, int threads, size_t smem, int* out) {
    struct Entry {
        const void* kernel;
        size_t smem;
        int dev, threads, blocks;
    };
    constexpr int kSlots = 64;
    thread_local Entry cache[kSlots];
    thread_local int used = 0;
    const void* kp = reinterpret_cast<const void*>(kernel);
    for (int i = 0; i < used; ++i) {
        const Entry& c = cache[i];
        if (c.kernel == kp && c.smem == smem && c.dev == dev && c.threads == threads) {
            *out = c.blocks;
            return cudaSuccess;
        }
    }
    int optin = 0;
    cudaError_t e = cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, optin);
    if (e != cudaSuccess) return e;
    if (smem > (size_t)optin) return cudaErrorInvalidValue;
    int b = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&b, kernel, threads, smem);
    if (e != cudaSuccess) return e;
    if (b < 1) return cudaErrorInvalidConfiguration;
    if (used < kSlots) cache[used++] = Entry{kp, smem, dev, threads, b};
    *out = b;
    return cudaSuccess;
}

struct PipeShape {
    Geom g;
    size_t smem;
    int warps;        // consumer warps
    int grid_per_sm;  // CTAs per SM in the grid (0: as many as fit)
};

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int store_vec(const void* p) {
    const uintptr_t a = reinterpret_cast<uintptr_t>(p);
    return (a & 15u) == 0 ? 16 : (a & 7u) == 0 ? 8 : (a & 3u) == 0 ? 4 : 2;
}

constexpr uint64_t kMinTiledElems = 4096;

template <typename K, typename A>
cudaError_t launch_pipe(K kernel, const A& args, const PipeShape& sh, cudaStream_t stream) {
    DevInfo di;
    cudaError_t e = dev_info(&di);
    if (e != cudaSuccess) return e;
    const int threads = 32 * sh.warps + 32;
    int bps = 1;
    e = pipe_blocks_per_sm(kernel, di.dev, threads, sh.smem, &bps);
    if (e != cudaSuccess) return e;
    if (sh.grid_per_sm > 0 && sh.grid_per_sm < bps) bps = sh.grid_per_sm;
    uint64_t grid = (uint64_t)di.sms * (uint64_t)bps;
    if (args.num_tiles < grid) grid = args.num_tiles;
    if (grid < 1) grid = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3((unsigned)threads);
    cfg.dynamicSmemBytes = sh.smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, kernel, args);
    count_launch();
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

// An ordered launch that may become resident before the previous kernel on the stream ends
// (the kernel waits for it with griddepcontrol.wait before touching memory).
template <typename K, typename A>
cudaError_t launch_ordered(K kernel, const A& args, unsigned grid, unsigned threads,
                           cudaStream_t stream) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(threads);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, args);
    count_launch();
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

unsigned plain_grid(uint64_t n, int sms, int per_sm = 8) {
    uint64_t blocks = (n + 255) / 256;
    const uint64_t cap = (uint64_t)sms * (uint64_t)per_sm;
    if (blocks > cap) blocks = cap;
    return (unsigned)(blocks ? blocks : 1);
}

// Consumer warps and stage split per Nd, measured on B200 (HBM GB/s of the fused step over
// geometries with 4 elements per thread): few ranks need more warps to hide the latency of the
// Adam arithmetic; many ranks need large stages so that a tile takes few chunks.
struct Variant {
    int warps;
    int target_stages;
};

Variant pick_variant(int nd) {
    if (nd <= 2) {
        Variant v{20, 2};
#ifdef ZK_ND2_WARPS
        v.warps = ZK_ND2_WARPS;
#endif
#ifdef ZK_ND2_STAGES
        v.target_stages = ZK_ND2_STAGES;
#endif
        return v;
    }
    if (nd <= 4) return {16, 2};
    if (nd <= 8) return {24, 3};
    if (nd <= 16) return {16, 2};
    return {20, 2};
}

// The small-call shape, also measured on B200 (graph-captured chains of 1 MiB and 16 MiB
// bucket calls in an overlap region): 12 consumer warps up to Nd = 8, 8 above; a call takes it
// when the large shape would give each SM fewer than `max_tiles_per_sm` tiles (at Nd <= 2 the
// ramp and tail of a launch weigh more, so calls up to 32 tiles per SM gain from it).
struct SmallVariant {
    int warps;
    int max_tiles_per_sm;
};

SmallVariant pick_small_variant(int nd) {
    SmallVariant v{nd <= 8 ? 12 : 8, nd <= 2 ? 32 : 4};
#ifdef ZK_SMALL_WARPS
    v.warps = ZK_SMALL_WARPS;
#endif
#ifdef ZK_SMALL_TILES_PER_SM
    v.max_tiles_per_sm = ZK_SMALL_TILES_PER_SM;
#endif
    return v;
}

}  // namespace
}  // namespace zk
