// Compressed reduce-scatter payload for sm_100a: int8 values with one fp32 scale per block of
// 128 elements ("ZeRO" (lastdictionary.com), main definition: extensions compress the
// communication, ZeRO++; the pages give no format, this is the library's).
//
//   quantize (each sending rank, on its own slice):
//     amax  = max |x| over the block (any inf/NaN poisons the block: scale NaN, q 0)
//     scale = amax / 127                      (IEEE binary32 division)
//     q     = round_half_even(x / scale), clamped to [-127, 127]; 0 when scale is 0
//     stored as the byte q + 128 (offset binary, 1..255)
//   owner's fused step:
//     s = fma(float(q_r), scale_r, s) for r = 0..nd-1 (one rounding each), red = s / nd,
//     then the same unscale, Adam, fp16 cast and write-back as the fp16 fused step.
//
// Layout: a rank's payload is an array of 132-byte records, one per block: the block's 128 value
// bytes, then its fp32 scale (a short last block is padded to a full record with the byte of
// q = 0). A tile of a
// multiple of 512 elements is then one contiguous, 16-byte-aligned run of records per rank:
// one bulk copy per rank and tile.
//
// Per parameter the owner reads nd * 132/128 payload bytes instead of 2 * nd: at Nd = 64 the
// fused step moves 92 bytes per parameter instead of 154. Per element and rank it issues a byte
// conversion (the mantissa-placement trick: a byte permute, then the bias removal) and a fused
// multiply-add, the float halves of both as packed two-wide fp32 instructions. The offset-binary
// byte is what the conversion places directly: a signed byte would need one more instruction per
// four values (a sign-bit flip), which at Nd = 64 cost about 2 % of the step.
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <cstring>

#include "zero_device.cuh"
#include "zero_internal.h"

namespace zk {

namespace {

constexpr int kQB = 128;                 // elements per scale block
constexpr int kRec = 132;                // bytes per record: 128 int8 values, one fp32 scale
constexpr uint64_t kQTileAlign = 512;    // tiles cover a multiple of 512 elements (528-byte runs)

struct QuantArgs {
    const uint16_t* g;
    uint8_t* rec;        // ceil(n/128) records (4-byte aligned: the API checks it)
    uint64_t n;
    int gvec;            // g 16-byte aligned: a thread's 8 values in one load
};

// Packed pairs of binary32 values (sm_100 executes two-wide fp32 add, multiply and fused
// multiply-add as one instruction; each half is an ordinary IEEE operation rounded to nearest
// even).
__device__ __forceinline__ uint64_t f2_pack(float a, float b) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
    return r;
}

__device__ __forceinline__ void f2_unpack(uint64_t r, float& a, float& b) {
    asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(r));
}

__device__ __forceinline__ uint64_t f2_add(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}

__device__ __forceinline__ uint64_t f2_sub(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}

__device__ __forceinline__ uint64_t f2_mul(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}

__device__ __forceinline__ uint64_t f2_fma(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}

// Thread h of a block's 128/V threads: the block's fp16 values V*h .. V*h+V-1 (V/8 16-byte
// loads), missing elements as +0.
template <int V>
__device__ __forceinline__ void quant_load(const QuantArgs& p, uint64_t b, int hl,
                                           uint4 (&u)[V / 8]) {
    const uint64_t i0 = b * kQB + (uint64_t)hl * V;
    if (p.gvec && i0 + V <= p.n) {
        const uint4* src = reinterpret_cast<const uint4*>(p.g + i0);
#pragma unroll
        for (int k = 0; k < V / 8; ++k) u[k] = src[k];
        return;
    }
    uint32_t h[V / 2];
#pragma unroll
    for (int j = 0; j < V / 2; ++j) {
        const uint32_t lo = i0 + 2 * j < p.n ? p.g[i0 + 2 * j] : 0u;
        const uint32_t hi = i0 + 2 * j + 1 < p.n ? p.g[i0 + 2 * j + 1] : 0u;
        h[j] = lo | hi << 16;
    }
#pragma unroll
    for (int k = 0; k < V / 8; ++k)
        u[k] = make_uint4(h[4 * k], h[4 * k + 1], h[4 * k + 2], h[4 * k + 3]);
}

// 1.5 * 2^23 + 128: y + kRintBias, for |y| < 2^21, rounds y to the nearest integer (ties to even,
// 128 being even) and leaves k + 128 in the sum's low mantissa byte.
constexpr float kRintBias = 12583040.0f;
// |y - k| at or above this (y within 2^-14 of a half-integer) takes the exact division.
constexpr float kTieGuard = 0.5f - 0x1p-14f;

// Byte q + 128 of four values, q = the integer nearest x / scale (ties to even), from
// y = x * fl(1/scale). |x / scale| <= 127 * (1 + 2^-23), so |y - x / scale| < 2^-16 (two
// roundings, relative 2^-24 each) and fl(x / scale) is within 2^-18 of x / scale: where y lies
// farther than 2^-15 from every half-integer, y and fl(x / scale) round to the same integer,
// so below the guard the reciprocal gives the IEEE quotient's q; at or above it the caller
// redoes the four values by division. |q| <= 127 needs no clamp: the quotient stays below 127.5.
__device__ __forceinline__ uint32_t quant_word(uint32_t h01, uint32_t h23, uint64_t rr,
                                               bool& near) {
    const float2 a = h2x2_to_f2(h01), b = h2x2_to_f2(h23);
    const uint64_t bias = f2_pack(kRintBias, kRintBias);
    const uint64_t y01 = f2_mul(f2_pack(a.x, a.y), rr), y23 = f2_mul(f2_pack(b.x, b.y), rr);
    const uint64_t c01 = f2_add(y01, bias), c23 = f2_add(y23, bias);
    // y - k, exact (k within 1/2 of y)
    const uint64_t t01 = f2_sub(y01, f2_sub(c01, bias)), t23 = f2_sub(y23, f2_sub(c23, bias));
    float t0, t1, t2, t3, c0, c1, c2, c3;
    f2_unpack(t01, t0, t1);
    f2_unpack(t23, t2, t3);
    f2_unpack(c01, c0, c1);
    f2_unpack(c23, c2, c3);
    near |= fabsf(t0) >= kTieGuard || fabsf(t1) >= kTieGuard || fabsf(t2) >= kTieGuard ||
            fabsf(t3) >= kTieGuard;
    const uint32_t lo = __byte_perm(__float_as_uint(c0), __float_as_uint(c1), 0x0040u);
    const uint32_t hi = __byte_perm(__float_as_uint(c2), __float_as_uint(c3), 0x0040u);
    return __byte_perm(lo, hi, 0x5410u);
}

// The same byte by IEEE division (the definition), for a thread with a value near a tie.
__device__ __forceinline__ uint32_t quant_word_div(uint32_t h01, uint32_t h23, float scale) {
    const float2 a = h2x2_to_f2(h01), b = h2x2_to_f2(h23);
    const float x[4] = {a.x, a.y, b.x, b.y};
    uint32_t w = 0;
#pragma unroll
    for (int j = 0; j < 4; ++j)
        w |= (uint32_t)(__float2int_rn(__fdiv_rn(x[j], scale)) + 128) << (8 * j);
    return w;
}

// V values per thread, 128/V threads per block of 128: a warp takes V/4 consecutive blocks per
// iteration and has the next iteration's loads in flight; the block's scale, its reciprocal and
// the reductions are paid once per V values. The block's max |x| is an integer max over the
// fp16 magnitude bits (ordered like the magnitudes, inf and NaN above every finite value), so a
// poisoned block is one compare.
template <int V>
__global__ void __launch_bounds__(256) quant_q8_kernel(const __grid_constant__ QuantArgs p) {
    static_assert(V == 8 || V == 16 || V == 32, "values per thread");
    pdl_enter(0);   // ordered after the kernels before it (see launch_ordered)
    constexpr int kTpb = kQB / V;      // threads per block of 128
    constexpr int kBpw = 32 / kTpb;    // blocks per warp and iteration
    const int lane = threadIdx.x & 31;
    const int part = lane / kTpb;
    const int hl = lane % kTpb;
    const uint64_t nblocks = (p.n + kQB - 1) / kQB;
    const uint64_t ngroups = (nblocks + kBpw - 1) / kBpw;
    const uint64_t nwarps = ((uint64_t)gridDim.x * blockDim.x) >> 5;
    uint64_t pg = ((uint64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    uint4 nx[V / 8];
#pragma unroll
    for (int k = 0; k < V / 8; ++k) nx[k] = make_uint4(0u, 0u, 0u, 0u);
    if (pg < ngroups) quant_load<V>(p, kBpw * pg + (uint64_t)part, hl, nx);
    for (; pg < ngroups; pg += nwarps) {
        const uint64_t b = kBpw * pg + (uint64_t)part;
        uint4 u[V / 8];
#pragma unroll
        for (int k = 0; k < V / 8; ++k) u[k] = nx[k];
        if (pg + nwarps < ngroups) quant_load<V>(p, b + kBpw * nwarps, hl, nx);
        const bool exists = b < nblocks;
        uint32_t mag = 0u;
#pragma unroll
        for (int k = 0; k < V / 8; ++k)
            mag = __vmaxu2(mag, __vmaxu2(__vmaxu2(u[k].x & 0x7fff7fffu, u[k].y & 0x7fff7fffu),
                                         __vmaxu2(u[k].z & 0x7fff7fffu, u[k].w & 0x7fff7fffu)));
        mag = max(mag & 0xffffu, mag >> 16);
        // reductions inside each block's group of lanes (xor offsets below kTpb stay in it)
#pragma unroll
        for (int o = kTpb / 2; o > 0; o >>= 1)
            mag = max(mag, __shfl_xor_sync(0xffffffffu, mag, o));
        const bool bad = mag >= 0x7c00u;
        const float scale = bad ? __uint_as_float(0x7fc00000u)
                                : __fdiv_rn(h2f((uint16_t)mag), 127.0f);
        uint32_t w[V / 4];
#pragma unroll
        for (int k = 0; k < V / 4; ++k) w[k] = 0x80808080u;   // q = 0
        if (!bad && scale != 0.0f) {
            const float r = __frcp_rn(scale);
            const uint64_t rr = f2_pack(r, r);
            bool near = false;
#pragma unroll
            for (int k = 0; k < V / 8; ++k) {
                w[2 * k] = quant_word(u[k].x, u[k].y, rr, near);
                w[2 * k + 1] = quant_word(u[k].z, u[k].w, rr, near);
            }
            if (near) {
#pragma unroll
                for (int k = 0; k < V / 8; ++k) {
                    w[2 * k] = quant_word_div(u[k].x, u[k].y, scale);
                    w[2 * k + 1] = quant_word_div(u[k].z, u[k].w, scale);
                }
            }
        }
        if (exists) {   // records are 4-byte aligned (132 = 4 * 33), V * hl too
            uint8_t* rec = p.rec + b * kRec;
            uint32_t* dst = reinterpret_cast<uint32_t*>(rec + hl * V);
#pragma unroll
            for (int k = 0; k < V / 4; ++k) dst[k] = w[k];
            if (hl == 0) *reinterpret_cast<float*>(rec + kQB) = scale;
        }
    }
}

// Values per thread of the quantizer, measured on B200 (the senders' side of the int8 lines,
// flat 2^28 / the 7.5B view, two passes): 8 values 0.62 / 0.66 of the peak, 16 values 0.77 /
// 0.82, 32 values 0.60 / 0.64 (96 registers: half the resident warps).
constexpr int kQuantVals = 16;

struct FusedQ8Args {
    const uint8_t* rec[kMaxRanks];   // each rank's records for this range
    const float* master_in;
    const float* m_in;
    const float* v_in;
    float* master_out;
    float* m_out;
    float* v_out;
    uint16_t* param_out;
    uint32_t* status;
    uint64_t n;
    uint64_t n_tiled;    // multiple of 512
    uint64_t num_tiles;
    Geom g;              // rank rows: rc runs of T/128 records (T*132/128 bytes each)
    uint32_t row;        // bytes of one rank's run in a stage
    int nd;
    int param_vec;
    AdamConsts a;
    const AdamConsts* ad;  // when not null: the constants, read from device memory at run time
    MeanConsts mc;
    int chained;         // programmatic launch chained to the previous call (see pdl_enter)
};

// acc + float(q) * scale with one rounding, from the stored byte q + 128
__device__ __forceinline__ float dequant_add(uint8_t code, float scale, float acc) {
    return __fmaf_rn(__int2float_rn((int)code - 128), scale, acc);
}

// Byte j of `biased` (q + 128, in 1..255) placed in the low mantissa bits of 2^23 gives the
// float 2^23 + q + 128; subtracting 2^23 + 128 leaves q exactly. Full-rate instructions instead
// of an integer-to-float conversion (a quarter-rate pipe), which otherwise bounds the owner's
// step at large Nd.
__device__ __forceinline__ float q_placed(uint32_t biased, int j) {
    return __uint_as_float(__byte_perm(biased, 0x4B000000u, 0x7440u | (uint32_t)j));
}

__device__ __forceinline__ void fused_q8_element(const FusedQ8Args& p, const AdamConsts& a,
                                                 uint64_t i, bool& bad) {
    if (i >= p.n) {
        atomicOr(p.status, ZERO_FLAG_BOUNDS);
        return;
    }
    float s = 0.0f;
    const uint64_t off = (i / kQB) * kRec;
    for (int r = 0; r < p.nd; ++r) {
        const uint8_t* rec = p.rec[r] + off;
        s = dequant_add(rec[i % kQB], *reinterpret_cast<const float*>(rec + kQB), s);
    }
    const float red = mean_of(s, p.mc);
    bad |= non_finite(red);
    float w = p.master_in[i], m = p.m_in[i], v = p.v_in[i];
    adam_elem(red, w, m, v, a);
    p.master_out[i] = w;
    p.m_out[i] = m;
    p.v_out[i] = v;
    p.param_out[i] = f2h(w);
}

__device__ __forceinline__ const float* q8_state_row(const FusedQ8Args& p, uint32_t k) {
    return k == 0 ? p.master_in : (k == 1 ? p.m_in : p.v_in);
}

// Producer warp: lane 0 posts the byte count, all lanes issue the row copies.
__device__ void produce_q8(const FusedQ8Args& p, uint64_t* full, uint64_t* empty, uint8_t* data) {
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
                bool w = true;
                if (lane == 0) w = mbar_wait(&empty[s], (use - 1) & 1u);
                if (!__shfl_sync(0xffffffffu, w, 0)) {
                    ok = false;
                    break;
                }
            }
            const uint32_t r0 = c * g.rc;
            const uint32_t nr = min(g.rc, (uint32_t)p.nd - r0);
            const bool with_state = c + 1 == g.nchunks;
            const uint32_t rb = ts.cnt / kQB * kRec, fb = ts.cnt * 4u;
            uint8_t* st = data + (size_t)s * g.stage_bytes;
            const bool sane = ts.base < p.n_tiled && (ts.cnt % kQTileAlign) == 0 && ts.cnt > 0 &&
                              r0 < (uint32_t)p.nd && nr <= g.rc && s < (uint32_t)g.stages;
            if (lane == 0) {
                if (!sane) atomicOr(p.status, ZERO_FLAG_BOUNDS);
                mbar_arrive_expect_tx(&full[s], sane ? nr * rb + (with_state ? 3u * fb : 0u) : 0u);
            }
            __syncwarp();
            if (!sane) continue;
            const uint32_t ncopy = nr + (with_state ? 3u : 0u);
            for (uint32_t j = (uint32_t)lane; j < ncopy; j += 32u) {
                if (j < nr) {
                    bulk_g2s(st + (size_t)j * p.row, p.rec[r0 + j] + ts.base / kQB * kRec, rb,
                             &full[s]);
                } else {
                    const uint32_t k = j - nr;
                    bulk_g2s(st + g.state_off + (size_t)k * T * 4u, q8_state_row(p, k) + ts.base,
                             fb, &full[s]);
                }
            }
        }
    }
    if (!ok && lane == 0) {
        atomicOr(p.status, ZERO_FLAG_TIMEOUT);
        for (uint32_t s = 0; s < (uint32_t)g.stages && s < it; ++s) {
            const uint32_t last = s + ((it - 1u - s) / (uint32_t)g.stages) * (uint32_t)g.stages;
            (void)mbar_wait(&full[s], (last / (uint32_t)g.stages) & 1u);
        }
    }
}

// Rank r's contribution to a thread's E accumulators (packed pairs ap): its record's scale and
// E bytes q + 128, converted by mantissa placement, added by fused multiply-adds.
template <int E>
__device__ __forceinline__ void q8_rank_fma(const uint8_t* rec, uint32_t e_in_rec,
                                            uint64_t (&ap)[E / 2]) {
    const uint64_t nbias = f2_pack(-8388736.0f, -8388736.0f);   // -(2^23 + 128)
    const float sc = *reinterpret_cast<const float*>(rec + kQB);
    const uint64_t ss = f2_pack(sc, sc);
#pragma unroll
    for (int k4 = 0; k4 < E / 4; ++k4) {
        const uint32_t biased =   // four bytes, each q + 128
            *reinterpret_cast<const uint32_t*>(rec + e_in_rec + 4 * k4);
        const uint64_t q01 = f2_add(f2_pack(q_placed(biased, 0), q_placed(biased, 1)), nbias);
        const uint64_t q23 = f2_add(f2_pack(q_placed(biased, 2), q_placed(biased, 3)), nbias);
        // acc + q * scale, one rounding each
        ap[2 * k4] = f2_fma(q01, ss, ap[2 * k4]);
        ap[2 * k4 + 1] = f2_fma(q23, ss, ap[2 * k4 + 1]);
    }
}

// kFixedRow: the rank loop steps from one rank's records to the next by the compile-time kRow
// (immediate load offsets) or by the launch's p.row (the same value, at run time); which is
// faster depends on Nd (see pick_variant_q8). kRC > 0: a chunk of exactly kRC ranks runs fully
// unrolled (no loop counter, every record at an immediate offset); a chunk of another length
// takes the general loop.
template <int W, int E, bool kDC, bool kFixedRow, int kRC = 0>
__global__ void __launch_bounds__(Warps<W>::kThreads, Warps<W>::kMinBlocks)
    fused_q8_tma_kernel(const __grid_constant__ FusedQ8Args p) {
    static_assert(E == 4 || E == 8, "a thread's values sit in one record");
    // bytes of one rank's run of records in a stage (the launcher's p.row, checked below)
    constexpr uint32_t kRow = (32u * W * E / kQB) * kRec;
    const uint32_t row = kFixedRow ? kRow : p.row;
    extern __shared__ __align__(128) uint8_t smem[];
    uint64_t* full = reinterpret_cast<uint64_t*>(smem);
    uint64_t* empty = full + kMaxStages;
    uint8_t* data = smem + kDataOffset;
    init_barriers(full, empty, p.g.stages, W);
    pdl_enter(p.chained);
    if ((threadIdx.x >> 5) == W) {
        produce_q8(p, full, empty, data);
        pdl_leave(p.chained);
        return;
    }
    ZK_STEP_CONSTS(p, a);
    const int lane = threadIdx.x & 31;
    const uint32_t T = p.g.tile;
    const uint32_t e0 = (uint32_t)threadIdx.x * E;
    bool bad = false;
    uint32_t it = 0;
    bool ok = p.row == kRow && T == 32u * W * E;   // self-check of the launch's shape
    if (!ok && threadIdx.x == 0) atomicOr(p.status, ZERO_FLAG_BOUNDS);
    for (uint64_t tile = blockIdx.x; ok && tile < p.num_tiles; tile += gridDim.x) {
        const TileSpan ts = tile_span(tile, T, p.n_tiled);
        const bool active = e0 < ts.cnt;
        float acc[E], w[E], m[E], v[E];
#pragma unroll
        for (int j = 0; j < E; ++j) acc[j] = 0.0f;
        for (uint32_t c = 0; c < p.g.nchunks; ++c, ++it) {
            const uint32_t s = it % p.g.stages;
            const uint32_t use = it / p.g.stages;
            if (!__all_sync(0xffffffffu, mbar_wait(&full[s], use & 1u))) {
                if (lane == 0) atomicOr(p.status, ZERO_FLAG_TIMEOUT);
                ok = false;
                break;
            }
            const uint8_t* st = data + (size_t)s * p.g.stage_bytes;
            if (active) {
                const uint32_t nr = min(p.g.rc, (uint32_t)p.nd - c * p.g.rc);
                // this thread's record in each rank's run; its E values share the scale
                const uint8_t* rec0 = st + (size_t)(e0 / kQB) * kRec;
                // the E accumulators as E/2 packed pairs: per rank and four values, one
                // 4-byte load (records are 4-byte aligned), two packed bias removals and two
                // packed fused multiply-adds
                constexpr int P = E / 2;
                uint64_t ap[P];
#pragma unroll
                for (int k = 0; k < P; ++k) ap[k] = f2_pack(acc[2 * k], acc[2 * k + 1]);
                // rank r's record sits `row` bytes after rank r-1's
                if (kRC > 0 && nr == (uint32_t)kRC) {
#pragma unroll
                    for (int r = 0; r < kRC; ++r)
                        q8_rank_fma<E>(rec0 + (size_t)r * kRow, e0 % kQB, ap);
                } else {
#pragma unroll(16 / E)
                    for (uint32_t r = 0; r < nr; ++r)
                        q8_rank_fma<E>(rec0 + (size_t)r * row, e0 % kQB, ap);
                }
#pragma unroll
                for (int k = 0; k < P; ++k) f2_unpack(ap[k], acc[2 * k], acc[2 * k + 1]);
                if (c + 1 == p.g.nchunks) {
                    const uint8_t* sf = st + p.g.state_off + (size_t)e0 * 4u;
                    lds_f32<E>(sf, w);
                    lds_f32<E>(sf + (size_t)T * 4u, m);
                    lds_f32<E>(sf + (size_t)T * 8u, v);
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[s]);
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
        stg_f16<E>(p.param_out + g0, w, p.param_vec);
    }
    // the < 512 elements past the last tile
    if (blockIdx.x == 0)
        for (uint64_t i = threadIdx.x; i < p.n - p.n_tiled; i += 32u * W)
            fused_q8_element(p, a, p.n_tiled + i, bad);
    flag_overflow(bad, p.status);
    pdl_leave(p.chained);
}

template <bool kDC>
__global__ void __launch_bounds__(256) fused_q8_plain_kernel(const __grid_constant__ FusedQ8Args p) {
    ZK_STEP_CONSTS(p, a);
    bool bad = false;
    const uint64_t stride = (uint64_t)gridDim.x * blockDim.x;
    for (uint64_t i = (uint64_t)blockIdx.x * blockDim.x + threadIdx.x; i < p.n; i += stride)
        fused_q8_element(p, a, i, bad);
    flag_overflow(bad, p.status);
}

// Consumer warps, values per thread and stage split per Nd for the int8 payload, measured on
// B200: the dequantizing accumulation issues about twice the instructions per byte of the fp16
// sum, so up to Nd = 16 the most warps win (Nd = 2/8/16: 6.4/6.7/6.6 TB/s with 24 warps against
// 5.0/5.4/5.5 with 16); above, 16 warps with the budget split in two (Nd = 32/64: 5.9/5.1 TB/s).
// Not better at Nd = 64 (flat 2^28, same box): 8 values per thread with 8, 12 or 16 warps
// (4.6-4.7 TB/s), three or four stages (4.7, 3.9), 12/20/24 warps with three stages (4.4-4.8),
// two CTAs per SM of 8 or 12 warps with half the shared memory each (5.0, 4.8). With the
// compile-time record stride (the current loop, 5.4 TB/s at Nd = 64): eight values per thread
// (4.8-5.0), scalar bias removal and fused multiply-adds instead of the packed pairs (4.9),
// packed bias removal with scalar fused multiply-adds (5.0), explicit 32-bit shared loads (5.3),
// inline byte permutes into register pairs (5.46, the same as the compiler's 5.46); dropping the
// sign-bit flip of signed bytes (offset-binary bytes, now the format) took it to 5.57.
// The record stride as a compile-time constant against the launch's value, flat 2^28, same box,
// two passes each (TB/s): Nd = 2 6.43 / 6.34, 4 6.22 / 6.55, 8 6.16 / 6.72, 16 6.68 / 6.84,
// 32 6.45 / 5.85, 64 5.54 / 4.98; so the run-time stride from Nd = 4 to 16. Above Nd = 48, 24
// consumer warps again (four chunks of 16 ranks per tile): Nd = 64 5.60 against 5.52 TB/s with 16
// warps, the 7.5B view 5.55 against 5.50 (two passes each); at Nd = 48 they lose (5.11 against
// 5.24). A rank loop that issues the next four or eight ranks' shared loads before the current
// ranks' arithmetic (explicit software pipelining) measured slower at every Nd (Nd = 64: 5.17 /
// 5.41 against 5.48 TB/s).
struct VariantQ8 {
    int warps;
    int elems;           // values per consumer thread and tile
    int target_stages;
    bool fixed_row;      // compile-time record stride in the rank loop
};

VariantQ8 pick_variant_q8(int nd) {
    VariantQ8 v = nd <= 16 || nd > 48 ? VariantQ8{24, 4, 2, true} : VariantQ8{16, 4, 2, true};
    v.fixed_row = nd < 4 || nd > 16;
#ifdef ZK_Q8_FIXED_ROW
    v.fixed_row = ZK_Q8_FIXED_ROW;
#endif
#ifdef ZK_Q8_WARPS
    v.warps = ZK_Q8_WARPS;
#endif
#ifdef ZK_Q8_ELEMS
    if (nd > ZK_Q8_ELEMS_MIN_ND) v.elems = ZK_Q8_ELEMS;
#endif
#ifdef ZK_Q8_TARGET_STAGES
    v.target_stages = ZK_Q8_TARGET_STAGES;
#endif
    return v;
}

// Ranks per chunk of the 24-warp shape at Nd = 64 (q8_shape with the default stage budget:
// chunks of 22, 22 and 20 ranks), for which the rank loop is instantiated fully unrolled. Same
// box, two alternating passes each: flat 2^28 5.59 -> 5.68 TB/s, the 7.5B view 5.56 -> 5.64.
constexpr int kRC24 = 22;

// Small calls (fewer than 4 tiles of the large shape per SM): as for the fp16 step, 12
// consumer warps up to Nd = 8 and 8 above, 100 KB of stages and one CTA per SM, so that the
// next call of an overlap region loads beside this one.
constexpr size_t kQ8SmallBudget = 100 * 1024;

// A rank's run of T/128 records per stage.
PipeShape q8_shape(int nd, int warps, int elems, int target_stages, size_t budget) {
    PipeShape sh;
    sh.warps = warps;
    sh.grid_per_sm = 0;
    Geom& g = sh.g;
    g.tile = (uint32_t)(32 * warps * elems);
    const size_t row = (size_t)g.tile / kQB * kRec;
    const size_t state = (size_t)g.tile * 12u;
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

// Grid of the quantizer (a grid-stride kernel of `threads` threads per block): the blocks its
// work needs, at most `waves` full waves of resident blocks (a further, partial wave would run
// the kernel's tail on part of the device).
template <typename K>
cudaError_t resident_grid(K kernel, const DevInfo& di, int threads, uint64_t blocks, int waves,
                          unsigned* grid) {
    int bps = 0;
    cudaError_t e = pipe_blocks_per_sm(kernel, di.dev, threads, 0, &bps);
    if (e != cudaSuccess) return e;
    const uint64_t cap = (uint64_t)di.sms * (uint64_t)bps * (uint64_t)waves;
    if (blocks > cap) blocks = cap;
    *grid = (unsigned)(blocks ? blocks : 1);
    return cudaSuccess;
}

}  // namespace

cudaError_t launch_quant_q8(uint64_t n, const uint16_t* grad, uint8_t* payload,
                            cudaStream_t stream) {
    QuantArgs p;
    p.g = grad;
    p.rec = payload;
    p.n = n;
    p.gvec = (reinterpret_cast<uintptr_t>(grad) & 15u) == 0;
    DevInfo di;
    cudaError_t e = dev_info(&di);
    if (e != cudaSuccess) return e;
    constexpr uint64_t kBpw = 32 / (kQB / kQuantVals);          // blocks per warp, 8 warps/CTA
    const uint64_t ngroups = ((n + kQB - 1) / kQB + kBpw - 1) / kBpw;
    // one full wave of resident blocks: with 16 values per thread 0.77 / 0.82 against 0.76 /
    // 0.80 with two waves and 0.74 / 0.79 with four. (With 8 values per thread two waves had
    // won, 0.64 against 0.63 with one and 0.60 with 8 blocks per SM; 6 or 8 resident blocks per
    // SM forced by launch bounds, registers spilled, and a second load in flight were slower.)
    unsigned grid = 1;
    e = resident_grid(quant_q8_kernel<kQuantVals>, di, 256, (ngroups + 7) / 8, 1, &grid);
    if (e != cudaSuccess) return e;
    return launch_ordered(quant_q8_kernel<kQuantVals>, p, grid, 256, stream);
}

cudaError_t launch_fused_q8(uint64_t n, int nd, const uint8_t* const* payload,
                            const float* master_in, const float* m_in, const float* v_in,
                            float* master_out, float* m_out, float* v_out, uint16_t* param_out,
                            const AdamConsts& a, const AdamConsts* ad, const MeanConsts& mc,
                            uint32_t* status, cudaStream_t stream) {
    FusedQ8Args p;
    memset(&p, 0, sizeof(p));
    bool all16 = aligned16(master_in) && aligned16(m_in) && aligned16(v_in) &&
                 aligned16(master_out) && aligned16(m_out) && aligned16(v_out);
    for (int r = 0; r < nd; ++r) {
        p.rec[r] = payload[r];
        all16 = all16 && aligned16(payload[r]);
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
    DevInfo di;
    cudaError_t e = dev_info(&di);
    if (e != cudaSuccess) return e;
    if (!all16 || n < kMinTiledElems) {
        if (ad)
            fused_q8_plain_kernel<true><<<plain_grid(n, di.sms), 256, 0, stream>>>(p);
        else
            fused_q8_plain_kernel<false><<<plain_grid(n, di.sms), 256, 0, stream>>>(p);
        count_launch();
        return cudaGetLastError();
    }
    const VariantQ8 var = pick_variant_q8(nd);
    const uint64_t big_tiles = n / (32ull * (uint64_t)var.warps * (uint64_t)var.elems);
    PipeShape sh;
    int elems = var.elems;
    if (big_tiles < 4ull * (uint64_t)di.sms) {
        elems = kElems;
        sh = q8_shape(nd, nd <= 8 ? 12 : 8, elems, 2, kQ8SmallBudget);
        sh.grid_per_sm = 1;
    } else {
        sh = q8_shape(nd, var.warps, elems, var.target_stages, kSmemBudget);
    }
    p.g = sh.g;
    p.row = sh.g.tile / kQB * kRec;
    p.n_tiled = n & ~(kQTileAlign - 1);
    p.num_tiles = (p.n_tiled + sh.g.tile - 1) / sh.g.tile;
    p.chained = overlap_next(stream) ? 1 : 0;
    // the instantiated shapes: (warps, values per thread) with 32 * warps * values a multiple
    // of 512, so that a tile is a whole number of 4-record runs
#define ZK_Q8_CASE(WW, EE)                                                                  \
    if (sh.warps == WW && elems == EE) {                                                   \
        if (var.fixed_row)                                                                 \
            return ad ? launch_pipe(fused_q8_tma_kernel<WW, EE, true, true>, p, sh, stream) \
                      : launch_pipe(fused_q8_tma_kernel<WW, EE, false, true>, p, sh, stream); \
        return ad ? launch_pipe(fused_q8_tma_kernel<WW, EE, true, false>, p, sh, stream)   \
                  : launch_pipe(fused_q8_tma_kernel<WW, EE, false, false>, p, sh, stream); \
    }
#ifndef ZK_Q8_NO_RC
    // Nd = 64 in the 24-warp shape: chunks of 22 ranks (22, 22, 20), the full ones unrolled
    if (sh.warps == 24 && elems == 4 && var.fixed_row && sh.g.rc == kRC24) {
        return ad ? launch_pipe(fused_q8_tma_kernel<24, 4, true, true, kRC24>, p, sh, stream)
                  : launch_pipe(fused_q8_tma_kernel<24, 4, false, true, kRC24>, p, sh, stream);
    }
#endif
    ZK_Q8_CASE(8, 4);
    ZK_Q8_CASE(12, 4);
    ZK_Q8_CASE(16, 4);
    ZK_Q8_CASE(24, 4);
#if defined(ZK_Q8_WARPS) || defined(ZK_Q8_ELEMS)
    // shapes measured and not kept (see pick_variant_q8), compiled for comparisons only
    ZK_Q8_CASE(20, 4);
    ZK_Q8_CASE(8, 8);
    ZK_Q8_CASE(12, 8);
    ZK_Q8_CASE(16, 8);
#endif
#undef ZK_Q8_CASE
    return cudaErrorInvalidConfiguration;
}

}  // namespace zk
