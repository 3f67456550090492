/* A stage-3 step driven from C through the C ABI, with no Python in the loop (test
 * infrastructure: built and run by tests/test_gpu_layer_sched.py on a GPU).
 *
 * A small layered list at Nd ranks: the fp16 parameters in Nd partitions, the layer scheduler
 * with two layer buffers on its own gather stream, every layer acquired in forward order (the
 * next one prefetched) and in backward order (the previous one prefetched) with its fused
 * update, then the commit. The first step copies every acquired layer back and compares it with
 * the parameter values it uploaded (a gather is a pure copy); the next `steps` steps measure
 * the host time of the scheduler's calls. Prints one JSON line. */
#define _POSIX_C_SOURCE 199309L
#include <cuda_runtime_api.h>
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>
#include <time.h>

#include "libzero.h"

#define CHECK(x)                                                                   \
    do {                                                                           \
        if ((x) != 0) {                                                            \
            fprintf(stderr, "%s failed at line %d\n", #x, __LINE__);               \
            return 1;                                                              \
        }                                                                          \
    } while (0)

static double now_us(void) {
    struct timespec ts;
    clock_gettime(CLOCK_MONOTONIC, &ts);
    return ts.tv_sec * 1e6 + ts.tv_nsec * 1e-3;
}

enum { kTensors = 6, kLayers = 3 };

int main(int argc, char** argv) {
    const int nd = argc > 1 ? atoi(argv[1]) : 8;
    const int steps = argc > 2 ? atoi(argv[2]) : 50;
    if (nd < 1 || nd > ZERO_MAX_RANKS || steps < 1) return 2;
    const uint64_t numels[kTensors] = {300000, 7000, 250000, 5000, 400000, 1000};
    const int per_layer[kLayers] = {2, 2, 2};
    zero_plan* plan;
    CHECK(zero_plan_create(numels, kTensors, nd, 3, 0, &plan));
    uint64_t psi, psi_p, S;
    int nb;
    CHECK(zero_plan_info(plan, &psi, &psi_p, &S, &nb));
    uint64_t offs[kTensors], bounds[kLayers + 1];
    CHECK(zero_plan_tensor_offsets(plan, offs));
    for (int l = 0, t = 0; l < kLayers; t += per_layer[l], ++l) bounds[l] = offs[t];
    bounds[kLayers] = psi;

    /* the parameters: finite fp16 bit patterns that encode their index */
    uint16_t* h_params = (uint16_t*)malloc(psi_p * 2);
    for (uint64_t i = 0; i < psi_p; ++i)
        h_params[i] = (uint16_t)(0x2000u + ((i * 2654435761u >> 22) & 0x1FFFu));
    uint16_t* parts[ZERO_MAX_RANKS];
    for (int q = 0; q < nd; ++q) {
        CHECK(cudaMalloc((void**)&parts[q], S * 2));
        CHECK(cudaMemcpy(parts[q], h_params + (uint64_t)q * S, S * 2, cudaMemcpyHostToDevice));
    }
    /* gradients (small finite values) and the ping-pong state */
    uint16_t* grads[ZERO_MAX_RANKS];
    for (int r = 0; r < nd; ++r) {
        CHECK(cudaMalloc((void**)&grads[r], psi_p * 2));
        CHECK(cudaMemset(grads[r], 0x10, psi_p * 2));
    }
    float* st[6];
    for (int i = 0; i < 6; ++i) {
        CHECK(cudaMalloc((void**)&st[i], psi_p * 4));
        CHECK(cudaMemset(st[i], 0, psi_p * 4));
    }
    uint32_t* status;
    CHECK(cudaMalloc((void**)&status, 4));
    uint64_t pool_elems;
    CHECK(zero_layer_sched_buf_elems(plan, kLayers, bounds, 2, &pool_elems));
    uint16_t* pool;
    CHECK(cudaMalloc((void**)&pool, pool_elems * 2));
    cudaStream_t compute, gather;
    CHECK(cudaStreamCreate(&compute));
    CHECK(cudaStreamCreate(&gather));
    zero_layer_sched* ls;
    CHECK(zero_layer_sched_create(plan, kLayers, bounds, (const uint16_t* const*)parts, pool,
                                  pool_elems, 2, (zero_stream_t)gather, &ls));
    const zero_adam_hparams hp = {1e-3f, 0.9f, 0.999f, 1e-8f, 1024.0f};
    zero_stream_t cs = (zero_stream_t)compute;
    uint16_t* h_layer = (uint16_t*)malloc(pool_elems * 2);
    int ok = 1;
    double acq_us = 0.0, rel_us = 0.0;
    long n_acq = 0;
    for (int step = 0; step <= steps; ++step) {
        const int check = step == 0;
        float** in = step % 2 ? st + 3 : st;
        float** out = step % 2 ? st : st + 3;
        CHECK(cudaMemsetAsync(status, 0, 4, compute));
        CHECK(zero_layer_sched_begin_step(ls, status, cs));
        for (int pass = 0; pass < 2; ++pass) {
            for (int i = 0; i < kLayers; ++i) {
                const int l = pass == 0 ? i : kLayers - 1 - i;
                const int next = pass == 0 ? (l + 1 < kLayers ? l + 1 : -1) : l - 1;
                uint16_t* w;
                double t0 = now_us();
                CHECK(zero_layer_sched_acquire(ls, l, next, cs, &w));
                acq_us += now_us() - t0;
                ++n_acq;
                const uint64_t lo = bounds[l], len = bounds[l + 1] - lo;
                if (check) {    /* the layer as acquired equals the uploaded values */
                    CHECK(cudaMemcpyAsync(h_layer, w, len * 2, cudaMemcpyDeviceToHost, compute));
                    CHECK(cudaStreamSynchronize(compute));
                    ok &= memcmp(h_layer, h_params + lo, len * 2) == 0;
                }
                t0 = now_us();
                CHECK(zero_layer_sched_release(ls, l, cs));
                rel_us += now_us() - t0;
                if (pass == 1) {
                    const uint64_t ghi = l == kLayers - 1 ? psi_p : bounds[l + 1];
                    const uint16_t* g[ZERO_MAX_RANKS];
                    for (int r = 0; r < nd; ++r) g[r] = grads[r] + lo;
                    CHECK(zero_stage3_step_fused(plan, lo, ghi - lo, g, in[0] + lo, in[1] + lo,
                                                 in[2] + lo, out[0] + lo, out[1] + lo,
                                                 out[2] + lo, parts, &hp, 1, status, cs));
                }
            }
        }
        CHECK(zero_stage3_step_commit(plan, in[0], in[1], in[2], out[0], out[1], out[2], parts,
                                      status, cs));
        if (check) {
            uint32_t flags = 0;
            if (zero_step_status(status, cs, &flags) != ZERO_OK) ok = 0;
            /* the updates have rewritten the partitions: only this step is compared */
            acq_us = rel_us = 0.0;
            n_acq = 0;
        }
    }
    uint32_t flags = 0;
    const zero_status fin = zero_step_status(status, cs, &flags);
    uint64_t gathers = 0;
    CHECK(zero_layer_sched_gathers(ls, &gathers));
    printf("{\"ok\": %s, \"status\": %d, \"flags\": %u, \"gathers\": %llu, \"steps\": %d, "
           "\"layers\": %d, \"host_us_acquire\": %.3f, \"host_us_release\": %.3f}\n",
           ok ? "true" : "false", (int)fin, flags, (unsigned long long)gathers, steps + 1,
           kLayers, acq_us / (double)n_acq, rel_us / (double)n_acq);
    zero_layer_sched_destroy(ls);
    zero_plan_destroy(plan);
    free(h_layer);
    free(h_params);
    return ok && fin == ZERO_OK ? 0 : 3;
}
