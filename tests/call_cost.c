/* Host cost of one libzero data-path call, measured from C with no Python in the loop
 * (test infrastructure: built and run by tests/test_gpu_call_cost.py on a GPU).
 *
 * One bucket call of zero_step_fused over n elements at nd ranks (default: a 1 MiB bucket of
 * fp16 gradient per rank, Nd = 8), repeated `calls` times on one stream:
 *   host_us_ordered  host time per call, outside an overlap region;
 *   host_us_region   host time per call, inside zero_overlap_begin/end;
 *   gpu_us_region    device time per call of the region's calls (CUDA events);
 * each a median over `reps` repetitions, the launches of a repetition fewer than the device's
 * launch queue holds so that the host never waits for the device. Consecutive calls use
 * different buffers (a ring of kSets), so that the calls of a region are independent, as a
 * region requires. Prints one JSON line. */
#define _POSIX_C_SOURCE 199309L
#include <cuda_runtime_api.h>
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
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

static int cmp_d(const void* a, const void* b) {
    const double x = *(const double*)a, y = *(const double*)b;
    return x < y ? -1 : x > y;
}

static double median(double* v, int n) {
    qsort(v, (size_t)n, sizeof(double), cmp_d);
    return v[n / 2];
}

int main(int argc, char** argv) {
    const uint64_t n = argc > 1 ? strtoull(argv[1], 0, 10) : (1u << 19);
    const int nd = argc > 2 ? atoi(argv[2]) : 8;
    const int calls = argc > 3 ? atoi(argv[3]) : 400;
    const int reps = 7;
    if (nd < 1 || nd > ZERO_MAX_RANKS || calls < 1 || n == 0) return 2;
    enum { kSets = 4 };
    uint16_t* grads[kSets][ZERO_MAX_RANKS];
    float* st[kSets][6];
    uint16_t* params[kSets];
    for (int k = 0; k < kSets; ++k) {
        for (int r = 0; r < nd; ++r) {
            CHECK(cudaMalloc((void**)&grads[k][r], n * 2));
            CHECK(cudaMemset(grads[k][r], 0, n * 2));
        }
        for (int i = 0; i < 6; ++i) {
            CHECK(cudaMalloc((void**)&st[k][i], n * 4));
            CHECK(cudaMemset(st[k][i], 0, n * 4));
        }
        CHECK(cudaMalloc((void**)&params[k], n * 2));
    }
    uint32_t* status;
    CHECK(cudaMalloc((void**)&status, 4));
    CHECK(cudaMemset(status, 0, 4));
    cudaStream_t s;
    CHECK(cudaStreamCreate(&s));
    cudaEvent_t e0, e1;
    CHECK(cudaEventCreate(&e0));
    CHECK(cudaEventCreate(&e1));
    const zero_adam_hparams hp = {1e-3, 0.9, 0.999, 1e-8, 1024.0};
    zero_stream_t zs = (zero_stream_t)s;
#define CALL(i)                                                                              \
    zero_step_fused(n, nd, (const uint16_t* const*)grads[(i) % kSets], st[(i) % kSets][0],     \
                    st[(i) % kSets][1], st[(i) % kSets][2], st[(i) % kSets][3],                \
                    st[(i) % kSets][4], st[(i) % kSets][5], params[(i) % kSets], &hp, 1,       \
                    status, zs)

    for (int i = 0; i < 50; ++i)   /* warm-up: occupancy caches, module load */
        CHECK(CALL(i));
    CHECK(cudaStreamSynchronize(s));

    double ordered[reps], region[reps], gpu[reps];
    for (int k = 0; k < reps; ++k) {
        double t0 = now_us();
        for (int i = 0; i < calls; ++i) CHECK(CALL(i));
        ordered[k] = (now_us() - t0) / calls;
        CHECK(cudaStreamSynchronize(s));

        t0 = now_us();
        CHECK(cudaEventRecord(e0, s));
        CHECK(zero_overlap_begin(zs));
        for (int i = 0; i < calls; ++i) CHECK(CALL(i));
        CHECK(zero_overlap_end(zs));
        CHECK(cudaEventRecord(e1, s));
        region[k] = (now_us() - t0) / calls;
        CHECK(cudaEventSynchronize(e1));
        float ms = 0.0f;
        CHECK(cudaEventElapsedTime(&ms, e0, e1));
        gpu[k] = 1e3 * ms / calls;
    }
    uint32_t flags = 0;
    CHECK(cudaMemcpy(&flags, status, 4, cudaMemcpyDeviceToHost));
    const double bytes = (double)(2 * nd + 26) * (double)n;
    const double g_us = median(gpu, reps);
    printf("{\"n\": %llu, \"nd\": %d, \"calls\": %d, \"host_us_ordered\": %.3f, "
           "\"host_us_region\": %.3f, \"gpu_us_region\": %.3f, \"bytes_per_call\": %.0f, "
           "\"gpu_gbs_region\": %.1f, \"status\": %u}\n",
           (unsigned long long)n, nd, calls, median(ordered, reps), median(region, reps), g_us,
           bytes, bytes / (g_us * 1e3), flags);
    return 0;
}
