/*
 * CPU oracle for the ZeRO stage-1/2 data-parallel step.
 *
 * TEST INFRASTRUCTURE ONLY. Only the tests, the smoke check and the benchmark's CPU-baseline
 * leg load this code. It shares no source, header, table or helper with the CUDA library and
 * never calls it. It is plain, slow, single-threaded C, built with -O2 -ffp-contract=off so
 * that every floating-point operation below is one IEEE-754 operation, rounded to nearest-even,
 * in the precision written.
 *
 * What it computes, and where the pages say so:
 *   - Model-state accounting (2 bytes fp16 params + 2 bytes fp16 grads + K bytes of fp32
 *     optimizer state per parameter, K = 12) and the per-device bytes of plain DP and of the
 *     three ZeRO-DP stages; communication volume per step:
 *       "ZeRO: particionar estados do treino entre GPUs", section "Como funciona";
 *       "ZeRO" (lastdictionary), main definition.
 *   - Flat partition of the parameter list into Nd contiguous shards, one owner each:
 *       "Como funciona" (states divided into Nd parts, each process updates its own part);
 *       "ZeRO-2" card, section "ZeRO-1에서 남은 낭비" (local grad [g_A, g_B, g_C] per GPU).
 *   - Buckets in backward order (B2, B1, B0), each reduce-scattered, own shard kept:
 *       "ZeRO-2" card, diagram and section "Gradient 생명주기".
 *   - Reduced gradient = mean over the Nd ranks of the fp16 local gradients, summed in fp32
 *     in rank order 0..Nd-1 (the order is our reading; the pages name no order).
 *   - Mixed-precision Adam on the owner's shard (fp32 master, momentum, variance), then the
 *     fp16 cast of the updated master written into the full parameter buffer (all-gather):
 *       "Como funciona"; "ZeRO-2" card, sections "Gradient 생명주기" and
 *       "왜 all-gather는 그대로 필요한가".
 *   - The update itself is the unpartitioned one ("ZeRO" (lastdictionary), "Usage note":
 *     ZeRO changes where state is stored, not how updates are computed).
 *
 * Parity pins live in tests/test_oracle_pins.py; none of them re-types the formulas below.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

#define ORC_OK 0
#define ORC_EINVAL 1

/* ------------------------------------------------------------------------------------------
 * binary16 <-> binary32, written from the IEEE 754-2008 definitions.
 * binary16: sign (1 bit), biased exponent (5 bits, bias 15), fraction (10 bits).
 *   exponent 1..30 : (-1)^s * 2^(e-15) * (1 + f/2^10)
 *   exponent 0     : (-1)^s * 2^-14 * (f/2^10)        (zero and subnormals)
 *   exponent 31    : infinity (f = 0) or NaN (f != 0)
 * ---------------------------------------------------------------------------------------- */

static uint32_t bits_of(float x) { uint32_t u; memcpy(&u, &x, 4); return u; }
static float float_of(uint32_t u) { float x; memcpy(&x, &u, 4); return x; }

float orc_h2f(uint16_t h)
{
    uint32_t s = (uint32_t)(h >> 15) & 1u;
    uint32_t e = (uint32_t)(h >> 10) & 0x1fu;
    uint32_t f = (uint32_t)h & 0x3ffu;
    if (e == 0x1f) {
        /* infinity, or a quiet NaN that keeps the fraction bits as payload */
        return float_of((s << 31) | 0x7f800000u | (f ? (0x00400000u | (f << 13)) : 0u));
    }
    /* Both branches are exact: the integer has at most 11 bits and the scale is a power of 2
     * that keeps the result inside the binary32 normal range. */
    float mag = (e == 0) ? ldexpf((float)f, -24) : ldexpf((float)(f | 0x400u), (int)e - 25);
    return s ? -mag : mag;
}

/* Round a binary32 value to the nearest binary16 value, ties to the even significand;
 * magnitudes that round beyond the largest finite value (65504) become infinity. */
uint16_t orc_f2h(float x)
{
    uint32_t u = bits_of(x);
    uint16_t sign = (uint16_t)((u >> 16) & 0x8000u);
    uint32_t ex = (u >> 23) & 0xffu;
    uint32_t man = u & 0x7fffffu;
    if (ex == 0xff) {
        if (man == 0) return (uint16_t)(sign | 0x7c00u);
        return (uint16_t)(sign | 0x7e00u | (man >> 13)); /* NaN stays a (quiet) NaN */
    }
    if (ex == 0) return sign; /* binary32 zero or subnormal: below 2^-126, rounds to zero */
    int e = (int)ex - 127;        /* |x| = m24 * 2^(e-23), m24 in [2^23, 2^24) */
    uint32_t m24 = man | 0x800000u;
    if (e >= 16) return (uint16_t)(sign | 0x7c00u); /* |x| >= 65536 */
    /* Spacing of binary16 values around |x|: 2^(e-10) in the normal range, 2^-24 below it. */
    int se = (e >= -14) ? (e - 10) : -24;
    /* |x| / spacing = m24 / 2^sh */
    int sh = se - (e - 23);
    uint32_t n;
    if (sh > 25) {
        n = 0; /* |x| / spacing < 1/4: rounds to zero */
    } else {
        uint32_t rem = m24 & ((1u << sh) - 1u);
        uint32_t half = 1u << (sh - 1);
        n = m24 >> sh;
        if (rem > half || (rem == half && (n & 1u))) n += 1u;
    }
    uint32_t bits;
    if (se == -24) {
        /* subnormal target: value = n * 2^-24; n == 1024 is exactly 2^-14, whose encoding is
         * also 1024 (exponent field 1, fraction 0) */
        bits = n;
    } else {
        /* normal target: n in [1024, 2048]; n == 2048 carries into the exponent field */
        bits = ((uint32_t)(e + 15) << 10) + (n - 1024u);
        if (bits >= 0x7c00u) bits = 0x7c00u;
    }
    return (uint16_t)(sign | bits);
}

void orc_h2f_array(uint64_t n, const uint16_t* h, float* out)
{
    for (uint64_t i = 0; i < n; i++) out[i] = orc_h2f(h[i]);
}

void orc_f2h_array(uint64_t n, const float* x, uint16_t* out)
{
    for (uint64_t i = 0; i < n; i++) out[i] = orc_f2h(x[i]);
}

/* ------------------------------------------------------------------------------------------
 * Model-state accounting ("Como funciona"; "ZeRO" (lastdictionary) main definition).
 * Bytes held by one device, for psi parameters and nd data-parallel processes:
 *   stage 0 (plain DP) : params 2psi, grads 2psi, optimizer K psi
 *   stage 1 (Pos)      : params 2psi, grads 2psi, optimizer K psi/nd
 *   stage 2 (Pos+g)    : params 2psi, grads 2psi/nd, optimizer K psi/nd
 *   stage 3 (Pos+g+p)  : params 2psi/nd, grads 2psi/nd, optimizer K psi/nd
 * A partitioned quantity is held as a shard of ceil(psi/nd) elements (the padded shard).
 * Communication per step, in elements: 2psi for DP, Pos and Pos+g (reduce-scatter plus
 * all-gather, psi each), 3psi for Pos+g+p (two parameter all-gathers plus the reduce-scatter).
 * out_bytes is [stage][params, grads, optim, total]; out_comm is [stage].
 * ---------------------------------------------------------------------------------------- */
int orc_state_bytes(uint64_t psi, int nd, int K, uint64_t* out_bytes, uint64_t* out_comm)
{
    if (nd < 1 || K < 0) return ORC_EINVAL;
    uint64_t shard = (psi + (uint64_t)nd - 1) / (uint64_t)nd;
    uint64_t p_full = 2 * psi, g_full = 2 * psi, o_full = (uint64_t)K * psi;
    uint64_t p_sh = 2 * shard, g_sh = 2 * shard, o_sh = (uint64_t)K * shard;
    uint64_t tab[4][3] = {
        {p_full, g_full, o_full},
        {p_full, g_full, o_sh},
        {p_full, g_sh, o_sh},
        {p_sh, g_sh, o_sh},
    };
    for (int s = 0; s < 4; s++) {
        out_bytes[4 * s + 0] = tab[s][0];
        out_bytes[4 * s + 1] = tab[s][1];
        out_bytes[4 * s + 2] = tab[s][2];
        out_bytes[4 * s + 3] = tab[s][0] + tab[s][1] + tab[s][2];
    }
    out_comm[0] = 2 * psi;
    out_comm[1] = 2 * psi;
    out_comm[2] = 2 * psi;
    out_comm[3] = 3 * psi;
    return ORC_OK;
}

/* ------------------------------------------------------------------------------------------
 * Partition plan.
 * The tensors are laid end to end in forward order; the flat list is padded with zeros to
 * psi_p = ceil(psi/nd)*nd; shard r is [r*S, (r+1)*S) with S = psi_p/nd and belongs to rank r.
 * Buckets are produced by the backward pass from the end of the flat list towards its start:
 * bucket k covers [max(0, psi_p - (k+1)B), psi_p - kB). bucket_elems = 0 means one bucket.
 * ---------------------------------------------------------------------------------------- */
int orc_plan(const uint64_t* numels, int n_tensors, int nd, uint64_t bucket_elems,
             uint64_t* tensor_off, uint64_t* psi, uint64_t* psi_p, uint64_t* shard,
             int64_t* n_buckets)
{
    if (n_tensors < 0 || nd < 1) return ORC_EINVAL;
    uint64_t total = 0;
    for (int t = 0; t < n_tensors; t++) {
        tensor_off[t] = total;
        total += numels[t];
    }
    uint64_t s = (total + (uint64_t)nd - 1) / (uint64_t)nd;
    *psi = total;
    *shard = s;
    *psi_p = s * (uint64_t)nd;
    uint64_t b = bucket_elems ? bucket_elems : *psi_p;
    if (*psi_p == 0) {
        *n_buckets = 0;
    } else {
        int64_t count = 0;
        uint64_t hi = *psi_p;
        while (hi > 0) { /* walk down from the top, one bucket at a time */
            hi = (hi > b) ? hi - b : 0;
            count++;
        }
        *n_buckets = count;
    }
    return ORC_OK;
}

int orc_bucket(uint64_t psi_p, uint64_t bucket_elems, int64_t k, uint64_t* lo, uint64_t* len)
{
    uint64_t b = bucket_elems ? bucket_elems : psi_p;
    uint64_t hi = psi_p;
    for (int64_t j = 0; j < k; j++) {
        if (hi == 0) return ORC_EINVAL;
        hi = (hi > b) ? hi - b : 0;
    }
    if (hi == 0 || k < 0) return ORC_EINVAL;
    *lo = (hi > b) ? hi - b : 0;
    *len = hi - *lo;
    return ORC_OK;
}

/* ------------------------------------------------------------------------------------------
 * Adam constants. Computed in double from the hyperparameters and the step t >= 1, each
 * rounded once to binary32 (the precision of the optimizer state, "Como funciona").
 * Adam as Kingma & Ba give it, with the bias corrections folded into the step size and the
 * denominator (the form torch.optim.Adam uses): step_size = lr/(1-beta1^t),
 * denom = sqrt(v)/sqrt(1-beta2^t) + eps.
 * ---------------------------------------------------------------------------------------- */
typedef struct {
    double lr, beta1, beta2, eps, loss_scale;
} orc_hparams;

typedef struct {
    float b1, omb1, b2, omb2, step_size, bc2s, eps, loss_scale;
} orc_scalars;

int orc_adam_scalars(const orc_hparams* hp, int64_t t, orc_scalars* s)
{
    if (t < 1) return ORC_EINVAL;
    double bc1 = 1.0 - pow(hp->beta1, (double)t);
    double bc2 = 1.0 - pow(hp->beta2, (double)t);
    s->b1 = (float)hp->beta1;
    s->omb1 = (float)(1.0 - hp->beta1);
    s->b2 = (float)hp->beta2;
    s->omb2 = (float)(1.0 - hp->beta2);
    s->step_size = (float)(hp->lr / bc1);
    s->bc2s = (float)sqrt(bc2);
    s->eps = (float)hp->eps;
    s->loss_scale = (float)hp->loss_scale;
    return ORC_OK;
}

/* ------------------------------------------------------------------------------------------
 * Reduce: the gradient of element i reduced over the nd ranks, as its owner keeps it after
 * the reduce-scatter. Sum in binary32, rank 0 first, then divide by nd (the mean).
 * g[r] points at rank r's local fp16 gradient for the same n elements.
 * ---------------------------------------------------------------------------------------- */
void orc_reduce_mean(uint64_t n, int nd, const uint16_t* const* g, float* red)
{
    float fnd = (float)nd;
    for (uint64_t i = 0; i < n; i++) {
        float s = 0.0f;
        for (int r = 0; r < nd; r++) s = s + orc_h2f(g[r][i]);
        red[i] = s / fnd;
    }
}

/* 1 if every value is finite (no inf, no NaN), else 0 */
int orc_all_finite(uint64_t n, const float* x)
{
    for (uint64_t i = 0; i < n; i++) {
        uint32_t u = bits_of(x[i]);
        if (((u >> 23) & 0xffu) == 0xffu) return 0;
    }
    return 1;
}

/* ------------------------------------------------------------------------------------------
 * The owner's update of its shard, one element at a time, from the reduced (still loss-scaled)
 * gradient:
 *   g      = red / loss_scale
 *   m      = beta1*m + (1-beta1)*g
 *   v      = beta2*v + (1-beta2)*(g*g)
 *   denom  = sqrt(v)/sqrt(1-beta2^t) + eps
 *   master = master - step_size*(m/denom)
 *   p16    = binary16(master)
 * Every product, quotient, sum and square root is its own rounded binary32 operation.
 * ---------------------------------------------------------------------------------------- */
void orc_adam(uint64_t n, const float* red, float* master, float* m, float* v, uint16_t* p16,
              const orc_scalars* s)
{
    for (uint64_t i = 0; i < n; i++) {
        float g = red[i] / s->loss_scale;
        float m_keep = s->b1 * m[i];
        float m_new = s->omb1 * g;
        float mt = m_keep + m_new;
        float gsq = g * g;
        float v_keep = s->b2 * v[i];
        float v_new = s->omb2 * gsq;
        float vt = v_keep + v_new;
        float root = sqrtf(vt);
        float denom = root / s->bc2s + s->eps;
        float ratio = mt / denom;
        float delta = s->step_size * ratio;
        float w = master[i] - delta;
        m[i] = mt;
        v[i] = vt;
        master[i] = w;
        if (p16) p16[i] = orc_f2h(w);
    }
}

/* ------------------------------------------------------------------------------------------
 * One owner's whole step on n elements of its shard (stage 1 with the full local gradients at
 * hand): reduce, check the whole range for overflow, and update only if it is all finite.
 * red_scratch holds n floats. Returns 1 if the step was skipped (state and p16 untouched).
 * ---------------------------------------------------------------------------------------- */
int orc_step(uint64_t n, int nd, const uint16_t* const* g, float* master, float* m, float* v,
             uint16_t* p16, const orc_hparams* hp, int64_t t, float* red_scratch)
{
    orc_scalars s;
    if (orc_adam_scalars(hp, t, &s) != ORC_OK) return -1;
    orc_reduce_mean(n, nd, g, red_scratch);
    if (!orc_all_finite(n, red_scratch)) return 1;
    orc_adam(n, red_scratch, master, m, v, p16, &s);
    return 0;
}

/* ------------------------------------------------------------------------------------------
 * Compressed reduce-scatter payload (int8 + one fp32 scale per block of 128 elements).
 * "ZeRO" (lastdictionary), main definition: extensions compress the communication (ZeRO++).
 * The pages give no format; the one used: for each block of ORC_QB consecutive elements of a
 * rank's slice (the last block may be short),
 *   amax  = max |x|                          (exact; any inf/NaN in the block poisons it)
 *   scale = amax / 127                        (binary32 division), NaN for a poisoned block
 *   q     = round_half_even(x / scale), clamped to [-127, 127]; 0 if scale is 0 or NaN
 * and the owner accumulates the ranks in order 0..nd-1 with one fused multiply-add each,
 * s = fma(float(q), scale, s) (the product and the sum rounded once, C99 fmaf), then divides by
 * nd, exactly as for fp16 slices.
 * ---------------------------------------------------------------------------------------- */
#define ORC_QB 128

static int finite_f32(float x) { return ((bits_of(x) >> 23) & 0xffu) != 0xffu; }

/* nearest integer to x, ties to even, for |x| < 2^23 */
static float rint_even(float x)
{
    float a = x < 0 ? -x : x;
    float f = (float)(int32_t)a;          /* truncation toward zero, exact */
    float r = a - f;                      /* exact: the fraction */
    if (r > 0.5f || (r == 0.5f && ((int32_t)f & 1))) f = f + 1.0f;
    return x < 0 ? -f : f;
}

void orc_quant_q8(uint64_t n, const uint16_t* g, int8_t* q, float* scales)
{
    for (uint64_t b0 = 0; b0 < n; b0 += ORC_QB) {
        uint64_t b1 = b0 + ORC_QB < n ? b0 + ORC_QB : n;
        float amax = 0.0f;
        int poisoned = 0;
        for (uint64_t i = b0; i < b1; i++) {
            float x = orc_h2f(g[i]);
            if (!finite_f32(x)) poisoned = 1;
            else {
                float a = x < 0 ? -x : x;
                if (a > amax) amax = a;
            }
        }
        float scale = poisoned ? float_of(0x7fc00000u) : amax / 127.0f;
        scales[b0 / ORC_QB] = scale;
        for (uint64_t i = b0; i < b1; i++) {
            if (poisoned || scale == 0.0f) { q[i] = 0; continue; }
            float k = rint_even(orc_h2f(g[i]) / scale);
            if (k > 127.0f) k = 127.0f;
            if (k < -127.0f) k = -127.0f;
            q[i] = (int8_t)k;
        }
    }
}

/* The owner's reduced gradient from nd int8 payloads (q[r], scales[r] cover the same n
 * elements, blocks counted from element 0). */
void orc_reduce_mean_q8(uint64_t n, int nd, const int8_t* const* q, const float* const* scales,
                        float* red)
{
    float fnd = (float)nd;
    for (uint64_t i = 0; i < n; i++) {
        float s = 0.0f;
        for (int r = 0; r < nd; r++) s = fmaf((float)q[r][i], scales[r][i / ORC_QB], s);
        red[i] = s / fnd;
    }
}

/* The same reduction on gathered samples: scale[r][i] is the scale of sample i's block. */
void orc_reduce_mean_q8_gathered(uint64_t n, int nd, const int8_t* const* q,
                                 const float* const* scale, float* red)
{
    float fnd = (float)nd;
    for (uint64_t i = 0; i < n; i++) {
        float s = 0.0f;
        for (int r = 0; r < nd; r++) s = fmaf((float)q[r][i], scale[r][i], s);
        red[i] = s / fnd;
    }
}
