/*
 * libzero -- the data-parallel hot path of ZeRO stages 1 and 2 on one NVIDIA B200 (sm_100a).
 *
 * ZeRO-DP keeps, per parameter, 2 bytes of fp16 weights, 2 bytes of fp16 gradients and
 * K = 12 bytes of fp32 optimizer state (master copy, momentum, variance), and partitions that
 * state among the Nd data-parallel processes: stage 1 (Pos) splits the optimizer state, stage 2
 * (Pos+g) also the gradients. Each gradient is reduced only on the owner of its partition by a
 * reduce-scatter, the owner updates its own 1/Nd of the parameters with mixed-precision Adam,
 * and an all-gather distributes the updated parameters.
 *   Sources: "ZeRO: particionar estados do treino entre GPUs" (upskillscore.com), section
 *   "Como funciona"; "ZeRO" (lastdictionary.com), main definition; "ZeRO-2" card
 *   (llm-engineer.pages.dev), sections "Gradient 생명주기" and "왜 all-gather는 그대로 필요한가".
 *
 * In this library the Nd ranks are separate buffers in the memory of ONE GPU: the
 * reduce-scatter is each owner reading its slice of every rank's gradient, and the all-gather
 * is each owner writing its updated fp16 shard into one full parameter buffer that stands for
 * every replica's copy.
 *
 * Conventions shared by every call:
 *   - fp16 values travel as uint16_t bit patterns (IEEE binary16); fp32 as float.
 *   - Every device pointer is caller-owned device memory of the current CUDA device. The
 *     library allocates no device memory; the plan and the scheduler are its only objects
 *     (host memory, plus CUDA events for the scheduler).
 *   - zero_stream_t is a cudaStream_t (NULL = the legacy default stream). Data-path calls are
 *     asynchronous and stream-ordered; only zero_step_status waits for the device.
 *   - Every call returns a zero_status and never aborts or throws. Host-detectable argument
 *     errors return at once and launch nothing. A failed CUDA launch returns ZERO_ECUDA.
 *   - Outcomes known only on the device go to a caller-owned 32-bit status word in device
 *     memory (d_status, the ZERO_FLAG_* bits). Zero it before the first call of each step.
 *   - Sizes and offsets are element counts (uint64_t) unless named *_bytes.
 *   - Thread safety: calls on different plans/schedulers may run concurrently; a plan is
 *     read-only after creation; a scheduler is used by one host thread at a time.
 */
#ifndef LIBZERO_H
#define LIBZERO_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* zero_stream_t; /* same type as cudaStream_t */

typedef enum {
    ZERO_OK = 0,
    ZERO_EINVAL = 1,        /* bad argument: null pointer, size, range, Nd, aliasing */
    ZERO_EALIGN = 2,        /* a pointer is not aligned to its element size */
    ZERO_ECUDA = 3,         /* a CUDA runtime call or kernel launch failed */
    ZERO_ENOMEM = 4,        /* host allocation failed, or a caller buffer is too small */
    ZERO_STEP_SKIPPED = 5   /* zero_step_status: the step was skipped on overflow */
} zero_status;

/* Bits of the device status word d_status. */
#define ZERO_FLAG_OVERFLOW 0x1u /* some reduced gradient of this step was inf or NaN */
#define ZERO_FLAG_SKIPPED 0x2u  /* the step was not applied (state and params unchanged) */
#define ZERO_FLAG_TIMEOUT 0x4u  /* a kernel's bounded wait gave up; its outputs are invalid */
#define ZERO_FLAG_BOUNDS 0x8u   /* a kernel's internal bounds self-check failed (a library bug):
                                   the access was skipped; outputs are invalid */

#define ZERO_MAX_RANKS 64       /* largest Nd a call accepts */

/* Human-readable name of a status code (static string). */
const char* zero_status_string(zero_status s);

/* Kernels this library has launched in this process so far (all entry points). */
uint64_t zero_kernel_launches(void);

/* Text of the last CUDA error behind a ZERO_ECUDA returned to this host thread ("" if none);
 * valid until the next libzero call on the thread. */
const char* zero_last_error(void);

/* ------------------------------------------------------------------------------------------
 * Partition plan.
 * "Como funciona": the model states are divided into Nd parts, one per data-parallel process;
 * "ZeRO-2" card, "ZeRO-1에서 남은 낭비": every GPU's local gradient is [g_A, g_B, g_C], one
 * slice per owner; diagram and "Gradient 생명주기": the backward pass hands over buckets in
 * reverse layer order (B2, B1, B0), each reduce-scattered at once.
 *
 * The n_tensors tensors (numels[i] elements each, in forward order) are laid end to end into
 * one flat list of psi elements, padded with zeros to psi_padded = ceil(psi/nd)*nd. Owner r
 * holds shard [r*S, (r+1)*S) with S = psi_padded/nd. Bucket k (k = 0 is produced first) is
 * [max(0, psi_padded - (k+1)*B), psi_padded - k*B) with B = bucket_elems (0: one bucket of
 * everything). stage is 1, 2 or 3 (recorded; the map is the same).
 * Errors: ZERO_EINVAL for out == NULL, numels == NULL with n_tensors > 0, n_tensors < 0,
 * nd outside [1, ZERO_MAX_RANKS], stage outside {1, 2, 3}, or psi == 0; ZERO_ENOMEM if the host
 * allocation fails. On success *out owns host memory released by zero_plan_destroy.
 * ---------------------------------------------------------------------------------------- */
typedef struct zero_plan zero_plan;

zero_status zero_plan_create(const uint64_t* numels, int n_tensors, int nd, int stage,
                             uint64_t bucket_elems, zero_plan** out);
void zero_plan_destroy(zero_plan* plan);

/* psi, psi_padded, shard length S and the bucket count; any output may be NULL. */
zero_status zero_plan_info(const zero_plan* plan, uint64_t* psi, uint64_t* psi_padded,
                           uint64_t* shard_elems, int* n_buckets);
/* Flat offset of each tensor (n_tensors values written to out). */
zero_status zero_plan_tensor_offsets(const zero_plan* plan, uint64_t* out);
/* Bucket k: its flat range [flat_lo, flat_lo + len) and the owners it touches,
 * owner_lo..owner_hi inclusive. ZERO_EINVAL if k is out of range. */
zero_status zero_plan_bucket(const zero_plan* plan, int k, uint64_t* flat_lo, uint64_t* len,
                             int* owner_lo, int* owner_hi);

/* ------------------------------------------------------------------------------------------
 * Model-state accounting, bytes held by one device ("Como funciona"; "ZeRO" (lastdictionary)):
 *   stage[0] plain DP  : params 2psi, grads 2psi,   optim K psi      (16 psi for K = 12)
 *   stage[1] Pos       : params 2psi, grads 2psi,   optim K psi/Nd   (4psi + 12psi/Nd)
 *   stage[2] Pos+g     : params 2psi, grads 2psi/Nd, optim K psi/Nd  (2psi + 14psi/Nd)
 *   stage[3] Pos+g+p   : params 2psi/Nd, grads 2psi/Nd, optim K psi/Nd (16psi/Nd)
 * A partitioned quantity counts ceil(psi/Nd) elements. Communication per step in elements:
 * 2psi (DP, Pos, Pos+g: reduce-scatter + all-gather), 3psi (Pos+g+p: two parameter
 * all-gathers + the reduce-scatter); comm_bytes_fp16 is twice that.
 * Errors: ZERO_EINVAL for out == NULL, nd < 1, K < 0, or psi so large that a byte count
 * would not fit in 64 bits (psi > UINT64_MAX / (K + 6)).
 * ---------------------------------------------------------------------------------------- */
typedef struct {
    uint64_t params, grads, optim, total;
} zero_bytes;

typedef struct {
    zero_bytes stage[4];
    uint64_t comm_elems[4];
    uint64_t comm_bytes_fp16[4];
} zero_state_report;

zero_status zero_state_bytes(uint64_t psi, int nd, int K, zero_state_report* out);

/* ------------------------------------------------------------------------------------------
 * Adam hyperparameters (host memory, read during the call only). Host-side constants are
 * computed from them in double and rounded once to fp32: beta1, 1-beta1, beta2, 1-beta2,
 * step_size = lr/(1-beta1^t), sqrt(1-beta2^t), eps, loss_scale.
 * Requirements: lr finite; 0 <= beta1, beta2 < 1; eps >= 0; loss_scale finite and > 0.
 * ---------------------------------------------------------------------------------------- */
typedef struct {
    double lr, beta1, beta2, eps, loss_scale;
} zero_adam_hparams;

/* The fp32 constants of one Adam step t, in the layout the kernels read them (40 bytes). */
typedef struct {
    float beta1, one_minus_beta1, beta2, one_minus_beta2;
    float step_size;      /* lr / (1 - beta1^t) */
    float bias2_sqrt;     /* sqrt(1 - beta2^t) */
    float eps;
    float loss_scale;     /* the unscale divisor */
    float inv_loss_scale; /* 1/loss_scale if loss_scale is a power of two, else 0 */
    int32_t loss_scale_pow2;
} zero_adam_consts;

/* Fill *out with the constants of step t (t >= 1) exactly as zero_adam_shard and
 * zero_step_fused compute them. Errors: ZERO_EINVAL (null pointers, t < 1, bad hparams). */
zero_status zero_adam_consts_for_step(const zero_adam_hparams* hp, int64_t step,
                                      zero_adam_consts* out);

/* ------------------------------------------------------------------------------------------
 * Bucketed reduce-scatter (stage 2). "ZeRO-2" card, "Gradient 생명주기": as soon as a bucket's
 * local gradient exists it is reduce-scattered; each GPU keeps only its reduced shard.
 *
 * For every element i of bucket k (flat index f = flat_lo + i):
 *   red = (sum over r = 0..nd-1, in that order, of fp32(rank_grads[r][i])) / nd   (fp32)
 *   owner_grad_shards[f / S][f % S] = red
 * and ZERO_FLAG_OVERFLOW is ORed into *d_status if any red is inf or NaN.
 *   rank_grads        : nd device pointers (host array), each to `len` fp16 values: rank r's
 *                       local gradient of bucket k. 2-byte aligned; 16-byte alignment takes
 *                       the fast path.
 *   owner_grad_shards : nd device pointers (host array), each to S fp32 values (4-byte
 *                       aligned): owner r's reduced-gradient shard. Only the part covered by
 *                       bucket k is written.
 * Errors: ZERO_EINVAL (null plan/pointers, k out of range, overlap between an output shard and
 * an input); ZERO_EALIGN; ZERO_ECUDA.
 * ---------------------------------------------------------------------------------------- */
zero_status zero_reduce_scatter_bucket(const zero_plan* plan, int k,
                                       const uint16_t* const* rank_grads,
                                       float* const* owner_grad_shards, uint32_t* d_status,
                                       zero_stream_t stream);

/* ------------------------------------------------------------------------------------------
 * Owner update of a shard (stages 1 and 2, unfused). "Como funciona": each process updates
 * only its part of the optimizer state; "ZeRO-2" card, "Gradient 생명주기": GPU r updates
 * parameter shard r from reduced-gradient shard r; "왜 all-gather는 그대로 필요한가": the
 * updated shards are gathered into every GPU's full parameters.
 *
 * If ZERO_FLAG_OVERFLOW (or ZERO_FLAG_TIMEOUT / ZERO_FLAG_BOUNDS: a reduce-scatter of the
 * step failed) is set in *d_status when the kernel runs, nothing is written except
 * ZERO_FLAG_SKIPPED into *d_status. Otherwise, in place, for i in [0, n):
 *   g = grad[i] / loss_scale
 *   m = beta1*m + (1-beta1)*g ;  v = beta2*v + (1-beta2)*(g*g)
 *   master = master - step_size * (m / (sqrt(v)/sqrt(1-beta2^t) + eps))
 *   param_out[i] = fp16(master), round to nearest even
 * every operation an IEEE fp32 operation rounded to nearest even, no fused multiply-add.
 *   grad, master, m, v : n fp32 each (device, 4-byte aligned; 16 bytes for the fast path)
 *   param_out          : n fp16 (device, 2-byte aligned), e.g. full_params + owner*S
 *   step               : t >= 1, the caller's counter (do not advance it on a skipped step)
 * Errors: ZERO_EINVAL (null pointers, t < 1, bad hyperparameters, overlapping arrays);
 * ZERO_EALIGN; ZERO_ECUDA. n == 0 launches nothing.
 * ---------------------------------------------------------------------------------------- */
zero_status zero_adam_shard(uint64_t n, const float* grad, float* master, float* m, float* v,
                            uint16_t* param_out, const zero_adam_hparams* hp, int64_t step,
                            uint32_t* d_status, zero_stream_t stream);

/* ------------------------------------------------------------------------------------------
 * Fused step: reduce-scatter + unscale + Adam + fp16 cast + all-gather write-back in one
 * pass, so the reduced gradient never reaches memory. Same arithmetic as the two calls above:
 *   red = (sum_{r=0..nd-1} fp32(rank_grads[r][i])) / nd, then the update of zero_adam_shard
 *   from (master_in, m_in, v_in)[i] into (master_out, m_out, v_out)[i], param_out[i] = fp16.
 * Inputs are never written, so a step with an inf/NaN anywhere can still be skipped after
 * the fact: call zero_step_commit once after the last zero_step_fused call of the step.
 * A step may be split into several calls (e.g. one per bucket) on disjoint ranges.
 * ZERO_FLAG_OVERFLOW is ORed into *d_status if any red is inf or NaN.
 *   n                 : elements in this call's range
 *   rank_grads        : nd device pointers (host array), each to n fp16 values of this range
 *   *_in / *_out      : n fp32 each; outputs must not overlap any input or each other
 *   param_out         : n fp16, e.g. full_params + flat offset of the range
 * Pointers must be aligned to their element size; when every gradient and state pointer is
 * 16-byte aligned the TMA-pipelined kernel runs, else a plain-load kernel.
 * Errors: ZERO_EINVAL (nd outside [1, 64], null pointers, t < 1, bad hyperparameters,
 * overlapping outputs); ZERO_EALIGN; ZERO_ECUDA. n == 0 launches nothing.
 * ---------------------------------------------------------------------------------------- */
zero_status zero_step_fused(uint64_t n, int nd, const uint16_t* const* rank_grads,
                            const float* master_in, const float* m_in, const float* v_in,
                            float* master_out, float* m_out, float* v_out, uint16_t* param_out,
                            const zero_adam_hparams* hp, int64_t step, uint32_t* d_status,
                            zero_stream_t stream);

/* zero_step_fused with the parameter all-gather in its epilogue. "ZeRO: particionar estados do
 * treino entre GPUs" (upskillscore.com), "Como funciona": the updated fp16 parameters of each
 * partition are all-gathered into every replica; "ZeRO-2" (llm-engineer.pages.dev), "왜
 * all-gather는 그대로 필요한가". Instead of one param_out, the kernel stores each fp16 value
 * into every replica: param_replicas is a host array of n_replicas (1..ZERO_MAX_RANKS) device
 * pointers, each to this range's n values in one replica's full parameter buffer (a peer
 * GPU's address where the replicas live on other GPUs, e.g. in NVLink-mapped symmetric memory;
 * plain stores, no multicast), pairwise disjoint and checked against the step's other buffers
 * like param_out. Same arithmetic, overflow flag and commit protocol as zero_step_fused; the
 * commit of such a step is zero_step_commit_replicas (a void step's repair reaches every
 * replica). Errors: as zero_step_fused, and ZERO_EINVAL for n_replicas outside 1..64, a null
 * array or entry, or overlapping replicas. */
zero_status zero_step_fused_replicas(uint64_t n, int nd, const uint16_t* const* rank_grads,
                                     const float* master_in, const float* m_in, const float* v_in,
                                     float* master_out, float* m_out, float* v_out,
                                     int n_replicas, uint16_t* const* param_replicas,
                                     const zero_adam_hparams* hp, int64_t step,
                                     uint32_t* d_status, zero_stream_t stream);

/* zero_step_commit for a step written with zero_step_fused_replicas: if the step is void, the
 * inputs are copied over the outputs and fp16(master_in) is written into every replica. Errors:
 * as zero_step_commit and zero_step_fused_replicas' replica checks. */
zero_status zero_step_commit_replicas(uint64_t n, const float* master_in, const float* m_in,
                                      const float* v_in, float* master_out, float* m_out,
                                      float* v_out, int n_replicas,
                                      uint16_t* const* param_replicas, uint32_t* d_status,
                                      zero_stream_t stream);

/* The calls of one step over several ranges (e.g. every bucket of a stage-1 step, in backward
 * order) as one call, so that a caller issuing many small calls pays one entry instead of one
 * per range. ranges[i] describes what zero_step_fused takes for range i (rank_grads: a host
 * array of nd device pointers). Every range is checked before anything is launched; then the
 * ranges are launched in order, exactly as `count` zero_step_fused calls on `stream` would be.
 * overlap != 0 declares them mutually independent, as a zero_overlap_begin/end region around
 * them would (the ranges of one step are: disjoint outputs, no output overlapping another
 * range's inputs); the library does not check that declaration. If a region is already open on
 * the stream, the calls join it. Errors: ZERO_EINVAL (count <
 * 0, null ranges, and anything zero_step_fused rejects for a range), ZERO_EALIGN, ZERO_ECUDA
 * (ranges before the failing one may have been launched). */
typedef struct {
    uint64_t n;
    const uint16_t* const* rank_grads;
    const float* master_in;
    const float* m_in;
    const float* v_in;
    float* master_out;
    float* m_out;
    float* v_out;
    uint16_t* param_out;
} zero_fused_range;

zero_status zero_step_fused_ranges(int nd, int count, const zero_fused_range* ranges,
                                   const zero_adam_hparams* hp, int64_t step, uint32_t* d_status,
                                   int overlap, zero_stream_t stream);

/* zero_adam_shard and zero_step_fused with the step's constants read from device memory when
 * the kernel runs (d_consts: a zero_adam_consts in device memory, 4-byte aligned), so that a
 * stream capture of a step (a CUDA graph) can be replayed for every step: before each replay
 * the caller copies that step's constants (zero_adam_consts_for_step) into *d_consts. Same
 * arithmetic and results as the calls above. Errors: as those calls (ZERO_EINVAL for a null
 * d_consts). */
zero_status zero_adam_shard_dc(uint64_t n, const float* grad, float* master, float* m, float* v,
                               uint16_t* param_out, const zero_adam_consts* d_consts,
                               uint32_t* d_status, zero_stream_t stream);
zero_status zero_step_fused_dc(uint64_t n, int nd, const uint16_t* const* rank_grads,
                               const float* master_in, const float* m_in, const float* v_in,
                               float* master_out, float* m_out, float* v_out,
                               uint16_t* param_out, const zero_adam_consts* d_consts,
                               uint32_t* d_status, zero_stream_t stream);

/* ------------------------------------------------------------------------------------------
 * Dynamic loss scaling on the device. The pages fix only a static picture (fp16 gradients,
 * mixed-precision Adam); this is the rule of Micikevicius et al., "Mixed Precision Training"
 * (ICLR 2018, section 3.2), as torch.cuda.amp.GradScaler states it: a step whose reduced
 * gradients overflow is skipped and the scale is multiplied by backoff_factor; after
 * growth_interval consecutive applied steps it is multiplied by growth_factor. Adam's t counts
 * applied steps only. Everything lives in device memory, so a step needs no host read:
 *   zero_scaler_prepare -> zero_step_fused_dc (per bucket) -> zero_step_commit
 *                       -> zero_scaler_update          (or ... zero_adam_shard_dc ... update)
 * and the whole sequence can be captured once as a CUDA graph.
 * ---------------------------------------------------------------------------------------- */
typedef struct {
    float scale;             /* the scale the next step's gradients carry */
    int32_t good_steps;      /* consecutive applied steps since the scale last changed */
    int64_t next_step;       /* Adam t of the next applied step (starts at 1) */
    int64_t skipped_steps;   /* steps skipped so far */
} zero_scaler_state;

typedef struct {
    float growth_factor;     /* e.g. 2 */
    float backoff_factor;    /* e.g. 0.5 */
    int32_t growth_interval; /* e.g. 2000, >= 1 */
} zero_scaler_params;

/* Host: out[i] = the constants of step first_step + i, i < count (as zero_adam_consts_for_step).
 * Copy the table to device memory for zero_scaler_prepare. Errors: ZERO_EINVAL. */
zero_status zero_adam_consts_table(const zero_adam_hparams* hp, int64_t first_step, int64_t count,
                                   zero_adam_consts* out);

/* Device, first call of a step: *d_status = 0 and *d_consts = d_table[t - 1] with t =
 * d_state->next_step and the loss scale replaced by d_state->scale. If t is outside
 * [1, table_len] the step is refused: *d_status = ZERO_FLAG_OVERFLOW | ZERO_FLAG_BOUNDS, so the
 * step's kernels skip it, zero_scaler_update leaves the scaler alone and zero_step_status
 * reports ZERO_ECUDA. All pointers device memory; d_state 8-byte aligned, the others 4.
 * Errors: ZERO_EINVAL (null, table_len < 1), ZERO_EALIGN, ZERO_ECUDA. */
zero_status zero_scaler_prepare(const zero_scaler_state* d_state, const zero_adam_consts* d_table,
                                int64_t table_len, zero_adam_consts* d_consts, uint32_t* d_status,
                                zero_stream_t stream);

/* Device, after the step's last kernel (zero_step_commit or the last zero_adam_shard_dc):
 * if *d_status has ZERO_FLAG_OVERFLOW the scale is multiplied by backoff_factor, good_steps
 * reset and skipped_steps counted; otherwise next_step and good_steps advance and the scale is
 * multiplied by growth_factor when good_steps reaches growth_interval. A status with
 * ZERO_FLAG_TIMEOUT or ZERO_FLAG_BOUNDS leaves the scaler unchanged.
 * Errors: ZERO_EINVAL (null pointers, growth_interval < 1, non-finite or non-positive
 * factors), ZERO_EALIGN, ZERO_ECUDA. */
zero_status zero_scaler_update(zero_scaler_state* d_state, const zero_scaler_params* params,
                               const uint32_t* d_status, zero_stream_t stream);

/* Close a step made of zero_step_fused calls, on the same stream, over the same range(s).
 * If ZERO_FLAG_OVERFLOW, ZERO_FLAG_TIMEOUT or ZERO_FLAG_BOUNDS is set (a gradient overflowed,
 * or a kernel of the step gave up and left part of its outputs unwritten):
 * (master_out, m_out, v_out) = (master_in, m_in, v_in), param_out = fp16(master_in), and
 * ZERO_FLAG_SKIPPED is set -- the step did not happen, and the fp16 parameters of the range
 * are restored too. Otherwise nothing is written. Either way the caller may then swap the
 * in/out buffers (zero_step_status still reports ZERO_ECUDA for the error bits).
 * Errors: as zero_step_fused. */
zero_status zero_step_commit(uint64_t n, const float* master_in, const float* m_in,
                             const float* v_in, float* master_out, float* m_out, float* v_out,
                             uint16_t* param_out, uint32_t* d_status, zero_stream_t stream);

/* Wait for `stream`, read *d_status into *flags_out (may be NULL) and map it to a status:
 * ZERO_STEP_SKIPPED if ZERO_FLAG_SKIPPED is set, ZERO_ECUDA if ZERO_FLAG_TIMEOUT or ZERO_FLAG_BOUNDS is
 * set or the copy fails, else ZERO_OK. This is the only call that blocks the host. */
zero_status zero_step_status(const uint32_t* d_status, zero_stream_t stream, uint32_t* flags_out);

/* ------------------------------------------------------------------------------------------
 * Stage 3 (Pos+g+p): the fp16 parameters are partitioned too. "Como funciona": a process that
 * needs a partition it does not own receives it from the owner; a step moves 3 psi -- a
 * parameter all-gather in the forward pass, another in the backward pass, and the gradient
 * reduce-scatter. "ZeRO" (lastdictionary.com), main definition: each layer's parameters are
 * gathered just in time for its computation and discarded afterwards.
 * Owner q's parameter partition is its own buffer of S fp16 values (flat elements
 * [q*S, (q+1)*S) of the plan's padded list); param_shards is a host array of the nd device
 * pointers. A step: for every layer in forward order zero_gather_params; for every layer in
 * backward order zero_gather_params, then zero_stage3_step_fused over the layer's gradient
 * bucket (its reduce-scatter, unscale, Adam, and the fp16 cast into the owners' partitions) --
 * the layer's range, the last layer's extended to psi_padded so that the zero padding is
 * updated as in stages 1 and 2 (the backward pass produces the end of the flat list first);
 * then zero_stage3_step_commit. Optimizer state as in stages 1-2: flat fp32 arrays, owner q's part at q*S.
 * ---------------------------------------------------------------------------------------- */

/* The just-in-time all-gather of one layer: out[i] = element flat_lo + i of the parameters,
 * taken from the partition of its owner, for i in [0, len); out stands for every rank's
 * gathered copy. A pure copy (bit-exact). out: len fp16 values, 2-byte aligned (16-byte
 * aligned stores after the first few elements); the partitions 2-byte aligned (each owner's
 * segment takes 16-, 4- or 2-byte loads by its alignment). d_status: the bounds self-check
 * bit. Errors: ZERO_EINVAL (null plan/pointers of an owner the range touches, range beyond
 * psi_padded, out overlapping a partition or the status word), ZERO_EALIGN, ZERO_ECUDA.
 * len == 0 launches nothing. */
zero_status zero_gather_params(const zero_plan* plan, uint64_t flat_lo, uint64_t len,
                               const uint16_t* const* param_shards, uint16_t* out,
                               uint32_t* d_status, zero_stream_t stream);

/* The owners' update of the flat range [flat_lo, flat_lo + len) (one layer's gradient bucket,
 * in backward order): zero_step_fused over each owner's part of the range, with that part's
 * fp16 values written into the owner's partition (param_shards[q] + (a - q*S) for the part
 * starting at flat element a). rank_grads: nd device pointers to the range's len fp16 local
 * gradients; master_in ... v_out: device pointers to the range's first element of the flat
 * fp32 arrays. Same arithmetic, overflow flag and commit protocol as zero_step_fused. Every
 * part is checked before any is launched. Errors: as zero_step_fused, and ZERO_EINVAL for a
 * range beyond psi_padded or overlapping partitions. */
zero_status zero_stage3_step_fused(const zero_plan* plan, uint64_t flat_lo, uint64_t len,
                             const uint16_t* const* rank_grads, const float* master_in,
                             const float* m_in, const float* v_in, float* master_out,
                             float* m_out, float* v_out, uint16_t* const* param_shards,
                             const zero_adam_hparams* hp, int64_t step, uint32_t* d_status,
                             zero_stream_t stream);

/* zero_stage3_step_fused with the step's constants read from device memory when the kernels
 * run (d_consts: a zero_adam_consts, 4-byte aligned, e.g. copied in before each replay or
 * written by zero_scaler_prepare), as zero_step_fused_dc is for zero_step_fused: a stage-3
 * step -- the layer scheduler's gathers, these updates and the commit -- can then be captured
 * once as a CUDA graph and replayed for every step. Same results as the by-value call with the
 * same constants. Errors: as zero_stage3_step_fused, and ZERO_EINVAL / ZERO_EALIGN for
 * d_consts. */
zero_status zero_stage3_step_fused_dc(const zero_plan* plan, uint64_t flat_lo, uint64_t len,
                                      const uint16_t* const* rank_grads, const float* master_in,
                                      const float* m_in, const float* v_in, float* master_out,
                                      float* m_out, float* v_out, uint16_t* const* param_shards,
                                      const zero_adam_consts* d_consts, uint32_t* d_status,
                                      zero_stream_t stream);

/* Close a stage-3 step: zero_step_commit on every owner's part, over the whole padded list
 * (master_in ... v_out: the flat fp32 arrays, psi_padded values each), the fp16 values of a
 * voided step restored into each owner's partition. Errors: as zero_step_commit. */
zero_status zero_stage3_step_commit(const zero_plan* plan, const float* master_in, const float* m_in,
                              const float* v_in, float* master_out, float* m_out, float* v_out,
                              uint16_t* const* param_shards, uint32_t* d_status,
                              zero_stream_t stream);

/* ------------------------------------------------------------------------------------------
 * Just-in-time layer scheduler for stage 3. "ZeRO" (lastdictionary.com), main definition: each
 * layer's parameters are gathered just in time for its computation and discarded afterwards;
 * "Como funciona": a partition a process does not own is received from its owner, once in the
 * forward pass and again in the backward pass. The scheduler runs the gathers
 * (zero_gather_params' kernel) on its own gather stream into a pool of n_bufs layer buffers and
 * orders everything with CUDA events, so the host never blocks:
 *   zero_layer_sched_begin_step(s, d_status, stream)   once per step, on the stream that ran the
 *                                                        previous step's updates and commit
 *   for each layer l of the pass:
 *     zero_layer_sched_acquire(s, l, next, compute, &p) layer l's fp16 values at p (compute waits
 *                                                        for the gather); `next`'s gather starts
 *     ... the layer's computation on `compute` reads p ...
 *     zero_layer_sched_release(s, l, compute)           p may be overwritten after this point
 * and in the backward pass, after release(l), the layer's update (zero_stage3_step_fused over
 * its gradient bucket) on the compute stream; then zero_stage3_step_commit. A gather and the
 * updates beside it touch disjoint ranges of the partitions as long as each layer's update
 * covers only its own range (the last layer's extended over the padding).
 *   layer_bounds : n_layers + 1 flat offsets, 0 = b[0] < b[1] < ... < b[n_layers], with
 *                  psi <= b[n_layers] <= psi_padded; layer l is [b[l], b[l+1]) (copied)
 *   param_shards : the nd owners' partitions, S fp16 values each, 2-byte aligned (copied)
 *   buf_mem      : zero_layer_sched_buf_elems(...) fp16 values of caller device memory, 16-byte
 *                  aligned, not overlapping a partition: n_bufs buffers of the longest layer
 *                  rounded up to 8 values. n_bufs >= 2 lets one gather run ahead; with more
 *                  buffers the gather stream waits for the compute stream less often (one wait
 *                  covers every buffer released on that stream so far).
 * A released layer is discarded (acquiring it again gathers it again); a prefetched layer that
 * is not acquired before its buffer is needed is dropped; begin_step drops every layer still
 * in a buffer (the partitions have changed since). The plan, the partitions and buf_mem must
 * outlive the scheduler; one host thread at a time may use it. A step can be captured into a
 * CUDA graph (with zero_stage3_step_fused_dc for the updates): capture it on one stream, pass
 * that stream to begin_step, acquire and release, so that the gather stream joins the capture
 * through begin_step's event and every wait stays inside the capture; acquire every layer the
 * captured step prefetches (an unused prefetch's gather would not be joined back into the
 * capturing stream, and CUDA refuses to end such a capture). The pages have no
 * scheduler interface; this is the library's runtime for the stage-3 data path.
 * Errors: ZERO_EINVAL (bad plan or bounds, null pointers, an acquire before the first
 * begin_step, a layer out of range or already acquired, release of a layer not acquired,
 * begin_step while a layer is acquired, a status word inside a partition or the buffers),
 * ZERO_EALIGN, ZERO_ENOMEM (buf_mem too small, every buffer holding an acquired layer, host
 * allocation), ZERO_ECUDA (event or launch failure).
 * ---------------------------------------------------------------------------------------- */
typedef struct zero_layer_sched zero_layer_sched;

zero_status zero_layer_sched_buf_elems(const zero_plan* plan, int n_layers,
                                       const uint64_t* layer_bounds, int n_bufs,
                                       uint64_t* elems);
zero_status zero_layer_sched_create(const zero_plan* plan, int n_layers,
                                    const uint64_t* layer_bounds,
                                    const uint16_t* const* param_shards, uint16_t* buf_mem,
                                    uint64_t buf_mem_elems, int n_bufs,
                                    zero_stream_t gather_stream, zero_layer_sched** out);
/* Start a step: its gathers OR their bounds flag into d_status (4-byte aligned) and wait for
 * the work enqueued on `stream` so far. */
zero_status zero_layer_sched_begin_step(zero_layer_sched* s, uint32_t* d_status,
                                        zero_stream_t stream);
/* Make `compute` wait until layer `layer` is gathered (gathering it now unless a prefetch
 * already did) and write its buffer's address to *layer_params; then, if 0 <= prefetch <
 * n_layers and a buffer is free, start the gather of layer `prefetch`. */
zero_status zero_layer_sched_acquire(zero_layer_sched* s, int layer, int prefetch,
                                     zero_stream_t compute, uint16_t** layer_params);
/* Layer `layer`'s readers are enqueued on `compute`: its buffer is free after them. */
zero_status zero_layer_sched_release(zero_layer_sched* s, int layer, zero_stream_t compute);
/* Number of gathers the scheduler has launched since creation. */
zero_status zero_layer_sched_gathers(const zero_layer_sched* s, uint64_t* count);
void zero_layer_sched_destroy(zero_layer_sched* s);

/* ------------------------------------------------------------------------------------------
 * Compressed reduce-scatter payload. "ZeRO" (lastdictionary.com), main definition: extensions
 * compress the communication (ZeRO++). The pages give no format; this library's: each rank's
 * slice travels as 8-bit values with one fp32 scale per block of ZERO_Q8_BLOCK elements
 * (blocks counted from the slice's first element), and the owner accumulates q*scale with
 * fused multiply-adds:
 *   scale = amax/127 (binary32), q = round_half_even(x/scale) clamped to [-127, 127],
 *   a block with an inf or NaN gets scale NaN and q = 0 (so the owner sees the overflow);
 *   q is stored as the unsigned byte q + 128 (offset binary, 1..255; 128 is q = 0).
 * ---------------------------------------------------------------------------------------- */
#define ZERO_Q8_BLOCK 128
#define ZERO_Q8_RECORD 132   /* bytes per block: 128 bytes q + 128, then the fp32 scale */

/* Bytes of the payload of n elements: ceil(n/128) records of 132 bytes. */
#define ZERO_Q8_PAYLOAD_BYTES(n) ((((uint64_t)(n) + 127u) / 128u) * 132u)

/* Quantize one rank's n fp16 gradients into its payload: record b holds q + 128 of elements
 * [128b, 128b+128) in bytes 0..127 (unused bytes of a short last block are 128) and the block's
 * scale in bytes 128..131. Device memory; payload 4-byte aligned (16 for the bulk-copy path of
 * zero_step_fused_q8). Errors: ZERO_EINVAL (null, overlap), ZERO_EALIGN, ZERO_ECUDA. */
zero_status zero_quantize_q8(uint64_t n, const uint16_t* grad, uint8_t* payload,
                             zero_stream_t stream);

/* zero_step_fused with int8 payloads: s = fma(float(q_r[i]), scale_r[i/128], s) for r = 0..nd-1
 * (each a binary32 fused multiply-add, one rounding), red = s/nd, then the same update, overflow
 * flag and commit protocol as zero_step_fused. rank_payload: nd device pointers (host array),
 * each to this range's ZERO_Q8_PAYLOAD_BYTES(n) bytes as zero_quantize_q8 wrote them (records
 * counted from the range's first element). 16-byte aligned payload and state pointers (and
 * n >= 4096) take the bulk-copy kernel. Errors: as zero_step_fused. */
zero_status zero_step_fused_q8(uint64_t n, int nd, const uint8_t* const* rank_payload,
                               const float* master_in, const float* m_in, const float* v_in,
                               float* master_out, float* m_out, float* v_out,
                               uint16_t* param_out, const zero_adam_hparams* hp, int64_t step,
                               uint32_t* d_status, zero_stream_t stream);

/* The int8 payload for stage 3's per-layer gradient reduce-scatter. A layer's range is split
 * at owner boundaries (as zero_stage3_step_fused splits it); a rank's payload for the range is
 * one segment per owner part, in owner order, each holding the part's records counted from the
 * part's first element (ZERO_Q8_PAYLOAD_BYTES(part length)) and rounded up to 16 bytes.
 * zero_stage3_payload_bytes_q8 gives the total; zero_stage3_quantize_q8 writes one rank's len
 * fp16 gradients of the range into that layout (grad 2-byte aligned, payload 16-byte aligned,
 * not overlapping); zero_stage3_step_fused_q8 is zero_stage3_step_fused with the nd ranks'
 * payloads (host array of nd device pointers) in place of their fp16 gradients, each part
 * reduced as zero_step_fused_q8 reduces it. Errors: as zero_stage3_step_fused and
 * zero_quantize_q8. */
zero_status zero_stage3_payload_bytes_q8(const zero_plan* plan, uint64_t flat_lo, uint64_t len,
                                         uint64_t* bytes);
zero_status zero_stage3_quantize_q8(const zero_plan* plan, uint64_t flat_lo, uint64_t len,
                                    const uint16_t* grad, uint8_t* payload, zero_stream_t stream);
zero_status zero_stage3_step_fused_q8(const zero_plan* plan, uint64_t flat_lo, uint64_t len,
                                      const uint8_t* const* rank_payload, const float* master_in,
                                      const float* m_in, const float* v_in, float* master_out,
                                      float* m_out, float* v_out, uint16_t* const* param_shards,
                                      const zero_adam_hparams* hp, int64_t step,
                                      uint32_t* d_status, zero_stream_t stream);
/* zero_stage3_step_fused_q8 with the step's constants read from device memory (d_consts, as
 * for zero_stage3_step_fused_dc), so that a stage-3 step from int8 payloads is captured once
 * as a CUDA graph. Errors: as zero_stage3_step_fused_q8, and ZERO_EINVAL / ZERO_EALIGN for
 * d_consts. */
zero_status zero_stage3_step_fused_q8_dc(const zero_plan* plan, uint64_t flat_lo, uint64_t len,
                                         const uint8_t* const* rank_payload,
                                         const float* master_in, const float* m_in,
                                         const float* v_in, float* master_out, float* m_out,
                                         float* v_out, uint16_t* const* param_shards,
                                         const zero_adam_consts* d_consts, uint32_t* d_status,
                                         zero_stream_t stream);

/* The int8 calls of one step over several ranges as one call, as zero_step_fused_ranges is for
 * zero_step_fused: ranges[i] describes what zero_step_fused_q8 takes for range i (rank_payload:
 * a host array of nd device pointers, each to that range's records). Every range is checked
 * before anything is launched; then the ranges are launched in order, exactly as `count`
 * zero_step_fused_q8 calls on `stream` would be. overlap != 0 declares them mutually
 * independent (not checked); a region already open on the stream is joined. Errors: ZERO_EINVAL
 * (count < 0, null ranges, and anything zero_step_fused_q8 rejects for a range), ZERO_EALIGN,
 * ZERO_ECUDA (ranges before the failing one may have been launched). */
typedef struct {
    uint64_t n;
    const uint8_t* const* rank_payload;
    const float* master_in;
    const float* m_in;
    const float* v_in;
    float* master_out;
    float* m_out;
    float* v_out;
    uint16_t* param_out;
} zero_fused_q8_range;

zero_status zero_step_fused_q8_ranges(int nd, int count, const zero_fused_q8_range* ranges,
                                      const zero_adam_hparams* hp, int64_t step,
                                      uint32_t* d_status, int overlap, zero_stream_t stream);

/* zero_step_fused_q8 with the step's constants read from device memory (d_consts: a
 * zero_adam_consts, 4-byte aligned, e.g. written by zero_scaler_prepare), as
 * zero_step_fused_dc: the call can be captured in a CUDA graph and replayed for every step,
 * with dynamic loss scaling on the device. Same results, bit for bit, as the by-value call with
 * the same constants. Errors: as zero_step_fused_q8, and ZERO_EINVAL / ZERO_EALIGN for
 * d_consts. */
zero_status zero_step_fused_q8_dc(uint64_t n, int nd, const uint8_t* const* rank_payload,
                                  const float* master_in, const float* m_in, const float* v_in,
                                  float* master_out, float* m_out, float* v_out,
                                  uint16_t* param_out, const zero_adam_consts* d_consts,
                                  uint32_t* d_status, zero_stream_t stream);

/* Self-test of the kernels' bounded waits (failure detection without a fault): launches the
 * fused pipeline on one tile with its copy-issuing warp switched off, so every consumer's wait
 * on shared-memory data expires after about one second; the kernel then sets
 * ZERO_FLAG_TIMEOUT in *d_status and returns, and the CUDA context stays usable. No other
 * memory is read or written. The pages have no counterpart; it checks this library's own
 * error path. Errors: ZERO_EINVAL (null), ZERO_EALIGN, ZERO_ECUDA. */
zero_status zero_selftest_timeout(uint32_t* d_status, zero_stream_t stream);

/* ------------------------------------------------------------------------------------------
 * Overlap of independent calls on one stream. The bulk-copy kernels of zero_step_fused(_dc),
 * zero_step_fused_q8 and zero_reduce_scatter_bucket are launched with programmatic stream
 * serialization: their CTAs may be scheduled while the kernel before them on the stream
 * drains, but by default each waits for that kernel to complete before it touches global
 * memory, so stream order is kept exactly.
 * Between zero_overlap_begin(stream) and zero_overlap_end(stream) the caller declares those
 * calls on `stream` mutually independent: none writes memory that another one of them reads
 * or writes, except the shared status word, into which they only OR flags. The per-bucket
 * calls of one step are such a set (disjoint ranges). Every such call after the region's first
 * may then run alongside the calls before it, and each completes only after all earlier ones,
 * so work enqueued after the region (zero_step_commit, a copy, an event) is ordered after the
 * whole region as usual. Calls that take the plain-load kernels, and all other calls, stay
 * ordered. Other work enqueued on the stream inside the region must be ordinary launches,
 * copies, event records or event waits (a kernel that itself uses programmatic dependent
 * launch, as some libraries' kernels do, needs the region closed before it); an event recorded
 * after a call completes only when that call and every call before it have. The bucket
 * scheduler's calls (zero_sched_end_bucket on its stream) may sit in a region.
 * Host-side state only (one flag per stream, thread-safe): both calls enqueue nothing and can
 * be used while a CUDA graph is captured. Close a region before its stream is destroyed (the
 * flag is keyed by the stream handle, which a later stream may reuse); at most 64 regions are
 * open at once. The launch path reads the flags without a lock. The pages have no counterpart;
 * this is a launch device of this library. Errors: ZERO_EINVAL (begin on a stream whose region
 * is open, end on a stream without one), ZERO_ENOMEM (64 regions already open).
 * ---------------------------------------------------------------------------------------- */
zero_status zero_overlap_begin(zero_stream_t stream);
zero_status zero_overlap_end(zero_stream_t stream);

/* ------------------------------------------------------------------------------------------
 * Stream-ordered bucket scheduler for stage 2. "ZeRO-2" card, "Gradient 생명주기": after a
 * bucket's reduce-scatter the GPU keeps its own reduced shard and releases the rest of the
 * local gradient. The local gradients of a bucket live in a staging slot (nd regions of
 * slot_stride fp16 values, slot_stride = the longest bucket rounded up to 8 elements); the
 * reduce-scatter runs on rs_stream once the producer has filled the slot, and the slot is
 * released (reused by a later bucket) when that reduce-scatter has finished -- all ordered by
 * CUDA events, without blocking the host.
 *   slot_mem          : n_slots*nd*slot_stride fp16 values of caller device memory, 16-byte
 *                       aligned (zero_sched_slot_elems gives the count)
 *   owner_grad_shards : nd device pointers (copied), as for zero_reduce_scatter_bucket
 *   d_status          : the step's status word
 * The scheduler keeps the plan's address and the slot memory: both must outlive it; one host
 * thread at a time may use a scheduler.
 * Errors: ZERO_EINVAL, ZERO_EALIGN, ZERO_ENOMEM (slot_mem too small or host allocation),
 * ZERO_ECUDA (event creation).
 * ---------------------------------------------------------------------------------------- */
typedef struct zero_sched zero_sched;

zero_status zero_sched_slot_elems(const zero_plan* plan, int n_slots, uint64_t* elems);
zero_status zero_sched_create(const zero_plan* plan, uint16_t* slot_mem, uint64_t slot_mem_elems,
                              int n_slots, float* const* owner_grad_shards, uint32_t* d_status,
                              zero_stream_t rs_stream, zero_sched** out);
/* Fused mode: the kernel launched for bucket k (on `stream`) is the fused step over the
 * bucket's range [lo, lo+len) of the flat padded buffer -- rank-ordered reduction, unscale,
 * Adam, fp16 cast and write-back, as zero_step_fused_dc with the step's constants read from
 * d_consts -- so the reduced gradient never reaches memory (the fused step applied to stage 2
 * bucket by bucket, with the same release of each slot after its kernel). master_in/m_in/v_in
 * and master_out/m_out/v_out: psi_p fp32 values each (flat, padded), param_out: psi_p fp16
 * values; zero_sched_rebind_fused points a later step at other buffers (ping-pong state), so
 * one scheduler serves every step. After the last bucket the caller makes its stream wait
 * (zero_sched_wait) and calls
 * zero_step_commit over all psi_p elements, which skips the whole step if any bucket
 * overflowed. Errors: as zero_sched_create, and ZERO_EINVAL for outputs that overlap the
 * inputs, each other or the staging slots. The pages' stage 2 keeps the reduced shard in
 * memory for a later optimizer step; this mode is this library's fusion of the two. */
zero_status zero_sched_create_fused(const zero_plan* plan, uint16_t* slot_mem,
                                    uint64_t slot_mem_elems, int n_slots, const float* master_in,
                                    const float* m_in, const float* v_in, float* master_out,
                                    float* m_out, float* v_out, uint16_t* param_out,
                                    const zero_adam_consts* d_consts, uint32_t* d_status,
                                    zero_stream_t stream, zero_sched** out);
/* The int8 payload in the bucket pipeline. "ZeRO" (lastdictionary.com), main definition:
 * ZeRO++ compresses the communication; the format is ZERO_Q8_BLOCK-value records (below).
 * Fused mode with each rank's part of a bucket arriving as int8 records: the staging slots
 * hold, per rank, ZERO_Q8_PAYLOAD_BYTES(len) bytes of records counted from the bucket's first
 * element (as zero_quantize_q8 writes them for the rank's len values of the bucket), in
 * regions of the longest bucket's record bytes rounded up to 16; the kernel launched for
 * bucket k is zero_step_fused_q8_dc over the bucket's range. slot_mem: 16-byte aligned,
 * zero_sched_slot_bytes_q8(...) bytes. The producer fills the regions that
 * zero_sched_begin_bucket_q8 returns (zero_sched_begin_bucket is rejected for such a
 * scheduler, and zero_sched_begin_bucket_q8 for the others). Rebind, wait and commit as in the
 * fp16 fused mode. Errors: as zero_sched_create_fused. */
zero_status zero_sched_slot_bytes_q8(const zero_plan* plan, int n_slots, uint64_t* bytes);
zero_status zero_sched_create_fused_q8(const zero_plan* plan, uint8_t* slot_mem,
                                       uint64_t slot_mem_bytes, int n_slots,
                                       const float* master_in, const float* m_in,
                                       const float* v_in, float* master_out, float* m_out,
                                       float* v_out, uint16_t* param_out,
                                       const zero_adam_consts* d_consts, uint32_t* d_status,
                                       zero_stream_t stream, zero_sched** out);
zero_status zero_sched_begin_bucket_q8(zero_sched* s, int k, zero_stream_t producer,
                                       uint8_t** rank_ptrs);
/* Between steps: point the fused scheduler at the next step's state, parameters and status
 * word (same layout and checks as zero_sched_create_fused), e.g. the swapped ping-pong buffers.
 * Kernels already enqueued keep the old pointers; the CUDA events and slots are reused, so a
 * step through a rebound scheduler creates nothing. Errors: ZERO_EINVAL (not a fused
 * scheduler, a bucket begun and not ended, null or overlapping buffers), ZERO_EALIGN. */
zero_status zero_sched_rebind_fused(zero_sched* s, const float* master_in, const float* m_in,
                                    const float* v_in, float* master_out, float* m_out,
                                    float* v_out, uint16_t* param_out, uint32_t* d_status);
/* Between steps, either mode: later bucket kernels OR their flags into d_status (e.g. one
 * status word per step). Errors: ZERO_EINVAL (null, a bucket begun and not ended, d_status
 * inside a buffer the kernels write or the slots), ZERO_EALIGN. */
zero_status zero_sched_rebind_status(zero_sched* s, uint32_t* d_status);
/* Choose the slot for bucket k, make `producer` wait until that slot is released, and write
 * the nd device pointers (rank r's region, bucket k's len values) the producer must fill.
 * ZERO_EINVAL if k is out of range or the slot holds a bucket that was begun and not yet
 * ended (with n_slots slots, bucket k and bucket k + n_slots share one). */
zero_status zero_sched_begin_bucket(zero_sched* s, int k, zero_stream_t producer,
                                    uint16_t** rank_ptrs);
/* The producer has enqueued the fill of bucket k on `producer`: the bucket's kernel (the
 * reduce-scatter, or the fused step in fused mode) is enqueued on the scheduler's stream after
 * it, followed by the release of its slot. */
zero_status zero_sched_end_bucket(zero_sched* s, int k, zero_stream_t producer);
/* Make `stream` wait for every reduce-scatter enqueued so far (e.g. before zero_adam_shard). */
zero_status zero_sched_wait(zero_sched* s, zero_stream_t stream);
/* Number of bucket kernels (reduce-scatter or fused) the scheduler has launched since creation. */
zero_status zero_sched_launches(const zero_sched* s, uint64_t* count);
void zero_sched_destroy(zero_sched* s);

#ifdef __cplusplus
}
#endif

#endif /* LIBZERO_H */
