/*
 * neox_shard.h -- C ABI of libneoxshard.so: the per-rank mixed-precision
 * optimizer step over an owned flat shard, as hand-written CUDA for sm_100a.
 *
 * What the step computes (pages, by title and section):
 *  - "GPT-NeoX: how it opened the door to democratised 100B-scale training"
 *    (ainews.cool), section "技术深度解析" (technical deep-dive): with ZeRO
 *    stage 1 the optimizer state is partitioned across the data-parallel
 *    ranks and each device updates only the shard it owns.  One handle of
 *    this library is one such shard on one GPU.
 *  - "OPT: Open Pre-trained Transformer Language Models" (ai-papers.xuzou.cn
 *    summary), section "计算设置" (compute setup): Adam state in FP32, sharded;
 *    weights in FP16; dynamic loss scaling against underflow.
 *  - same page, section "瓶颈" (bottlenecks): about 16 bytes of model state
 *    per parameter (FP16 weight + FP16 grad + FP32 master, m, v).
 *  - same page, section "方法适配" (method adaptation): a gradient pre-divide
 *    factor, global-norm gradient clipping at 1.0 or 0.3, and resetting the
 *    dynamic loss scaler / restarting from a checkpoint where it is healthy.
 *  - The pages never write Adam out; the update is the textbook AdamW
 *    (Loshchilov & Hutter, decoupled weight decay) with bias correction.
 *
 * One call of neox_shard_step, for K gradient buffers g_0..g_{K-1} (16-bit,
 * numel elements each) carrying the current loss scale S:
 *   1. g_i = fl32( (sum_k fl32(g_k,i * fl32(1/predivide))) * fl32(1/(post*S)) ),
 *      post = K/predivide, the sum taken in buffer order in FP32;
 *   2. overflow = any g_i not finite (or the norm not finite);
 *   3. norm = sqrt(sum_i g_i^2)  (pre-clip, unscaled);
 *   4. loss scaler: overflow -> counter = 0, skip, and the hysteresis count
 *      H drops by one (not below 0); when it is 0, S = max(S/factor,
 *      min_scale); applied -> counter+1, at scale_window S = S*factor (if
 *      finite), counter = 0, H = max(hysteresis, 1).  With hysteresis 0 or 1
 *      every overflow lowers the scale;
 *   5. unless skipped: t = t+1; c = clip/(norm+1e-6) if that is < 1 (else 1);
 *      for every element: gh = g*c; m = b1*m + (1-b1)*gh; v = b2*v + (1-b2)*gh*gh;
 *      p = p*(1 - lr*wd_seg) - (lr/bc1) * m / (sqrt(v)/sqrt(bc2) + eps),
 *      bc1 = 1-b1^t, bc2 = 1-b2^t; w = RNE16(p).
 *      With optimizer = NEOX_SGD the update is instead plain SGD with the
 *      same decoupled decay, p = p*(1 - lr*wd_seg) - lr*gh, and m, v are
 *      neither read nor written (same page, "方法适配": SGD was tried in
 *      place of Adam).
 *
 * Threading: a handle is used by one host thread at a time.  Different
 * handles are independent.  All functions are host functions.
 */
#ifndef NEOX_SHARD_H
#define NEOX_SHARD_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    NEOX_OK = 0,
    NEOX_ERR_INVALID_ARGUMENT = 1, /* nothing launched, no state changed      */
    NEOX_ERR_CUDA = 2,             /* a CUDA call failed; see neox_last_error */
    NEOX_ERR_OUT_OF_MEMORY = 3,    /* device or pinned allocation failed      */
    NEOX_ERR_UNSUPPORTED = 4       /* e.g. the device is not sm_100           */
} neox_status;

typedef enum { NEOX_FP16 = 0, NEOX_BF16 = 1 } neox_dtype;

/* A run of elements [offset, offset+numel) with its own weight decay (biases
 * and LayerNorm parameters typically use 0).  A table must be sorted by
 * offset and tile [0, numel) exactly, each segment non-empty. */
typedef struct {
    uint64_t offset;
    uint64_t numel;
    float weight_decay;
} neox_segment;

/* The update rule of pass 2. */
typedef enum { NEOX_ADAMW = 0, NEOX_SGD = 1 } neox_optimizer;

typedef struct {
    float beta1, beta2;   /* in [0, 1)                                      */
    float eps;            /* >= 0                                           */
    float clip_norm;      /* global-norm clip; <= 0 disables clipping       */
    float predivide;      /* > 0; each buffer is scaled by 1/predivide
                             before the sum, the sum by predivide/K after    */
    float init_scale;     /* > 0: the loss scale at create                  */
    float scale_factor;   /* >= 1: backoff divisor and growth multiplier    */
    float min_scale;      /* >= 0: floor of the scale after a backoff       */
    int32_t scale_window; /* >= 1: applied steps between growths            */
    int32_t hysteresis;   /* >= 0: overflows since the last growth (or
                             create / set_state) before the scale is
                             lowered; 0 or 1 = at every overflow           */
    int32_t optimizer;    /* neox_optimizer; 0 = NEOX_ADAMW                 */
} neox_hparams;

/* The shard.  numel may be 0 (a rank that owns nothing still takes part in
 * the scaler).  master / exp_avg / exp_avg_sq are caller-owned device FP32
 * arrays of numel elements (NULL allowed only when numel == 0); they must be
 * 4-byte aligned and must outlive the handle.  The caller initialises them
 * (typically m = v = 0) and the 16-bit working weights to RNE16(master). */
typedef struct {
    uint64_t numel;
    neox_dtype wdtype;            /* working-weight type (params of the step) */
    neox_dtype gdtype;            /* gradient type                            */
    const neox_segment* segs;     /* host array; NULL = one segment [0,numel)  */
    int32_t nsegs;
    float default_weight_decay;   /* weight decay when segs == NULL           */
    float* master;
    float* exp_avg;
    float* exp_avg_sq;
    int32_t max_grads;            /* largest K the caller will pass (0 = 1);
                                     K >= 5 makes create reserve numel*4 bytes
                                     of FP32 scratch so pass 2 reads one FP32
                                     sum instead of re-reading K buffers       */
    int32_t flags;                /* 0 or NEOX_SHARD_ACCUMULATE                */
} neox_shard_desc;

/* neox_shard_desc.flags: reserve the FP32 sum buffer whatever max_grads is,
 * and use it at every K: pass 1 writes the FP32 sum of the K buffers, pass 2
 * reads it instead of re-reading them.  Meant for gradient buffers in peer
 * memory (the ZeRO-2 form below), which pass 1 then reads over NVLink once. */
#define NEOX_SHARD_ACCUMULATE 1

typedef struct {
    int32_t overflow;          /* 1: non-finite gradient; the step was skipped */
    float grad_norm;           /* pre-clip L2 norm of the unscaled gradient;
                                  +inf when overflow                          */
    float clip_coef;           /* coefficient applied to the gradient (1 = no
                                  clipping); 0 when overflow                  */
    float loss_scale;          /* S that this step's gradients carried        */
    float loss_scale_next;     /* S to multiply the next loss by              */
    int32_t good_steps;        /* scaler counter after this step              */
    int64_t applied_steps;     /* t after this step                           */
} neox_step_result;

typedef struct neox_shard neox_shard;

/* Create a handle for one shard on CUDA device `device`.
 * Validates desc and hp (NEOX_ERR_INVALID_ARGUMENT on any violation, nothing
 * allocated), checks the device is compute capability 10.x (else
 * NEOX_ERR_UNSUPPORTED), copies the segment table to the device and allocates
 * the handle's scratch: a few KB of per-block partial sums, a 64-byte device
 * scalar block, a pinned 64-byte result slot, and (max_grads >= 5) an FP32
 * accumulation buffer of numel elements.  The loss scale starts at
 * hp->init_scale with zero counters.  *out is set only on NEOX_OK. */
neox_status neox_shard_create(const neox_shard_desc* desc, const neox_hparams* hp,
                              int device, neox_shard** out);

/* One optimizer step (steps 1-5 above) on cuda_stream (a cudaStream_t; NULL =
 * the legacy default stream).
 *   grads:     host array of num_grads DEVICE pointers, each to numel 16-bit
 *              gradients of desc->gdtype, 2-byte aligned, read only;
 *   num_grads: K in [1, 64];
 *   params:    DEVICE pointer to numel 16-bit working weights of
 *              desc->wdtype, 2-byte aligned, written only when the step is
 *              applied; must not overlap any other array;
 *   lr:        learning rate of this step, finite and >= 0;
 *   out:       host result, filled on NEOX_OK.
 * Arrays may start at any element offset: when every array has the same
 * element offset from a 1024-byte boundary the kernels peel a head of up to
 * 511 elements and stream from that common boundary with 16-byte vectors
 * (or the coarsest common 512-, 256- or 128-byte boundary); with only a
 * common 16-byte residue they peel less; otherwise they fall back to
 * narrower vectors.  The results are the same in every case.  The call is
 * stream-ordered and returns after the step has finished on the GPU (it
 * synchronises cuda_stream only).  Overflow is
 * not an error: it returns NEOX_OK with out->overflow = 1.  On
 * NEOX_ERR_INVALID_ARGUMENT nothing was launched; on NEOX_ERR_CUDA the shard
 * state is undefined. */
neox_status neox_shard_step(neox_shard* h, const void* const* grads, int32_t num_grads,
                            void* params, float lr, void* cuda_stream, neox_step_result* out);

/* The same step, enqueued on cuda_stream without waiting for it, so that a
 * training loop never blocks on the optimizer and a CUDA graph can capture it.
 * The differences from neox_shard_step:
 *   - nothing is read back to the host: the GPU writes the step's result into
 *     `result` (device memory or pinned host memory the caller owns, 8-byte
 *     aligned; NULL = not written) when pass 1 finishes;
 *   - the bias corrections bc1 = 1-b1^t, bc2 = 1-b2^t are formed on the GPU
 *     in double from the device copy of t (pow in double; the synchronous
 *     step forms them on the host), so the state agrees with the synchronous
 *     step within the step's tolerances rather than bit for bit;
 *   - when lr_device is non-NULL the learning rate is read from that device
 *     float at run time (a captured graph can then change it without
 *     re-capture) and `lr` is ignored;
 *   - profiling events are not recorded (launches are still counted).
 * It launches only kernels (no allocation, copy or synchronisation), so it can
 * be captured into a CUDA graph once the handle has run one step outside a
 * capture.  The arrays and `result` must stay valid until the step finishes.
 * Once a handle has issued an asynchronous step (whose graph replays the
 * library cannot see), its scaler state lives on the device only:
 * neox_shard_get_state and neox_shard_set_state then wait for the whole
 * device (cudaDeviceSynchronize) and read or write the device copy, and
 * neox_shard_step forms its bias corrections on the device as well. */
neox_status neox_shard_step_async(neox_shard* h, const void* const* grads, int32_t num_grads, void* params,
                                  float lr, const float* lr_device, void* cuda_stream, neox_step_result* result);

/* The step split around the one exchange data-parallel ranks need.
 *
 * With ZeRO stage 1/2 every rank owns one shard ("GPT-NeoX: how it opened the
 * door to democratised 100B-scale training" (ainews.cool), "技术深度解析"),
 * but the overflow flag and the global gradient norm -- hence the loss-scale
 * trajectory and the clip coefficient -- are properties of the whole model.
 * Each rank therefore runs:
 *   1. neox_shard_grad_stats: pass 1 over its shard; writes two doubles to
 *      stats_device: [0] = sum of squares of its unscaled gradients,
 *      [1] = 1.0 if any of them is not finite, else 0.0;
 *   2. an all-reduce (SUM) of those 16 bytes across the ranks, by the caller
 *      (e.g. NCCL through torch.distributed), on the same stream;
 *   3. neox_shard_apply: one single-thread kernel takes the step's decisions
 *      (overflow = [1] > 0, norm = sqrt([0]), scaler, clip coefficient, t)
 *      from the reduced statistics, then pass 2 updates the shard; it waits
 *      for the step and fills `out` like neox_shard_step.
 * Every rank then holds the same scale, counters and clip coefficient.  The
 * grads, num_grads and params of both calls must be the same (pass 2 re-reads
 * the gradients; params fixes the vector layout); stats_device is 8-byte
 * aligned device memory the caller owns.  With one rank (no all-reduce) the
 * two calls give exactly the result of neox_shard_step. */
neox_status neox_shard_grad_stats(neox_shard* h, const void* const* grads, int32_t num_grads, void* params,
                                  void* cuda_stream, double* stats_device);
neox_status neox_shard_apply(neox_shard* h, const void* const* grads, int32_t num_grads, void* params, float lr,
                             const double* stats_device, void* cuda_stream, neox_step_result* out);

/* Extra destinations of the updated 16-bit working weights, written by pass 2
 * with the same bytes as `params` (and never on a skipped step).  Under ZeRO
 * the updated weight shards are all-gathered to every rank ("GPT-NeoX: how it
 * opened the door to democratised 100B-scale training" (ainews.cool),
 * "技术深度解析": reduce-scatter / all-gather); given, for each peer, a
 * peer-mapped pointer to this rank's slice of that peer's full-weight buffer
 * (CUDA IPC or peer access over NVLink), the cast itself performs that
 * all-gather with direct stores, with no separate collective.  Any
 * device-accessible memory works (local buffers too).
 *   dsts: host array of n device pointers (2-byte aligned), n in [0, 8];
 *         n = 0 removes the copies.  Each destination receives numel elements.
 * The pointers must stay valid for every later step; the vector layout takes
 * them into account (a destination with another residue mod 16 bytes makes
 * the kernels use narrower vectors).  A destination in another rank's memory
 * is written without any ordering against that rank's own work: its reads of
 * the buffer must wait for this rank's step, and this rank's step must wait
 * for its earlier reads (the ordering rules of the ZeRO-2 section below). */
neox_status neox_shard_set_weight_copies(neox_shard* h, void* const* dsts, int32_t n);

/* ------------------------------------------------------------------------
 * ZeRO-2: the gradient reduce-scatter fused with pass 1, through CUDA IPC.
 *
 * Under ZeRO stage 2 every rank holds the full gradient of its own
 * micro-batches, and the owner of each flat slice needs the sum over the
 * ranks of that slice ("GPT-NeoX: how it opened the door to democratised
 * 100B-scale training" (ainews.cool), "技术深度解析": DP + ZeRO pairs with
 * reduce-scatter / all-gather; the OPT summary, "方法适配": the pre-divide is
 * applied before that cross-rank sum).  The step's K-buffer ingest is that
 * sum: pass neox_shard_step (or grad_stats / apply) the K = world-size
 * pointers peer_j + rank * slice_bytes, one per rank j, where peer_j is rank
 * j's full gradient buffer mapped into this process (neox_ipc_open; this
 * rank's own buffer directly).  Pass 1 then reads every rank's copy of this
 * rank's slice straight from its owner's HBM over NVLink, pre-divides, sums
 * in FP32 in rank order and reduces the norm, with no reduce-scatter
 * collective and no staging copy; with NEOX_SHARD_ACCUMULATE the FP32 sum
 * stays in local memory for pass 2.  The split step's 16-byte all-reduce
 * then gives every rank the same decision, and neox_shard_set_weight_copies
 * pointed at the peers' full-weight buffers performs the all-gather.
 *
 * Ordering between the ranks is the caller's.  The library orders work only
 * on the stream it is given and cannot see the peers' streams, so on every
 * rank's stream the caller must place:
 *   1. before the rank's pass 1 of a step (neox_shard_step or
 *      neox_shard_grad_stats): a point after which every rank's gradient
 *      buffer of that step is complete, because pass 1 reads the peers'
 *      buffers;
 *   2. after the rank's pass 2 (neox_shard_step or neox_shard_apply), before
 *      the rank writes its gradient buffer again (its next backward) or reads
 *      its full-weight buffer (its next forward): a point after which every
 *      rank's step has finished, because pass 1 -- and pass 2, which re-reads
 *      the gradients when no FP32 sum is kept (K < 5 without
 *      NEOX_SHARD_ACCUMULATE) -- reads this rank's gradient buffer, and every
 *      rank's pass 2 stores into this rank's full-weight buffer.
 * Both are barriers across the ranks' streams: a one-element all-reduce
 * (e.g. NCCL) enqueued on the step's stream, or interprocess events
 * (cudaIpcGetEventHandle / cudaIpcOpenEventHandle) that each rank records
 * on its stream and the others wait on with cudaStreamWaitEvent, once they
 * know the record has been issued (a wait refers to the last record issued
 * before it).  The statistics all-reduce between the passes is not such a
 * point for either.  The Python package's zero.zero2_step places both.
 *
 * The calls below wrap CUDA IPC (one node; handles are plain bytes that the
 * caller exchanges, e.g. with torch.distributed).  Errors: NEOX_ERR_CUDA
 * (message in neox_ipc_last_error(), per thread) or
 * NEOX_ERR_INVALID_ARGUMENT for NULL arguments.
 * ------------------------------------------------------------------------ */
typedef struct {
    unsigned char bytes[64];   /* a cudaIpcMemHandle_t, opaque */
} neox_ipc_handle;

/* Export the device allocation that contains dev_ptr: *handle names the whole
 * allocation (cudaMalloc'd memory; not stream-ordered or virtual-memory
 * allocations), *offset is dev_ptr's byte offset inside it. */
neox_status neox_ipc_export(const void* dev_ptr, neox_ipc_handle* handle, uint64_t* offset);
/* Map an allocation another process exported into this process's current
 * device (peer access enabled lazily); *base is its start: add the
 * exporter's offset.  A process cannot open a handle it exported itself, and
 * opens each handle once (share the mapping).  Close before the exporter
 * frees the memory. */
neox_status neox_ipc_open(const neox_ipc_handle* handle, void** base);
neox_status neox_ipc_close(void* base);
const char* neox_ipc_last_error(void);

/* Replace the hyperparameters (e.g. the clip 1.0 -> 0.3 change, or a switch
 * to NEOX_SGD); the current loss scale and counters are kept (init_scale is
 * ignored here), and so is the hysteresis count, which takes a new
 * `hysteresis` at the next growth or set_state.  Switching the optimizer
 * leaves m and v as they are. */
neox_status neox_shard_set_hparams(neox_shard* h, const neox_hparams* hp);

/* Scaler / step-count state, for checkpoint and resume.  Any pointer may be
 * NULL.  set_state validates scale > 0 finite, good >= 0, t >= 0, and resets
 * the hysteresis count to max(hysteresis, 1): it is the loss-scaler reset of
 * the OPT summary, "方法适配". */
neox_status neox_shard_get_state(const neox_shard* h, float* scale, int32_t* good, int64_t* t);
neox_status neox_shard_set_state(neox_shard* h, float scale, int32_t good, int64_t t);

/* The hysteresis count H of step 4 (overflows still tolerated before the next
 * back-off), for an exact checkpoint: set it after set_state on resume.
 * set_hysteresis validates count >= 0.  Waits for asynchronous steps as
 * get_state / set_state do. */
neox_status neox_shard_get_hysteresis(const neox_shard* h, int32_t* count);
neox_status neox_shard_set_hysteresis(neox_shard* h, int32_t count);

/* Free what create allocated (never the caller's arrays).  NULL is a no-op. */
void neox_shard_destroy(neox_shard* h);

/* Static strings. */
const char* neox_status_string(neox_status s);
/* The last error message of this handle ("" if none); NULL handle -> the last
 * error of a failed create on this thread. */
const char* neox_last_error(const neox_shard* h);

/* Model-state bytes of numel parameters: 16-bit working weight + 16-bit grad
 * + FP32 master, m and v = 16 bytes per parameter (host arithmetic only). */
uint64_t neox_model_state_bytes(uint64_t numel, neox_dtype wdtype, neox_dtype gdtype);

/* Device bytes the handle itself owns (scratch, scalars, segment table). */
uint64_t neox_shard_scratch_bytes(const neox_shard* h);

/* Per-kernel timing: when enabled, each step records CUDA events around its
 * two passes on the step's stream and accumulates their durations (read after
 * the step's own synchronisation, so no extra wait).  `launches` counts every
 * kernel this handle launched since create, timing on or off. */
typedef struct {
    int64_t steps;             /* steps timed since the last reset            */
    int64_t launches;          /* kernels launched by this handle             */
    double grad_pass_ms;       /* total of pass 1 (ingest, flag, norm, scaler) */
    double update_pass_ms;     /* total of pass 2 (AdamW + cast)              */
    double last_grad_pass_ms;
    double last_update_pass_ms;
} neox_profile;

neox_status neox_shard_set_profiling(neox_shard* h, int32_t enable);
neox_status neox_shard_get_profile(const neox_shard* h, neox_profile* out);
neox_status neox_shard_reset_profile(neox_shard* h);

/* ------------------------------------------------------------------------
 * Multi-tensor (non-flat) shard.
 *
 * The same step over a shard made of many separately allocated tensors (one
 * shard per parameter, as FSDP does when it shards parameter by parameter
 * instead of flattening them): mathematically the flat step over the
 * tensors' concatenation with one weight-decay segment per tensor, including
 * the single global norm, flag and scaler.  "OPT: Open Pre-trained
 * Transformer Language Models" (ai-papers.xuzou.cn summary), sections
 * "计算设置" / "方法适配": FSDP shards the model state across ranks.
 *
 * All pointers are bound at create: every tensor's FP32 master / exp_avg /
 * exp_avg_sq (4-byte aligned), its 16-bit working weights (params) and its
 * num_grads 16-bit gradient buffers (2-byte aligned), all device memory the
 * caller owns and keeps alive.  Each tensor chooses its own vector width and
 * head peel from its own pointers.  A tensor may have numel 0 (its pointers
 * are then ignored).  The steps are then launched with only the learning
 * rate.  The tensors that stream 8-element vectors (those whose arrays share
 * a 16-byte residue) form one sequence of vectors: pass 1 deals it to the
 * threads with a fixed assignment (so the norm is deterministic), the SGD
 * pass takes it in chunks from a counter; the AdamW pass takes the vectors
 * of all tensors as one sequence in chunks from a counter; tensors with
 * narrower vectors are covered grid-stride one after another.
 * ------------------------------------------------------------------------ */
typedef struct {
    uint64_t numel;
    float weight_decay;
    float* master;
    float* exp_avg;
    float* exp_avg_sq;
    void* params;                 /* 16-bit working weights                   */
    const void* const* grads;     /* host array of num_grads device pointers  */
} neox_tensor;

typedef struct {
    int32_t ntensors;             /* >= 0                                     */
    int32_t num_grads;            /* K in [1, 64], the same for every tensor  */
    neox_dtype wdtype, gdtype;
    const neox_tensor* tensors;   /* host array of ntensors                   */
} neox_tensor_set;

typedef struct neox_multi neox_multi;

/* Validate every tensor (NEOX_ERR_INVALID_ARGUMENT before any CUDA call),
 * choose each tensor's layout, and copy the tensor table, the sequence table
 * and the gradient pointer table to the device. */
neox_status neox_multi_create(const neox_tensor_set* set, const neox_hparams* hp, int device, neox_multi** out);
/* One step, as neox_shard_step (blocking on cuda_stream). */
neox_status neox_multi_step(neox_multi* h, float lr, void* cuda_stream, neox_step_result* out);
/* One step, as neox_shard_step_async (no host read-back, graph-capturable). */
neox_status neox_multi_step_async(neox_multi* h, float lr, const float* lr_device, void* cuda_stream,
                                  neox_step_result* result);
/* Point the tensors at other gradient buffers: `grads` is a host array of
 * ntensors * num_grads device pointers (tensor-major), each with the same
 * address residue as the buffer it replaces (the tensor's vector layout is
 * kept).  Waits for the device, then copies the tables (synchronous). */
neox_status neox_multi_rebind_grads(neox_multi* h, const void* const* grads);
neox_status neox_multi_set_hparams(neox_multi* h, const neox_hparams* hp);
neox_status neox_multi_get_state(const neox_multi* h, float* scale, int32_t* good, int64_t* t);
neox_status neox_multi_set_state(neox_multi* h, float scale, int32_t good, int64_t t);
neox_status neox_multi_get_hysteresis(const neox_multi* h, int32_t* count);
neox_status neox_multi_set_hysteresis(neox_multi* h, int32_t count);
/* Per-pass timing of synchronous steps, as neox_shard_set_profiling /
 * get_profile / reset_profile (the same neox_profile record). */
neox_status neox_multi_set_profiling(neox_multi* h, int32_t enable);
neox_status neox_multi_get_profile(const neox_multi* h, neox_profile* out);
neox_status neox_multi_reset_profile(neox_multi* h);
void neox_multi_destroy(neox_multi* h);
const char* neox_multi_last_error(const neox_multi* h);

/* ------------------------------------------------------------------------
 * Step without a handle and without any allocation.
 *
 * The pages have no counterpart to this entry point; it is a library service.
 * Some callers may not allocate device or pinned memory at all: code running
 * inside a device-memory allocator's own hook (a cudaMalloc there re-enters
 * the allocator), runtimes that give all device memory to their own pool up
 * front, and loops that must not let cudaMalloc / cudaFree synchronise the
 * device.  neox_shard_create allocates, so those callers use this function
 * instead.  It runs the same two kernels as neox_shard_step and calls no
 * cudaMalloc, cudaMallocHost, cudaFree or other allocating routine.  Its
 * scratch (per-block partial sums, the 64-byte scalar block, the segment
 * table) is one static device array of about 68 KiB, which every GPU that
 * loads this library holds until the process exits.
 *
 * Limits: at most 1024 segments (a longer table is rejected with
 * NEOX_ERR_INVALID_ARGUMENT and a message); K in [1, 64].  There is no FP32
 * gradient-sum buffer (it would need numel*4 bytes), so K >= 5 re-reads the K
 * buffers in pass 2; desc->max_grads and desc->flags are ignored.  numel itself
 * is not limited.
 * The scaler state below has no hysteresis count, so hp->hysteresis must be
 * 0 or 1 (a larger value is rejected); hp->optimizer is honoured.
 *
 * Arguments are those of neox_shard_create + neox_shard_step; desc->numel,
 * dtypes, segment table and the caller-owned master / exp_avg / exp_avg_sq
 * describe the shard.  *state carries the loss-scaler state in (the scale this
 * step's gradients carry, the counter, t) and receives it back after the step;
 * start with {init_scale, 0, 0}.  hp->init_scale is ignored.  Runs on the
 * calling thread's current CUDA device and on cuda_stream; returns after the
 * step has finished (it synchronises cuda_stream only).
 *
 * Set-up: the first call on each device (with that device current) does the
 * set-up: it checks the device, looks up the address of the static array on
 * that device (cudaGetSymbolAddress; host code cannot use the array's name as
 * a device address) and loads every kernel instance the call can launch --
 * CUDA loads kernels lazily, at their first launch, which takes device memory
 * -- so that no later call, whatever its dtypes, K or update rule, takes any.
 * Make that first call before any stream capture begins, and before the
 * memory it must not touch is handed out.  Every call looks the address up
 * again (that allocates nothing) and repeats the set-up when the device's
 * context is not the one it was done in (after cudaDeviceReset, say).
 *
 * Sharing: every call on a device uses the same static array, and the array
 * keeps the previous call's contents.  Each call reloads what must start
 * fresh (the scalar block with its ticket counter set to zero, and the segment
 * table) on its own stream, so calls one after another are independent.  Calls
 * that overlap on the GPU (concurrent streams, or threads calling at the same
 * time) race on the array and give wrong results: serialise them.
 *
 * Errors as neox_shard_step; the message of the last failed call on this
 * thread is neox_noalloc_last_error().
 * ------------------------------------------------------------------------ */
typedef struct {
    float scale;     /* loss scale the step's gradients carry (> 0)   */
    int32_t good;    /* consecutive applied steps (>= 0)               */
    int64_t t;       /* applied steps so far (>= 0)                    */
} neox_scaler_state;

neox_status neox_shard_step_noalloc(const neox_shard_desc* desc, const neox_hparams* hp,
                                    neox_scaler_state* state, const void* const* grads, int32_t num_grads,
                                    void* params, float lr, void* cuda_stream, neox_step_result* out);
const char* neox_noalloc_last_error(void);

#ifdef __cplusplus
}
#endif

#endif /* NEOX_SHARD_H */
