/*
 * mpk.h — C ABI of a persistent-megakernel decoder for NVIDIA B200 (sm_100a).
 *
 * One decoding iteration of a decoder-only transformer is compiled into a task
 * graph of fused operations and executed by ONE persistent kernel launch that
 * stays resident for every iteration of a run: scheduler warps hand task
 * descriptors to worker SMs, workers gate each task on global-memory event
 * counters, and the last task of an iteration advances `step` and writes the
 * next token into `tokens` without returning to the host.
 *
 * Sources of the interface (web pages about Mirage Persistent Kernel, MPK):
 *  [EN]  "Mirage Persistent Kernel: Fusing Multi-GPU LLM Inference into One
 *        Kernel Launch" — sections "How MPK Works", "Getting Started", "The API".
 *  [ZH]  "Mirage Persistent Kernel：把 LLM 推理压进单个 GPU 内核" — sections
 *        "工作机制：持久内核与任务图", "关键 API 与张量管理", "真正的限制".
 *  [DE]  "Mirage Persistent Kernel kompiliert LLM-Inferenz in einen Persistent
 *        Kernel" — sections "Betrieb und Konfiguration", "Grenzen der
 *        README-Aussagen".
 *
 * Conventions for every call:
 *  - Return value: MPK_OK (0) or a negative mpk_error.  On error the context is
 *    unchanged and mpk_last_error(ctx) describes the failure.
 *  - Pointers documented "device" are CUDA device addresses of the current
 *    device; "host" pointers are plain host memory.
 *  - Tensors are dense, contiguous, row-major; dims are int64 extents, outermost
 *    first.  Every tensor must start on a 16-byte boundary.
 *  - Not thread-safe: one host thread drives a context at a time.
 */
#ifndef MPK_H
#define MPK_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define MPK_ABI_VERSION 4

#if defined(__GNUC__)
#define MPK_API __attribute__((visibility("default")))
#else
#define MPK_API
#endif

typedef struct mpk_ctx mpk_ctx;

typedef enum {
    MPK_OK = 0,
    MPK_ERR_INVALID_ARG = -1, /* NULL pointer, bad count, bad enum value        */
    MPK_ERR_SM_FORMULA = -2,  /* worker/scheduler split does not fit the GPU     */
    MPK_ERR_UNSUPPORTED = -3, /* valid request this build does not implement     */
    MPK_ERR_NOT_FOUND = -4,   /* unknown tensor name                             */
    MPK_ERR_SHAPE = -5,       /* tensor extents do not fit the operation         */
    MPK_ERR_DTYPE = -6,       /* tensor element type does not fit the operation  */
    MPK_ERR_STATE = -7,       /* call out of order (e.g. run before compile)     */
    MPK_ERR_CUDA = -8,        /* a CUDA runtime call failed                      */
    MPK_ERR_TIMEOUT = -9,     /* a device-side wait exceeded its time limit      */
    MPK_ERR_ABORTED = -10,    /* the run was aborted on request                  */
    MPK_ERR_DEVICE = -11      /* device-side consistency check failed            */
} mpk_error;

/* MPK_FP32T, the activations passed between operations: 8 bytes per element,
 * the fp32 value in the low 32 bits and a version tag in the high 32 bits.  A
 * writer stores value and tag in one 8-byte store; a reader waits until the
 * element carries the tag of the write it needs, so no flag or fence is needed
 * between producing and consuming operations.  Tag of a write by operation p
 * in iteration n of a run (n counted from 0): n * num_operations + p + 1; the
 * library zeroes every MPK_FP32T tensor at the start of each run. */
typedef enum { MPK_BF16 = 0, MPK_FP32 = 1, MPK_INT32 = 2, MPK_INT64 = 3, MPK_FP32T = 4 } mpk_dtype;

/* Memory category of a library-allocated tensor ([EN] "The API"; [ZH]
 * "关键 API 与张量管理"): CUDA memory of this GPU, or NVSHMEM symmetric memory
 * for remote GPU access.  Only MPK_IO_CUDA is implemented (one GPU). */
typedef enum { MPK_IO_CUDA = 0, MPK_IO_NVSHMEM = 1 } mpk_io;

/* Fused operations of the task graph ([EN] "The API": operations are chained
 * to build the graph; rmsnorm_linear_layer is the one the pages name).
 * Number format: weights and the KV cache are bf16; every activation (the
 * residual stream x, normed inputs h, q/k/v, the attention output o, the MLP
 * product a, logits) is fp32; dot products accumulate in fp32.  The
 * activation tensors passed between operations (x, q, k, v, o, a below,
 * written "fp32") are registered as MPK_FP32T: fp32 values carrying version
 * tags; MPK_ERR_DTYPE otherwise. */
typedef enum {
    /* x[r,:] = fp32(E[tokens[r, step[r]], :]).
     * weights[0] = E bf16 [V,H]; outputs[0] = x fp32 [R,H].  grid_dim = R tasks. */
    MPK_OP_EMBED = 1,
    /* RMSNorm feeding one or more linear layers stacked by rows:
     * h = x / sqrt(mean(x^2) + eps) * w_norm; y_i = W_i h.
     * inputs[0] = x fp32 [R,K]; weights[0] = w_norm bf16 [K];
     * weights[1..3] = W_i bf16 [N_i,K]; outputs[0..2] = y_i fp32 [R,N_i]
     * (output i belongs to weight i+1).  grid_dim = row-block tasks. */
    MPK_OP_RMSNORM_LINEAR = 2,
    /* Per request r at position s = step[r], per kv head j: RMSNorm over the
     * head dim and rotate-half RoPE of q (its query-head group) and k, append
     * bf16 k and v at position s of the cache, causal grouped-query attention
     * over positions 0..s (split into grid_dim.y chunks, merged by
     * log-sum-exp), o = attention output.
     * inputs = q fp32 [R,Hq*d], k fp32 [R,Hkv*d], v fp32 [R,Hkv*d];
     * weights = q_norm bf16 [d], k_norm bf16 [d], k_cache, v_cache bf16
     * [L,R,Hkv,S,d]; outputs[0] = o fp32 [R,Hq*d].  layer selects the cache
     * slice; rope_theta the RoPE base.  grid_dim = (Hkv, C, R), C <= 256:
     * task (j, c, r) attends to chunk c of C of request r's positions (a
     * split that never depends on the other requests); a request that is not
     * active publishes zeros as its output.  With a prefill graph the cache
     * holds the graph's requests (Rq of them, dims[1]), R is the column count. */
    MPK_OP_ATTENTION = 3,
    /* x += W a.  inputs[0] = a fp32 [R,K]; weights[0] = W bf16 [N,K];
     * outputs[0] = x fp32 [R,N] (read and written in place).  When K exceeds
     * MPK_MAX_GEMV_K the reduction is split into the fewest ks equal segments
     * of at most MPK_MAX_GEMV_K (each a multiple of 256): task t computes
     * segment t % ks of row block t / ks, and the last segment task of a row
     * block to finish adds the ks partial sums to x in segment order.  grid_dim
     * must then give a multiple of ks tasks (MPK_ERR_SHAPE otherwise). */
    MPK_OP_LINEAR_RESIDUAL = 4,
    /* h = rmsnorm(x) * w_norm; a = silu(W_gate h) * (W_up h).
     * inputs[0] = x fp32 [R,K]; weights = w_norm [K], W_gate [I,K], W_up [I,K];
     * outputs[0] = a fp32 [R,I]. */
    MPK_OP_RMSNORM_LINEAR_SILU_MUL = 5,
    /* z = W_lm (rmsnorm(x) * w_norm) in fp32; greedy argmax (lowest index on
     * ties); then, per active request: tokens[r, s+1] = argmax if that slot
     * holds -1, pred[r, s+1] = argmax, step[r] = s + 1 ([EN] "How MPK Works":
     * the runtime advances `step` after every iteration).  inputs[0] = x;
     * weights = w_norm [K], W_lm [V,K]; outputs[0] (optional, may be NULL) =
     * pred int64 [R,S].  Must be the last operation of the graph. */
    MPK_OP_RMSNORM_LMHEAD_ARGMAX = 6,
    /* RMSNORM_LINEAR for the stacked q/k/v projections fused with ATTENTION:
     * the projection rows are split per kv head j (its G query heads, its key
     * and its value: G*d + 2d rows) into grid_dim.x tasks per head, and the
     * last of those tasks to finish computes head j's attention directly (one
     * pass over positions 0..s, no split-K).  inputs[0] = x fp32 [R,K];
     * weights = w_norm [K], Wq [Hq*d,K], Wk [Hkv*d,K], Wv [Hkv*d,K], q_norm [d],
     * k_norm [d], k_cache, v_cache [L,R,Hkv,S,d]; outputs = q [R,Hq*d],
     * k, v [R,Hkv*d] (fp32 scratch), o fp32 [R,Hq*d].
     * grid_dim = (tasks per kv head, Hkv, R).  Meant for short contexts; long
     * ones use RMSNORM_LINEAR followed by ATTENTION with split-K. */
    MPK_OP_RMSNORM_QKV_ATTENTION = 7
} mpk_op;

typedef struct { int32_t x, y, z; } mpk_dim3;

#define MPK_MAX_IO 8
/* Longest reduction (input length K) one GEMV task holds in shared memory. */
#define MPK_MAX_GEMV_K 4096

/* One fused operation.  Unused name slots are NULL.  grid_dim gives the number
 * of tasks (thread blocks) x*y*z; block_dim the threads per task (a multiple
 * of 32, at most mpk_worker_threads()).  [EN] "The API": both are specified per
 * fused layer, and the total number of thread blocks should be a multiple of
 * the number of workers (a warning, not an error, when it is not).
 *
 * Several requests (R = 2..MPK_MAX_BATCH): the projection operations
 * (RMSNORM_LINEAR, LINEAR_RESIDUAL, RMSNORM_LINEAR_SILU_MUL,
 * RMSNORM_LMHEAD_ARGMAX) run on the tensor cores as [R,K] x W^T contractions
 * (tcgen05: weight tiles of MPK_BATCH_BM rows x 64 by TMA, every fp32 input
 * split into bf16 hi + lo parts so the products see it to ~16 bits, fp32
 * accumulation in tensor memory).  Their grid_dim is then (gx, gy, 1): the N
 * rows form nb = ceil(N / MPK_BATCH_BM) row blocks (gate/up: of one matrix)
 * and the reduction gy segments (gy <= K / 64); task t computes segment
 * t / gx for the row blocks [u*nb/gx, (u+1)*nb/gx), u = t % gx (gx <= nb).
 * With gy > 1 the last segment task of a row block to finish adds the partial
 * sums in segment order.  A task whose segment is longer than
 * MPK_BATCH_MAX_PASS_K runs it in passes and then holds at most
 * MPK_BATCH_SLOTS row blocks.  Graphs of 9..MPK_MAX_BATCH requests run
 * every contraction 16 requests wide (the weights are still read once per
 * iteration); their limits are MPK_BATCH_WIDE_MAX_PASS_K and
 * MPK_BATCH_WIDE_SLOTS; more requests fail mpk_compile with
 * MPK_ERR_UNSUPPORTED.  K must be a multiple of 64 and stacked matrices
 * start at multiples of MPK_BATCH_BM rows (MPK_ERR_UNSUPPORTED otherwise);
 * RMSNORM_QKV_ATTENTION takes one request.  A prefill graph
 * (mpk_options.prefill_tokens) takes at most MPK_MAX_PREFILL positions per
 * iteration. */
#define MPK_MAX_BATCH 16
#define MPK_MAX_PREFILL 8
#define MPK_BATCH_BM 128
#define MPK_BATCH_MAX_PASS_K 1536
#define MPK_BATCH_SLOTS 16
#define MPK_BATCH_WIDE_MAX_PASS_K 768
#define MPK_BATCH_WIDE_SLOTS 8
typedef struct {
    int32_t op;                         /* mpk_op */
    const char *inputs[MPK_MAX_IO];
    const char *weights[MPK_MAX_IO];
    const char *outputs[MPK_MAX_IO];
    mpk_dim3 grid_dim;
    mpk_dim3 block_dim;
    int32_t layer;                      /* ATTENTION: layer index into the cache */
    int32_t capture_slot;               /* hidden-state capture slot, -1 = none  */
    float eps;                          /* RMSNorm epsilon                       */
    float rope_theta;                   /* ATTENTION: RoPE base                  */
} mpk_layer;

typedef struct {
    int32_t profiling;      /* 1: record a per-task timeline ([EN] "Getting Started": --profiling) */
    int32_t sched_lookahead;/* scheduler dispatch window in operations (<=0: default 4)   */
    double timeout_s;       /* limit of every device-side wait (<=0: default 2 s)        */
    int32_t max_timeline;   /* timeline entries kept when profiling (<=0: 1<<20)         */
    int32_t prefetch_kb;    /* L2 prefetch distance per worker ahead of the shared-memory
                               weight ring, KiB (<=0: off)                                 */
    int32_t dynamic_tasks;  /* > 0: the one-request GEMV operations (all but the fused
                               projections + attention) hand their tasks out through a
                               shared counter: each worker claims the next task when its
                               weight ring has room, so the work follows the workers that
                               are ahead; <= 0 (default): fixed mapping, task t on worker
                               (t + offset) % W.  The tensor-core projections over several
                               requests are always claimed this way.  Results are
                               identical either way.                                     */
    int32_t debug_stall_op; /* fault injection for tests: k > 0 makes operation k-1 wait
                               for an input nothing will produce (a version of the next
                               iteration, or one completion more than its dependency
                               delivers), so that wait runs out and the run ends with
                               MPK_ERR_TIMEOUT (0: off)                                    */
    int32_t poll_inputs;    /* several requests: > 0 makes every tensor-core projection
                               read its input element by element (poll each tagged word,
                               apply the RMSNorm, split into bf16 hi/lo) instead of the
                               rows its writer publishes in the shared-memory layout;
                               <= 0 (default): published rows wherever the graph allows.
                               The RMSNorm factor then scales the input instead of the
                               products, so results agree to rounding, not bit for bit. */
    int32_t prefill_tokens; /* T in 2..MPK_MAX_PREFILL: a prefill graph.  Its activations
                               have T rows, the columns of the tensor-core projections;
                               its KV cache [L, Rq, Hkv, S, d] holds Rq requests (tokens
                               [Rq, S], step [Rq], pred [Rq, S]), served one after
                               another in request order.  Every iteration advances ONE
                               request q by T positions: column c consumes tokens[q,
                               step[q] + c], appends its K/V there and attends to
                               positions 0 .. step[q] + c (the chunk's earlier positions
                               from this iteration's k and v, the rest from the cache),
                               so a prompt is ingested T tokens per iteration instead of
                               one.  Column c's argmax goes to pred[q, step[q] + c + 1]
                               and to tokens[q, step[q] + c + 1] when that slot holds -1;
                               step[q] advances past the last active column.  A
                               request's last chunk may be partial (step_end); a request
                               with step -1 is skipped.  <= 1 (default): one position
                               per request per iteration.                                 */
    int32_t kv_page_size;   /* > 0: paged KV caches for the ATTENTION operations.  The
                               caches are [L, P, Hkv, kv_page_size, d] (P pages shared by
                               all requests) and an MPK_INT32 tensor named "kv_pages",
                               [R, max_pages], maps page i of request r (positions
                               i * kv_page_size ..) to its page of the caches; the
                               longest sequence is max_pages * kv_page_size positions.
                               kv_page_size must be a multiple of 128.  A page index
                               outside 0..P-1 ends the run with MPK_ERR_DEVICE (nothing
                               is read or written there).  The fused projections +
                               attention operation needs a contiguous cache
                               (UNSUPPORTED otherwise).  <= 0 (default): contiguous
                               caches [L, R, Hkv, S, d].                                  */
} mpk_options;

/* Library build facts. */
MPK_API int mpk_abi_version(void);
/* Threads per worker block available to a task. */
MPK_API int mpk_worker_threads(void);
/* Number of SMs of the current device, or a negative mpk_error. */
MPK_API int mpk_device_sm_count(void);

/*
 * Check a worker/scheduler split against an SM count without touching a GPU
 * ([EN] "How MPK Works", [ZH] "真正的限制", [DE] "Betrieb und Konfiguration"):
 * num_workers + (num_local + num_remote) / 4 == sm_count, with num_local +
 * num_remote a multiple of 4.  Returns MPK_OK, MPK_ERR_INVALID_ARG (negative
 * counts, no local scheduler), MPK_ERR_SM_FORMULA or MPK_ERR_UNSUPPORTED
 * (num_remote > 0: remote schedulers serve other GPUs).
 */
MPK_API int mpk_validate_split(int sm_count, int num_workers, int num_local_schedulers, int num_remote_schedulers);

/*
 * Create a context on the current device.  [EN] "How MPK Works", [ZH]
 * "真正的限制", [DE] "Betrieb und Konfiguration": num_workers +
 * (num_local_schedulers + num_remote_schedulers) / 4 must equal the number of
 * SMs, so the scheduler count must be a multiple of 4.  Remote schedulers serve
 * other GPUs; this build is single-GPU, so num_remote_schedulers must be 0.
 * Errors: INVALID_ARG (out NULL, negative counts, num_local_schedulers == 0),
 * SM_FORMULA (sum or multiple-of-4 rule broken), UNSUPPORTED (remote > 0,
 * device not sm_100, no cooperative launch), CUDA.  *out receives the context.
 */
MPK_API int mpk_create(int num_workers, int num_local_schedulers, int num_remote_schedulers,
               mpk_ctx **out);

/* Register a caller-owned device tensor under `name` ([EN] "The API":
 * attach_input).  The memory is borrowed: it must stay valid until
 * mpk_destroy.  Errors: INVALID_ARG (NULL, ndim outside 1..5, extent < 1,
 * duplicate name, misaligned pointer), STATE (after compile). */
MPK_API int mpk_attach_input(mpk_ctx *ctx, const char *name, void *dev_ptr, mpk_dtype dtype, int ndim,
                     const int64_t *dims);

/* Allocate a library-owned, zero-filled device tensor ([EN] "The API":
 * new_tensor with io_category).  *dev_ptr_out (may be NULL) receives its
 * address; it is freed by mpk_destroy.  Errors: INVALID_ARG, UNSUPPORTED
 * (MPK_IO_NVSHMEM), STATE, CUDA. */
MPK_API int mpk_new_tensor(mpk_ctx *ctx, const char *name, mpk_dtype dtype, int ndim, const int64_t *dims,
                   mpk_io io, void **dev_ptr_out);

/* Device address of a registered tensor, or NULL (unknown name). */
MPK_API void *mpk_tensor_ptr(mpk_ctx *ctx, const char *name);

/*
 * Compile the operations, in order, into the task graph ([EN] "Getting
 * Started": compile() is an explicit step).  Each operation depends on the one
 * before it; the first depends on the last operation of the previous
 * iteration.  Checks every name, dtype and shape, splits every operation into
 * grid_dim tasks, assigns event counters and allocates the run-time workspace.
 * opts may be NULL (defaults).  Errors: INVALID_ARG, NOT_FOUND, SHAPE, DTYPE,
 * UNSUPPORTED, STATE (compiled twice), CUDA.  mpk_warnings() lists the
 * non-fatal findings (task counts not a multiple of num_workers).
 */
MPK_API int mpk_compile(mpk_ctx *ctx, const mpk_layer *layers, int n_layers, const mpk_options *opts);

/* Newline-separated warnings from mpk_compile ("" when none). */
MPK_API const char *mpk_warnings(mpk_ctx *ctx);

/*
 * Run decoding iterations in ONE persistent kernel launch on `stream` (a
 * cudaStream_t; NULL = legacy default stream), asynchronously.  step: device
 * int32 [R]; tokens: device int64 [R,S] (R = num_requests, S = seq_length)
 * with -1 in slots to generate; step_end: device int32 [R] or NULL.  R must
 * equal the graph's request count (a prefill graph: its cache's) and S-1 must not
 * exceed the KV cache length; an attached pred tensor must be [R,S].  A
 * prefill graph (mpk_options.prefill_tokens = T) advances one request at a
 * time by T positions per iteration, each position with the semantics below.  Request r takes
 * part in iterations while step[r] < min(step_end[r], S-1) (NULL: S-1); each
 * iteration consumes tokens[r, step[r]], appends K/V at that position and
 * advances step[r] by one ([EN] "How MPK Works": step and tokens are the meta
 * tensors; the runtime increments step).  The kernel returns when no request
 * is active.  A later call continues from the current step (resume).
 * Errors: INVALID_ARG, STATE (not compiled), CUDA (launch failed).  Device
 * failures surface through mpk_status after the stream is synchronised.
 */
MPK_API int mpk_run(mpk_ctx *ctx, int32_t *step, int64_t *tokens, int num_requests, int64_t seq_length,
            const int32_t *step_end, void *stream);

/* Same iterations, one ordinary kernel launch per operation (no scheduler, no
 * event waits; the stream orders the operations).  Reads step/step_end to the
 * host first (synchronises `stream`).  Used to compare against the persistent
 * kernel and to measure launch overhead. */
MPK_API int mpk_run_op_by_op(mpk_ctx *ctx, int32_t *step, int64_t *tokens, int num_requests,
                     int64_t seq_length, const int32_t *step_end, void *stream);

/* Capture, during iteration `iter` of the next runs (counted from 0 within a
 * run; -1 = off), the fp32 logits into logits [R,V] and the residual stream
 * into hidden [slots,R,H] (slot = an operation's capture_slot).  Device
 * pointers, either may be NULL. */
MPK_API int mpk_set_capture(mpk_ctx *ctx, int iter, float *logits, float *hidden);

/* Device status of the last run (synchronises nothing: call after the stream
 * is synchronised).  MPK_OK, MPK_ERR_TIMEOUT, MPK_ERR_ABORTED or
 * MPK_ERR_DEVICE; details in mpk_last_error. */
MPK_API int mpk_status(mpk_ctx *ctx);

/* Ask a running kernel to stop (host-mapped flag, safe while the kernel runs).
 * The scheduler warps read it at every iteration boundary and long waits read
 * it now and then; the run then reports MPK_ERR_ABORTED.  `step`, `tokens` and
 * the KV cache stay consistent: a later mpk_run resumes from `step` and
 * produces what an uninterrupted run would have. */
MPK_API int mpk_request_abort(mpk_ctx *ctx);

/* Number of timeline records of the last profiled run, and a copy of up to
 * `cap` of them into host memory `out` (MPK_TIMELINE_FIELDS x uint64 each,
 * %globaltimer ns): packed task id (iter<<32 | op<<16 | task), worker, task
 * popped, dependency met, task done, prologue done (0 if none), first weight
 * stage ready (0 if none), first weight stage issued by the producer (0 if
 * none), total time the task waited for weight stages (a duration), last
 * weight stage ready (0 if none), every consumer warp done with its weight
 * rows (0 if none). */
#define MPK_TIMELINE_FIELDS 11
MPK_API int mpk_timeline(mpk_ctx *ctx, uint64_t *out, int cap);

/*
 * Final RMSNorm + LM head + greedy argmax that allocates nothing.  The MPK
 * pages have no counterpart to this call; it exists for callers that cannot
 * allocate device memory (for example a serving framework whose memory pool
 * owns all device memory and forbids cudaMalloc / cudaFree, which would also
 * synchronise the device, on its decode path).
 *
 * For each request r < num_requests: h = x[r] / sqrt(mean(x[r]^2) + eps)
 * * norm_w (fp32), z = w_lm h in fp32, tokens_out[r] = argmax z (lowest index on
 * ties), and logits_out[r, :] = z when logits_out is not NULL.
 *   x          device fp32 [num_requests, K]
 *   norm_w     device bf16 [K]
 *   w_lm       device bf16 [V, K] (16-byte aligned)
 *   tokens_out device int64 [num_requests]
 *   logits_out device fp32 [num_requests, V] or NULL
 *   stream     cudaStream_t (NULL: legacy default stream); asynchronous.
 * Limits: 1 <= num_requests <= MPK_NOALLOC_MAX_REQUESTS, K a multiple of 8 up
 * to MPK_NOALLOC_MAX_K; larger sizes return MPK_ERR_INVALID_ARG / MPK_ERR_SHAPE,
 * and eps must be positive and finite (else MPK_ERR_INVALID_ARG).  The message
 * of a failed call is in mpk_noalloc_last_error() of the calling thread.
 * Scratch: a fixed __device__ array of 2 * MPK_NOALLOC_MAX_REQUESTS 64-bit
 * words (1 KiB) inside this library; every GPU that loads the library holds it
 * until the process exits.  Each call clears it on `stream` before use.  All
 * calls share it, so calls that overlap on the GPU (on different streams, or
 * from different threads) race and must be serialised by the caller.  The
 * first call on a device looks up the array's device address (set-up done once
 * per device and context, with that device current; a device whose context was
 * reset gets a fresh lookup on its next call); make that first call before any
 * stream capture.  No cudaMalloc, cudaFree or allocating library routine is
 * called.
 */
#define MPK_NOALLOC_MAX_REQUESTS 64
#define MPK_NOALLOC_MAX_K 16384
MPK_API int mpk_lmhead_argmax_noalloc(const float *x, const uint16_t *norm_w, const uint16_t *w_lm,
                                      int num_requests, int K, int V, float eps, int64_t *tokens_out,
                                      float *logits_out, void *stream);

/* Message of this thread's last failed mpk_lmhead_argmax_noalloc call ("" if none). */
MPK_API const char *mpk_noalloc_last_error(void);

/* Free the context and every library-owned allocation. */
MPK_API int mpk_destroy(mpk_ctx *ctx);

/* Last error message of ctx (or of the last failed mpk_create when ctx is NULL). */
MPK_API const char *mpk_last_error(mpk_ctx *ctx);

#ifdef __cplusplus
}
#endif

#endif /* MPK_H */
