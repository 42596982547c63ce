/*
 * muonadamw.h - C ABI of the B200 (sm_100a) MuonAdamW optimizer-step library.
 *
 * The library updates optimizer state and parameters in place, on the GPU.
 * Every argument is a plain pointer or size. A pointer marked "device" must
 * point into memory that the calling context's current CUDA device can read
 * and write. "host" pointers are read by the CPU during the call and are not
 * kept afterwards. Streams are passed as `void*` holding a `cudaStream_t`
 * (NULL = the legacy default stream).
 *
 * Ownership: the caller owns every tensor, optimizer-state buffer, workspace
 * and stream. A plan (ma_plan_t) owns only host metadata.
 *
 * Errors: every entry point validates all of its arguments before it launches
 * anything, so a call that returns an error has changed nothing. Launches are
 * asynchronous on the given stream and the host never blocks. A kernel that
 * hits an internal time limit (a bounded wait that ran out) records
 * MA_ERR_TIMEOUT in a per-device status word, which ma_device_status() reads.
 * No entry point ever falls back to the CPU.
 *
 * Method sources (cited by page title and section):
 *  [P1] "How nanochat Combines Muon and AdamW in a Single Optimizer":
 *       "Parameter Grouping Strategy", "The MuonAdamW Class Architecture",
 *       "AdamW Step Implementation", "Muon Step Implementation".
 *  [P2] "Qwen Training Details: Full-Network Muon Optimizer and Residual
 *       Stream Design", "Confirmed".
 *  [P3] "nemo_automodel.components.optim.muown_triton", API of _prepare,
 *       _finish and _supported.
 *  [P4] "Guidelines for whether to use muon for parameters" (Muon issue 31).
 *  [P5] "MuonClip Optimizer": "Newton-Schulz Orthogonalization", "Momentum",
 *       "Design Decisions".
 */
#ifndef MUONADAMW_H
#define MUONADAMW_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define MA_VERSION 1

typedef enum {
    MA_OK = 0,
    MA_ERR_NULL = 1,        /* a required pointer is NULL                        */
    MA_ERR_SHAPE = 2,       /* a size or shape is negative or inconsistent        */
    MA_ERR_DTYPE = 3,       /* unknown dtype code                                 */
    MA_ERR_ALIGN = 4,       /* a pointer or row length breaks an alignment rule   */
    MA_ERR_WORKSPACE = 5,   /* workspace NULL, too small or misaligned            */
    MA_ERR_UNSUPPORTED = 6, /* a valid request this build does not implement      */
    MA_ERR_CUDA = 7,        /* a CUDA runtime call failed                         */
    MA_ERR_TIMEOUT = 8,     /* a device-side bounded wait ran out (status word)   */
    MA_ERR_ARG = 9,         /* a hyperparameter is out of its domain              */
    MA_ERR_BOUNDS = 10      /* debug builds: a guarded device index fell outside  */
                            /* its buffer and the access was skipped (status word) */
} ma_status_t;

typedef enum { MA_F32 = 0, MA_BF16 = 1 } ma_dtype_t;
typedef enum { MA_MUON = 0, MA_ADAMW = 1 } ma_kind_t;

/* Role of a tensor in the model. Muon is meant for hidden matrices whose input
 * and output are RMS-normed [P4]. Embedding and unembedding (head) matrices are
 * 2-D but belong with AdamW [P1 "AdamW Step Implementation"; P4]. Some
 * projections are forced onto AdamW for stability [P2]. */
typedef enum {
    MA_ROLE_HIDDEN = 0,
    MA_ROLE_EMBED = 1,
    MA_ROLE_UNEMBED = 2,
    MA_ROLE_FORCE_ADAMW = 3
} ma_role_t;

#define MA_MAX_NS_STEPS 16      /* Newton-Schulz iterations per step             */
#define MA_MAX_GROUPS 32        /* parameter groups per plan                     */
#define MA_MAX_BATCH 256        /* matrices per muon_step_batched call           */

/* Muon hyperparameters [P1 "Muon Step Implementation"; P5].
 *  lr, weight_decay: W <- W*(1 - lr*weight_decay) - lr*s*O (decoupled decay).
 *  beta: EMA momentum m <- beta*m + (1-beta)*g (0.95 default [P5 "Momentum"]).
 *  nesterov: direction u = beta*m + (1-beta)*g when nonzero, else u = m.
 *  eps: X0 = u / (||u||_F + eps).
 *  ns_steps: Newton-Schulz iterations, 1..MA_MAX_NS_STEPS (5 [P5]).
 *  coeffs: polynomial X <- aX + b(XX^T)X + c(XX^T)^2 X per iteration; with
 *      n_coeffs == 1 row 0 is used for every iteration, otherwise n_coeffs must
 *      equal ns_steps. The cubic of [P5] is (1.5, -0.5, 0).
 *  scale_mode: 0: s = sqrt(max(1, R/C)); 1: s = sqrt(R/C); 2: s = 1, with R x C
 *      the global shape of the matrix (or head slice) [P3 _finish].
 *  heads: rows split into `heads` equal slices, each orthogonalised on its own
 *      [P2 per-head orthogonalisation]; 1 = the whole matrix.
 *  precision: 0 = bf16 tensor-core operands with fp32 accumulation;
 *      1 = fp32 arithmetic throughout (a correctness mode).
 *  cautious: nonzero applies the weight decay only where the orthogonalised
 *      update O and the weight W have the same sign (O*W > 0), i.e. where the
 *      update already moves W towards zero. [P1 "Muon Step Implementation"]
 *      names "cautious weight decay" without defining it; this is a reading. */
typedef struct {
    float lr, beta, weight_decay, eps;
    int32_t nesterov, ns_steps, n_coeffs;
    float coeffs[MA_MAX_NS_STEPS][3];
    int32_t scale_mode, heads, precision;
    int32_t cautious;
} ma_muon_hparams_t;

/* AdamW hyperparameters [P1 "AdamW Step Implementation"; P3 _finish: bias
 * corrections are runtime scalars]. `step` is the 1-based index of the step
 * being taken; the bias corrections 1 - beta^step are formed in double on the
 * host. Update: m <- b1 m + (1-b1) g; v <- b2 v + (1-b2) g^2;
 * p <- p (1 - lr wd) - lr (m / (1-b1^t)) / (sqrt(v / (1-b2^t)) + eps). */
typedef struct {
    float lr, beta1, beta2, eps, weight_decay;
    int64_t step;
} ma_adamw_hparams_t;

/* A parameter group: `kind` dispatch as in [P1 "The MuonAdamW Class Architecture"]. */
typedef struct {
    int32_t kind;                /* ma_kind_t */
    ma_muon_hparams_t muon;      /* used when kind == MA_MUON  */
    ma_adamw_hparams_t adamw;    /* used when kind == MA_ADAMW */
} ma_group_t;

/* One tensor of the model. All buffers are device, fp32 row-major contiguous,
 * 16-byte aligned, except grad, which is fp32 or bf16 (grad_dtype).
 * state0/state1: Muon: momentum (state1 unused, may be NULL);
 *                AdamW: exp_avg, exp_avg_sq. State starts at zero. */
typedef struct {
    float* param;
    const void* grad;
    int32_t grad_dtype;          /* ma_dtype_t */
    float* state0;
    float* state1;
    int32_t ndim;                /* 0, 1 or 2 */
    int64_t shape[2];
    int32_t role;                /* ma_role_t */
    int32_t group;               /* index into the group table */
} ma_tensor_t;

typedef struct ma_plan ma_plan_t;

/* ---------------------------------------------------------------- host-only */

const char* ma_status_string(int status);
int ma_version(void);

/* sizeof of the ABI structs, for bindings to check their layouts:
 * 0 ma_tensor_t, 1 ma_group_t, 2 ma_muon_hparams_t, 3 ma_adamw_hparams_t,
 * 4 ma_shard_slot_t, 5 ma_shard_bucket_t; else 0. */
size_t ma_struct_size(int which);

/* Partition by tensor rank [P1 "Parameter Grouping Strategy"; P4]:
 * ndim <= 1 -> MA_ADAMW; ndim == 2 with role HIDDEN -> MA_MUON; ndim == 2 with
 * role EMBED / UNEMBED / FORCE_ADAMW -> MA_ADAMW; ndim >= 3 -> MA_ERR_UNSUPPORTED.
 * t: host array of n tensors (only ndim and role are read). kind_out: host
 * array of n ints. Host-only, no CUDA call, bit-exact and deterministic. */
int ma_partition(const ma_tensor_t* t, int n, int32_t* kind_out);

/* Owner rank per tensor for a data-parallel step over `world_size` ranks
 * [P1 "Distributed Training Support": each rank updates its share of the
 * parameters; P3: matrix batches are independent]: Muon matrices by greedy
 * largest-Newton-Schulz-flops-first onto the least-loaded rank, AdamW tensors
 * the same way by element count, ties to the lower rank and the lower tensor
 * index. Every tensor gets exactly one owner. t, groups: host arrays (shapes,
 * roles, groups and each Muon group's heads/ns_steps are read). owner_out:
 * host array of n ints. Errors as ma_partition, MA_ERR_ARG for world_size < 1
 * or a bad group index. Host-only, no CUDA call. */
int ma_assign_owners(const ma_tensor_t* t, int n, const ma_group_t* groups, int ngroups,
                     int world_size, int32_t* owner_out);

/* Flat-buffer layout of a sharded data-parallel step [P1 "Distributed
 * Training Support": each rank reduces the gradients it needs, updates its
 * share of the parameters and passes the result on; P3: matrix batches are
 * independent, and a matrix must be complete on the rank that orthogonalises
 * it].
 *
 * Every rank keeps the parameters (and, with the same element offsets, the
 * gradients) of the whole model in one flat buffer of `total` elements, cut
 * into buckets. Bucket b spans [start, start + world_size * seg) and rank r's
 * segment of it is [start + r * seg, start + (r + 1) * seg): the part that
 * rank r receives from a reduce-scatter of the bucket's gradients, updates,
 * and hands to an all-gather of the bucket's parameters.
 *  - Muon matrices are owned whole. Matrices of one shape and group (in
 *    order of appearance) fill buckets of world_size * k of them, k as many
 *    as fit seg_cap (at least one); matrix j of such a bucket belongs to rank
 *    j % world_size. The last (count % world_size) matrices of each class
 *    are left over and fill mixed buckets, in order of appearance, each
 *    closing before the matrix that would take its average per-rank share
 *    past seg_cap; a mixed bucket is packed largest matrix first onto the
 *    least-loaded rank (ties: lower rank, then lower index). A Muon segment
 *    is as long as its bucket's most loaded rank needs; within it, matrices
 *    sit in order of appearance.
 *  - An AdamW bucket holds AdamW tensors in order of appearance, laid end to
 *    end; AdamW is elementwise, so its segments split them by element range
 *    and a tensor may straddle segments (owner -1).
 * Buckets are ordered by their first tensor's index. Every tensor offset,
 * bucket start and segment length is a multiple of MA_SHARD_ALIGN elements,
 * so every piece a rank updates starts 16-byte aligned for fp32 and bf16.
 * Padding elements belong to no tensor. An AdamW bucket closes before the
 * tensor that would take its per-rank share past seg_cap. Every bucket holds
 * at least one tensor.
 *  t, groups: host arrays (shape, ndim, role and group are read).
 *  slots: host array of n entries (out). buckets: host array of at least n
 *  entries (out); nbuckets, total (out).
 * Errors: as ma_partition; MA_ERR_ARG for world_size < 1, seg_cap < 1, a bad
 * group index or a group whose kind differs from the tensor's; MA_ERR_SHAPE
 * for a negative extent or a layout beyond 2^50 elements. Host-only. */
#define MA_SHARD_ALIGN 64

typedef struct {
    int32_t bucket;   /* index of the bucket that holds the tensor        */
    int32_t owner;    /* owning rank of a Muon matrix; -1 for AdamW       */
    int64_t offset;   /* element offset of the tensor in the flat buffers */
} ma_shard_slot_t;

typedef struct {
    int32_t kind;     /* MA_MUON or MA_ADAMW                              */
    int32_t count;    /* tensors in the bucket                            */
    int64_t start;    /* element offset of the bucket                     */
    int64_t seg;      /* elements of one rank's segment                   */
} ma_shard_bucket_t;

int ma_shard_layout(const ma_tensor_t* t, int n, const ma_group_t* groups, int ngroups,
                    int world_size, int64_t seg_cap, ma_shard_slot_t* slots,
                    ma_shard_bucket_t* buckets, int* nbuckets, int64_t* total);

/* ---------------------------------------------------------------- Muon */

/* Workspace bytes that muon_step_batched needs for `batch` matrices of R x C
 * with these hyperparameters (0 for an empty batch; SIZE_MAX for invalid input). */
size_t muon_workspace_bytes(int batch, int64_t R, int64_t C, const ma_muon_hparams_t* hp);

/* One Muon step on `batch` same-shape R x C matrices [P1 "Muon Step
 * Implementation": stacked matrices, momentum, orthogonalisation, decay, write
 * back; P3 _prepare/_finish: fp32 weights and momentum mutated in place,
 * gradients preserved, scale from the global shape; P5: EMA momentum and the
 * Newton-Schulz cubic].
 *  W, M: host arrays of `batch` device pointers to fp32 R x C row-major
 *        (weights, momentum), updated in place.
 *  G:    host array of `batch` device pointers to R x C gradients (gdt), read only.
 *  hp:   host pointer. ws: device workspace of ws_bytes >= muon_workspace_bytes(),
 *        256-byte aligned, contents scratch.
 * Requires C % 8 == 0 and 16-byte aligned W/M/G; R % hp->heads == 0, and
 * W and M buffers that do not overlap (MA_ERR_ARG). A batch whose workspace
 * exceeds 4 GiB runs as consecutive sub-batches (halved until each fits),
 * reusing the start of ws; the results are the same. */
int muon_step_batched(int batch, int64_t R, int64_t C, float* const* W, const void* const* G,
                      int gdt, float* const* M, const ma_muon_hparams_t* hp, void* ws,
                      size_t ws_bytes, void* stream);

/* Newton-Schulz iterations alone, no normalisation [P5 "Newton-Schulz
 * Orthogonalization"]: for each of `batch` bf16 m x n row-major matrices with
 * m <= n, X <- aX + b(XX^T)X (+ c(XX^T)^2 X) for `steps` iterations.
 * X_in (device, read only) and X_out (device) hold batch*m*n bf16 values
 * (uint16 bit patterns), n % 8 == 0, 16-byte aligned. coeffs: host array of
 * n_coeffs triples (1 or steps). ws: device, >= ns_iterate_workspace_bytes(). */
size_t ns_iterate_workspace_bytes(int batch, int64_t m, int64_t n);
int ns_iterate_bf16(int batch, int64_t m, int64_t n, const uint16_t* X_in, uint16_t* X_out,
                    const float* coeffs, int n_coeffs, int steps, void* ws, size_t ws_bytes,
                    void* stream);

/* Muon step without a caller workspace. The paper has no counterpart; this
 * entry point exists for callers that cannot call cudaMalloc: plugins and hooks
 * inside a host framework that owns the device allocator and hands out no
 * scratch buffer, processes that reserve all their memory up front under a
 * fixed budget, and loops that cannot accept the device-wide synchronisation a
 * cudaMalloc may cause. Same arguments and results as muon_step_batched, minus
 * ws/ws_bytes. Its scratch is a file-scope device array of
 * MA_STATIC_SCRATCH_BYTES, which every GPU that loads the library holds until
 * the process exits.
 *  - Limit: returns MA_ERR_WORKSPACE, before launching anything, when
 *    muon_workspace_bytes(batch, R, C, hp) > MA_STATIC_SCRATCH_BYTES.
 *  - Set-up: the first call on each device looks up the array's device
 *    address (cudaGetSymbolAddress) with that device current; make that first
 *    call before any stream capture begins.
 *  - Sharing: every call on a device uses the same array and leaves its
 *    contents behind. Nothing in it needs to start at zero (each call writes
 *    every scratch value before reading it), but calls that overlap on the GPU
 *    (different streams, or different host threads) race on it.
 *  - Allocates nothing: no cudaMalloc, cudaFree or allocating library call. */
#define MA_STATIC_SCRATCH_BYTES ((size_t)64 << 20)
int muon_step_batched_noalloc(int batch, int64_t R, int64_t C, float* const* W, const void* const* G,
                              int gdt, float* const* M, const ma_muon_hparams_t* hp, void* stream);

/* ---------------------------------------------------------------- AdamW */

/* One AdamW step on n tensors in one multi-tensor launch sequence
 * [P1 "AdamW Step Implementation"]. P, M, V: host arrays of n device pointers
 * to fp32 (param, exp_avg, exp_avg_sq), updated in place. G: host array of n
 * device pointers to gradients of dtype gdt, read only. numel: host array of n
 * element counts (0 allowed). hp: host pointer. */
int adamw_step_fused(int n, float* const* P, const void* const* G, int gdt, float* const* M,
                     float* const* V, const int64_t* numel, const ma_adamw_hparams_t* hp,
                     void* stream);

/* ---------------------------------------------------------------- whole step */

/* Build a plan for a parameter table [P1 "The MuonAdamW Class Architecture"]:
 * partition, same-shape Muon buckets (first-appearance order), batching and
 * workspace sizing. t, groups: host arrays, copied. *ws_bytes: in = largest
 * workspace the caller will provide (0 = no limit), out = the bytes that
 * muonadamw_step needs (Muon buckets are split into sub-batches to fit).
 * Consecutive sub-batches whose Newton-Schulz chains take the same kernels
 * (tensor-core path, same iteration count, same iterations with c != 0) share
 * launches when their summed workspace fits: within the cap when one is given,
 * else within the larger of the biggest sub-batch and 4 GiB. Parameters and
 * optimizer state of different tensors (and a tensor's own state buffers)
 * must not overlap: MA_ERR_ARG otherwise. */
int ma_plan_create(const ma_tensor_t* t, int n, const ma_group_t* groups, int ngroups,
                   ma_plan_t** out, size_t* ws_bytes);

/* One MuonAdamW step over the planned table: one multi-tensor AdamW pass over
 * every AdamW tensor, then each Muon bucket. groups: host array with this
 * step's hyperparameters (same count and kinds as at plan time; lr schedules
 * and the AdamW step counter change here). ws: device, >= the planned size. */
int muonadamw_step(ma_plan_t* plan, const ma_group_t* groups, void* ws, size_t ws_bytes,
                   void* stream);

/* One MuonAdamW step whose gradients start in host memory (for example
 * gradients offloaded to the CPU). host_grads: host array of n pointers, one
 * per planned tensor in table order, each to that tensor's gradient in its
 * grad_dtype (numel elements; page-locked memory makes the copies
 * asynchronous). The library copies each gradient into the tensor's device
 * grad buffer on copy_stream, in the order the step consumes them (Muon
 * sub-batches first, the AdamW tensors last), records an event after each
 * group of copies, and makes `stream` wait for that event before the group's
 * kernels: later copies overlap earlier compute. The copies wait for all work
 * queued on `stream` before the call, since they overwrite the device
 * gradients. copy_stream may equal stream (no overlap). Results equal those of
 * muonadamw_step on the same gradients. Host buffers must stay valid and
 * unchanged until the step completes. */
int muonadamw_step_from_host(ma_plan_t* plan, const ma_group_t* groups, const void* const* host_grads, void* ws,
                             size_t ws_bytes, void* stream, void* copy_stream);

/* The same step as muonadamw_step, replayed from a CUDA graph (the launch
 * cost of a whole step is one graph launch; for small parameter sets the step
 * is launch-bound). The first call, and any call whose workspace, device or
 * Muon hyperparameters other than lr and weight_decay differ from those of the
 * captured step, captures the step on a stream the plan owns and instantiates
 * it (host cost of an eager step plus instantiation; nothing runs until the
 * launch). Every other call writes the new AdamW hyperparameters and step and
 * the new Muon lr and weight_decay into the captured kernels' parameters and
 * launches the graph on `stream`. Results are bit-identical to those of
 * muonadamw_step with the same arguments. In fp32 mode (precision 1) a change
 * of a Muon lr or weight_decay also re-captures. Must not be called while
 * `stream` or this thread is capturing. The plan keeps the graph until it is
 * destroyed. */
int muonadamw_step_graph(ma_plan_t* plan, const ma_group_t* groups, void* ws, size_t ws_bytes, void* stream);

/* How many times muonadamw_step_graph captured this plan's graph (tests,
 * benchmarks). 0 for a NULL plan. */
int ma_plan_graph_captures(const ma_plan_t* plan);

/* A text description of what muonadamw_step runs for this plan with these
 * hyperparameters: the workspace, the AdamW tensors, each Muon bucket (group,
 * shape, count, gradient dtype, heads, sub-batch size) and each segment of
 * launches (which sub-batches share Newton-Schulz launches). buf: host buffer
 * of len bytes, always NUL-terminated; MA_ERR_SHAPE when the text was cut to
 * fit. Host-only, no CUDA call. */
int ma_plan_describe(const ma_plan_t* plan, const ma_group_t* groups, char* buf, size_t len);

/* Number of kernel launches the last muonadamw_step, muonadamw_step_graph or
 * muonadamw_step_from_host issued (for a graph step: the kernels in the graph). */
int ma_plan_last_launches(const ma_plan_t* plan);

void ma_plan_destroy(ma_plan_t* plan);

/* ---------------------------------------------------------------- profiling */

/* Kernel classes for ma_profile_collect. */
#define MA_PROF_ADAMW 0         /* multi-tensor AdamW                          */
#define MA_PROF_MOMENTUM 1      /* momentum + Nesterov + norm partials         */
#define MA_PROF_FINALIZE 2      /* norm finalize                               */
#define MA_PROF_NS_GRAM 3       /* Newton-Schulz A = X X^T (tcgen05 or fp32)   */
#define MA_PROF_NS_APPLY 4      /* Newton-Schulz X' = aX + BX (not the last)   */
#define MA_PROF_NS_GRAMSQ 5     /* symmetric m x m products: A^2 (c != 0), and */
                                /* the Gram-space chain's Q, A P and P A P     */
#define MA_PROF_NS_FINAL 6      /* last apply, fused with decay and W update   */
#define MA_PROF_MOMENTUM_SIDE 7 /* momentum pass and norm finalize run under   */
                                /* the Newton-Schulz chain of the batch before */
                                /* it (side stream)                            */
#define MA_PROF_NS_Q1 8         /* Gram-space chain: Q_1 = a I + b A_0         */
#define MA_PROF_CLASSES 9

/* When on != 0, every kernel the library launches on this thread's current
 * device is bracketed by two CUDA events recorded on its launch stream. Off by
 * default; costs two event records per launch when on. */
int ma_profile_enable(int on);

/* Wait for the recorded events, then, per class (arrays of MA_PROF_CLASSES,
 * host, any may be NULL), store the summed device time in ms, the launch
 * count, and the algorithmic work of those launches: flops for the
 * Newton-Schulz classes (symmetric Gram counted as m(m+1)n, apply as 2m^2n,
 * per unit), DRAM bytes for the memory-bound classes (AdamW 26 B/element with
 * bf16 gradients and 28 with fp32; momentum pass 12 / 14 B/element, +2 when X
 * is fp32), and for the Newton-Schulz classes the bytes of reading each
 * operand and writing each result once (the final apply adds 8 B per weight).
 * Clears the record. */
int ma_profile_collect(double* ms_out, int64_t* launches_out, double* flops_out, double* bytes_out);

/* ---------------------------------------------------------------- status */

/* Synchronise `stream`, return the per-device status word (MA_OK or the first
 * device-side error recorded since the last reset) and, if reset != 0, clear it. */
int ma_device_status(void* stream, int reset);

/* The status of a plan's steps: synchronise `stream` (the stream the plan's
 * steps were launched on), then read and clear the status word of the current
 * device, as ma_device_status(stream, 1) does. Returns MA_ERR_NULL for a NULL
 * plan, MA_ERR_CUDA when the device cannot be reached, else MA_OK or the
 * first device-side error (MA_ERR_TIMEOUT) since the last read. */
int ma_plan_status(ma_plan_t* plan, void* stream);

/* Enqueue on `stream` a copy of the current device's status word into
 * host_dst (one int32, host; page-locked memory makes the copy asynchronous).
 * The value is valid once the stream has passed the copy; the word is not
 * reset. Lets a training loop read every step's status without stalling the
 * host. MA_ERR_NULL for a NULL destination. */
int ma_device_status_async(int32_t* host_dst, void* stream);

/* Set the limit, in nanoseconds, of every device-side bounded wait (default
 * 2e9). Takes effect for launches issued after the call. */
int ma_set_wait_limit_ns(int64_t limit_ns);

/* Momentum overlap for plans created after the call (on: 1, off: 0, the
 * default; MA_ERR_ARG otherwise). A plan created with it on, whose step has
 * two or more Muon sub-batches, takes a workspace of two halves used by the
 * sub-batches in turn, and runs each sub-batch's momentum pass and norm
 * finalize on a low-priority stream of its own while the Newton-Schulz chain
 * of the sub-batch before it runs (a cap then bounds the two halves
 * together). Results are bit-identical either way. It is off by default
 * because it is slower on a B200: the side kernels' blocks share SMs with the
 * persistent Newton-Schulz CTA pairs, each pair walks a fixed share of the
 * tiles, and every launch then ends with its slowest pair; on the 7B-shaped
 * set the step took 270 ms with it and 251.5 ms without on the same GPU. */
int ma_set_momentum_overlap(int on);

/* 1 in the debug build of the library (libmuonadamw_debug.so, compiled with
 * -DMA_DEBUG), else 0. The debug build checks every hand-computed device
 * index against the extent of its buffer before the access; a failed check
 * records MA_ERR_BOUNDS in the status word and skips the access. Its results
 * are otherwise bit-identical to the release build's. */
int ma_debug_build(void);

/* Self-test of the bounded wait: launch one block that waits on a barrier
 * phase that nothing completes, with a wait limit of limit_ns. The kernel
 * returns after the limit and records MA_ERR_TIMEOUT in the status word;
 * the context stays usable. Returns the launch status (MA_OK if launched). */
int ma_selftest_wait_timeout(int64_t limit_ns, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* MUONADAMW_H */
