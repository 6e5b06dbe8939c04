/*
 * dmuon.h -- C ABI of the B200 (sm_100a) batched Muon update.
 *
 * The method: for every 2-D weight matrix W with gradient g and fp32
 * momentum buffer buf,
 *   buf  <- momentum * buf + g                    (two fp32 roundings, no FMA)
 *   M    <- g + momentum * buf   (Nesterov)   or   M <- buf
 *   X0   <- M / (||M||_F + 1e-7), taken as its transpose when rows > cols
 *   X    <- 1.5 X - 0.5 (X X^T) X                 (k times)
 *   W    <- W (1 - lr * weight_decay) - lr * X    (X transposed back)
 *
 * Sources (page title, section):
 *   DMuon blog post "DMuon：让矩阵正交化优化器达到接近 AdamW 的分布式训练开销"
 *     - "Muon 核心：Newton-Schulz 迭代": normalisation, the cubic step, and the
 *       newton_schulz() listing (transpose when rows > cols, +1e-7 on the norm);
 *     - "代码实现 / Vanilla Muon": momentum mul_/add_, the update p -= lr * X,
 *       and skipping parameters without a gradient.
 *   DMuon training guide "训练指南"
 *     - "第 4 步：创建优化器" (lr, momentum, ns_steps, nesterov, weight_decay);
 *     - "超参数指南" (Nesterov input grad + mu * buf).
 * Weight decay is read as decoupled, on the pre-update weight (the guide
 * names the parameter without a formula).
 *
 * Conventions shared by every entry point
 *   - Matrices are dense and row-major: element (r, c) at base[r * cols + c].
 *   - Every pointer argument is a DEVICE pointer owned by the caller, except
 *     the arrays of pointers / shapes themselves, which are HOST arrays read
 *     during the call only, and the page-locked host buffers named host_* of
 *     dmuon_muon_step_batched_host.  Updated tensors are written in place.
 *   - Calls are asynchronous: they only enqueue work on `stream` (a
 *     cudaStream_t; NULL is the legacy default stream) and never wait for the
 *     device.  Device pointers must stay valid until the stream reaches that
 *     work.  Tensor addresses are checked to be device memory (host memory,
 *     page-locked or not, is refused with DMUON_ERR_INVALID_ARG).
 *   - Errors are returned before anything is enqueued; the message is in
 *     dmuon_last_error() (per host thread).  NaN/Inf in the data propagate and
 *     are not reported.
 *   - Launch plans (descriptors, TMA tensor maps, tile tables) depend on the
 *     shapes, types, options and scratch address of a call, not on the tensor
 *     addresses: a call with new shapes builds one on the host and uploads it
 *     with small kernels on `stream`; later calls with the same shapes reuse
 *     it, and new tensor addresses are written into it (descriptors and the
 *     tensor maps through which the bf16 prologue reads gradients and momentum
 *     buffers) by one small kernel per group, in stream order.  Library memory (plans, the per-stream
 *     scratch arena) comes from a library memory pool in stream order
 *     (cudaMallocFromPoolAsync / cudaFreeAsync); a plan evicted from the cache
 *     (more than 64) is freed after the latest work that used it.  The first
 *     call on a device also sets the device up (kernel attributes, the pool).
 *   - CUDA graphs: the Muon-step entry points can be captured once their
 *     shapes have a plan (an eager call first).  While the stream captures,
 *     every tensor address is written into the plan by a captured patch
 *     kernel, so each replay updates the tensors it was captured with,
 *     whatever eager calls ran in between.  A call that would need a new plan
 *     or a larger scratch arena during capture is refused with
 *     DMUON_ERR_UNSUPPORTED before anything is enqueued.
 */
#ifndef DMUON_H_
#define DMUON_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* dmuon_stream_t; /* same type as cudaStream_t */

/* Element types. */
enum { DMUON_F32 = 0, DMUON_BF16 = 1 };

/* Return codes (0 = success, negative = error, nothing was enqueued). */
enum {
  DMUON_OK = 0,
  DMUON_ERR_INVALID_ARG = -1,  /* NULL pointer, size < 1, steps < 0, count < 0, misaligned element pointer */
  DMUON_ERR_UNSUPPORTED = -2,  /* dtype, or a size beyond the limits below */
  DMUON_ERR_NO_WORKSPACE = -3, /* workspace too small, or allocation failed */
  DMUON_ERR_CUDA = -4,         /* a CUDA runtime call failed (see dmuon_last_error) */
  DMUON_ERR_TIMEOUT = -5       /* a bounded device-side wait gave up (see dmuon_device_status) */
};

/* Size limits: min(rows, cols) <= DMUON_MAX_M, max(rows, cols) <= DMUON_MAX_N. */
#define DMUON_MAX_M 32768
#define DMUON_MAX_N (1 << 24)
#define DMUON_MAX_STEPS 1000

/* Shape and storage types of one matrix.  The momentum buffer is always fp32.
 * param_dtype selects the arithmetic: bf16 parameters run the iteration with
 * bf16 operands (fp32 accumulation); fp32 parameters use tf32 operands with
 * fp32 storage. */
typedef struct {
  int64_t rows, cols;
  int32_t param_dtype, grad_dtype;
} dmuon_shape;

/*
 * dmuon_ns_orthogonalize -- Newton-Schulz orthogonalisation of one bf16
 * matrix, in place: X <- NS_steps(X) with the normalisation and implicit
 * transpose of the blog's newton_schulz() listing ("Muon 核心" section).
 *   X       device pointer, rows x cols (m x n here) bf16, row-major; read and
 *           overwritten with the result (same layout, bf16, round-to-nearest).
 *   m, n    rows and cols, >= 1.
 *   steps   number of cubic steps, >= 0 (0 returns the normalised input).
 * Scratch memory comes from a library-owned per-stream arena (grown on
 * demand in stream order from the library's memory pool, kept until
 * dmuon_release_cache()).
 */
int dmuon_ns_orthogonalize(void* X, int64_t m, int64_t n, int steps, dmuon_stream_t stream);

/* Same, with element type `dtype` (DMUON_BF16 or DMUON_F32) and
 * caller-provided scratch of ws_bytes >= dmuon_ns_workspace_bytes(m, n, dtype)
 * (device memory, any contents; it must not be used by anything else until
 * the stream has finished the call). */
int dmuon_ns_orthogonalize_ex(void* X, int64_t m, int64_t n, int steps, int dtype,
                              void* workspace, size_t ws_bytes, dmuon_stream_t stream);
size_t dmuon_ns_workspace_bytes(int64_t m, int64_t n, int dtype);

/*
 * dmuon_muon_step_batched -- one Muon update of `count` matrices, with one
 * launch per stage for a whole group of them (the per-parameter loop of the
 * blog's Vanilla Muon, "代码实现" section, done as grouped kernels).  A call
 * of more than 2^28 elements runs as consecutive groups of at most about
 * that many (in the order given, at most 32 groups, one after the other on
 * the stream and sharing one scratch region); the result of each matrix does
 * not depend on the grouping.  With gradient clipping the call is one group.
 *   params[i]  device pointer to W_i (rows x cols, param_dtype), updated in place.
 *   grads[i]   device pointer to g_i (rows x cols, grad_dtype), read only; NULL
 *              skips matrix i entirely (no momentum, no update), as the blog
 *              skips parameters whose grad is None.
 *   bufs[i]    device pointer to the fp32 momentum buffer (rows x cols),
 *              updated in place.
 *   shapes[i]  host array, see dmuon_shape.
 *   lr, momentum, weight_decay   scalars (fp32); nesterov != 0 enables the
 *              Nesterov input; ns_steps >= 0.
 * No two matrices may overlap in memory.  count == 0 is a no-op.
 * Scratch as for dmuon_ns_orthogonalize.
 */
int dmuon_muon_step_batched(void* const params[], const void* const grads[], float* const bufs[],
                            const dmuon_shape shapes[], int count, float lr, float momentum,
                            int nesterov, float weight_decay, int ns_steps, dmuon_stream_t stream);

/* Same with caller-provided scratch of ws_bytes >= dmuon_workspace_bytes(). */
int dmuon_muon_step_batched_ex(void* const params[], const void* const grads[], float* const bufs[],
                               const dmuon_shape shapes[], int count, float lr, float momentum,
                               int nesterov, float weight_decay, int ns_steps, void* workspace,
                               size_t ws_bytes, dmuon_stream_t stream);

/*
 * Options of dmuon_muon_step_batched_opts.  Fill with
 * dmuon_step_options_default() (the pages' defaults: lr 0.02, momentum 0.95,
 * Nesterov, 5 steps of the cubic 1.5 / -0.5 iteration, no weight decay, no lr
 * scaling, no clipping), then change fields.
 *   ns_a, ns_b      coefficients of the cubic step X <- a X + b (X X^T) X
 *                   (the training guide's custom NewtonSchulz coefficients,
 *                   "超参数指南"; the blog's step is a = 1.5, b = -0.5).
 *   ns_c            != 0: the quintic step X <- a X + b A X + c A^2 X with
 *                   A = X X^T (the same custom coefficients read as a degree-5
 *                   odd polynomial; the pages print none).  A^2 is formed as a
 *                   symmetric product (upper tiles): one more launch and
 *                   m^3 more useful FLOPs per step, and one more m x m matrix
 *                   of scratch.  struct_size may also be the size without
 *                   this last field (then the step is cubic).
 *   lr_scale        DMUON_LR_PLAIN: lr as given.  DMUON_LR_SQRT_MAX: each
 *                   matrix uses lr * 0.2 * sqrt(max(rows, cols)) in place of lr
 *                   everywhere in its update (the guide's "internally scaled
 *                   per-param" note), weight decay included.
 *   max_grad_norm   > 0: Muon-only gradient clipping before the momentum
 *                   update (the guide's "梯度裁剪" section): with
 *                   ||g|| = sqrt(sum of g^2 over every matrix of the call),
 *                   each gradient enters the momentum as fl32(g * c),
 *                   c = fl32(min(1, max_grad_norm / (||g|| + 1e-6))).  The
 *                   gradient tensors themselves are not modified.
 *   grad_norm_out   optional DEVICE pointer (fp32): receives ||g|| when
 *                   clipping is on.
 */
enum { DMUON_LR_PLAIN = 0, DMUON_LR_SQRT_MAX = 1 };
typedef struct {
  size_t struct_size; /* sizeof(dmuon_step_options) */
  float lr, momentum, weight_decay;
  int nesterov, ns_steps;
  float ns_a, ns_b;
  int lr_scale;
  float max_grad_norm;
  float* grad_norm_out;
  float ns_c; /* quintic coefficient (0: the cubic step); see above */
} dmuon_step_options;
void dmuon_step_options_default(dmuon_step_options* opts);

/* One Muon update of `count` matrices with options (arguments otherwise as
 * dmuon_muon_step_batched).  workspace may be NULL (library arena) or a
 * caller buffer of ws_bytes >= dmuon_workspace_bytes_opts() (which equals
 * dmuon_workspace_bytes() for the cubic step). */
int dmuon_muon_step_batched_opts(void* const params[], const void* const grads[], float* const bufs[],
                                 const dmuon_shape shapes[], int count, const dmuon_step_options* opts,
                                 void* workspace, size_t ws_bytes, dmuon_stream_t stream);
/* Scratch bytes for dmuon_muon_step_batched_opts with these options (the
 * quintic step needs one more m x m matrix per matrix); 0 for invalid input. */
size_t dmuon_workspace_bytes_opts(const dmuon_shape shapes[], int count, const dmuon_step_options* opts);

/*
 * dmuon_muon_step_batched_reduce -- the owner's update of an owner-partitioned
 * data-parallel step (the quick start's "刚才发生了什么": each projection has
 * one owner that reduces its gradient and runs Newton-Schulz on it) with the
 * gradient reduction fused into the update: matrix i's gradient is the mean
 * of `world` buffers, grads[r * count + i] for r = 0 .. world-1, which the
 * prologue reads directly.  In a multi-GPU job these are other GPUs' buffers
 * mapped into this process (peer access, CUDA IPC or symmetric memory; the
 * caller makes sure every rank's gradient is complete first); any device
 * pointers work.  The mean is defined exactly: an fp32 sum in rank order,
 * then one fp32 division by `world` (round to nearest), so the momentum
 * buffers are reproducible bit for bit.  world == 1 is
 * dmuon_muon_step_batched_opts.
 *   grads      world * count device pointers, rank-major; for a matrix either
 *              every rank's pointer is NULL (the matrix is skipped) or none.
 *   world      1 .. 64.  Other arguments as dmuon_muon_step_batched_opts
 *              (clipping, when on, uses the norm of the mean gradients).
 */
int dmuon_muon_step_batched_reduce(void* const params[], const void* const grads[], float* const bufs[],
                                   const dmuon_shape shapes[], int count, int world,
                                   const dmuon_step_options* opts, void* workspace, size_t ws_bytes,
                                   dmuon_stream_t stream);

/*
 * dmuon_muon_step_batched_host -- the same Muon update (the blog's Vanilla
 * Muon step, "代码实现" section) for a caller whose gradients arrive in, and
 * whose updated weights must return to, page-locked host memory.  The
 * transfers overlap the update: the matrices are cut, in order, into
 * `chunks` consecutive groups of about equal gradient bytes (chunks <= 0:
 * one group per ~64 MiB of gradients; at most DMUON_MAX_CHUNKS and at most
 * one group per matrix).  Every group's gradients are uploaded on a library
 * copy stream; group c is updated on `stream` as soon as its upload has
 * landed (while later groups upload) and its weights are downloaded on a
 * second library copy stream while later groups compute.  The copy schedule
 * is this library's; the pages have no counterpart of it.  Device results
 * are bit-identical to dmuon_muon_step_batched_opts on the same tensors.
 *   params[i]       device W_i, updated in place (the resident weights).
 *   grads[i]        device staging buffer for g_i (rows x cols, grad_dtype),
 *                   overwritten with host_grads[i].
 *   bufs[i]         device fp32 momentum buffer, updated in place.
 *   host_grads[i]   page-locked host g_i (cudaHostAlloc or cudaHostRegister
 *                   memory), read only; NULL skips matrix i entirely.
 *   host_params[i]  page-locked host buffer of W_i's size that receives the
 *                   updated W_i; NULL: matrix i is not downloaded.
 *   opts            as for dmuon_muon_step_batched_opts, but max_grad_norm
 *                   must be 0: a global norm needs every gradient before the
 *                   first update, which would serialise the uploads.
 * Ordering: the uploads start after the work enqueued on `stream` before the
 * call; work enqueued on `stream` after the call starts after the last
 * download.  The host buffers must not be touched until then.  The two copy
 * streams are created on a device's first call and kept.  Errors: pageable
 * host memory or max_grad_norm > 0 -> DMUON_ERR_UNSUPPORTED, chunks >
 * DMUON_MAX_CHUNKS -> DMUON_ERR_INVALID_ARG, otherwise as
 * dmuon_muon_step_batched_opts; after an argument or allocation error nothing
 * is enqueued (a DMUON_ERR_CUDA from a copy or a launch may leave the groups
 * before it enqueued).  workspace:
 * NULL (library arena) or ws_bytes >= dmuon_workspace_bytes() of the whole
 * set (which covers every group).
 */
#define DMUON_MAX_CHUNKS 32
int dmuon_muon_step_batched_host(void* const params[], void* const grads[], float* const bufs[],
                                 const void* const host_grads[], void* const host_params[],
                                 const dmuon_shape shapes[], int count, const dmuon_step_options* opts,
                                 int chunks, void* workspace, size_t ws_bytes, dmuon_stream_t stream);

/*
 * dmuon_adamw_step_batched -- AdamW for the parameters the Muon path does
 * not orthogonalise (the training guide's second parameter group of
 * dmuon.Muon, "第 4 步：创建优化器": adamw_lr, adamw_betas, adamw_eps,
 * adamw_weight_decay), all tensors of the call in one launch.  Per element,
 * with c1 = fl32(1 - beta1), c2 = fl32(1 - beta2), bc1 = 1 - beta1^step,
 * bc2 = 1 - beta2^step:
 *   m <- fl(fl(beta1 m) + fl(c1 g))                 (two roundings, bit-exact)
 *   v <- fl(fl(beta2 v) + fl(fl(c2 g) g))
 *   p <- p (1 - lr wd) - (lr / bc1) m / (sqrt(v) / sqrt(bc2) + eps)   (fp32)
 *   params[i], grads[i]: device pointers of descs[i].numel elements
 *   (param_dtype / grad_dtype: DMUON_BF16 or DMUON_F32), any shape, flat;
 *   grads[i] == NULL skips tensor i.  exp_avgs[i], exp_avg_sqs[i]: fp32
 *   device buffers of the same length, updated in place.  step >= 1 is the
 *   step count including this one.  No scratch memory is used.
 */
typedef struct {
  int64_t numel;
  int32_t param_dtype, grad_dtype;
} dmuon_tensor_desc;
int dmuon_adamw_step_batched(void* const params[], const void* const grads[], float* const exp_avgs[],
                             float* const exp_avg_sqs[], const dmuon_tensor_desc descs[], int count,
                             float lr, float beta1, float beta2, float eps, float weight_decay,
                             int64_t step, dmuon_stream_t stream);

/*
 * dmuon_clip_grad_norm_buckets -- gradient clipping of several gradient
 * groups at once, each group ("segment") with its own norm and coefficient:
 * the training guide's fused clipping of the regular / Muon / AdamW
 * gradients ("梯度裁剪", "regular / Muon / AdamW 的融合 CUDA 裁剪"), which
 * computes every segment's norm, clip coefficient and in-place scaling in
 * one pass over the gradients while keeping per-segment semantics.  For each
 * segment s, as for the Muon-only clip of dmuon_step_options:
 *   ||g||_s = sqrt(sum of g^2 over every tensor of segment s)   (fp64 sums)
 *   c_s     = fl32(min(1, max_norms[s] / (||g||_s + 1e-6)))     (a NaN norm gives 1)
 *   g      <- fl32(g * c_s), rounded to nearest for bf16 storage, in place
 * Segments with c_s == 1 are not rewritten (the scaling is the identity).
 * The sums have a fixed order: results are identical run to run.
 *   grads[i]    device pointer of descs[i].numel elements (flat, any shape),
 *               updated in place; NULL skips tensor i.
 *   descs[i]    numel >= 1, dtype DMUON_BF16 or DMUON_F32, segment in [0, nseg).
 *   max_norms   HOST array of nseg values > 0; +inf measures a segment
 *               without scaling it.
 *   nseg        1 .. DMUON_MAX_SEGMENTS.  A segment without tensors has norm 0.
 *   norms_out   optional DEVICE pointer to nseg floats: ||g||_s before clipping.
 *   coefs_out   optional DEVICE pointer to nseg floats: c_s.
 *   workspace   NULL (library arena of the stream) or device scratch of
 *               ws_bytes >= dmuon_clip_workspace_bytes(), 256-byte aligned.
 * Launches: one norm pass, one block per segment for the coefficients, one
 * scale pass (more launches only past 512 tensors).  Errors as for the other
 * entry points; nothing is enqueued after an argument error.
 */
#define DMUON_MAX_SEGMENTS 64
typedef struct {
  int64_t numel;
  int32_t dtype, segment;
} dmuon_grad_desc;
size_t dmuon_clip_workspace_bytes(const dmuon_grad_desc descs[], int count, int nseg);
int dmuon_clip_grad_norm_buckets(void* const grads[], const dmuon_grad_desc descs[], int count,
                                 const float max_norms[], int nseg, float* norms_out, float* coefs_out,
                                 void* workspace, size_t ws_bytes, dmuon_stream_t stream);

/* Scratch bytes that suffice for dmuon_muon_step_batched_ex on these shapes
 * (matrices with a NULL gradient may be left out or counted; counting them
 * over-estimates): the need of the whole set as one group, which covers any
 * grouping of it.  Returns 0 for invalid shapes. */
size_t dmuon_workspace_bytes(const dmuon_shape shapes[], int count, int ns_steps);

/* Last error message of the calling host thread ("" if none). */
const char* dmuon_last_error(void);

/* Static description of the compiled backend, e.g.
 * "cubic NS · tcgen05 SYRK+GEMM · sm_100a" (cf. the training guide's
 * get_ns_backend() self-check in "日志与调试"). */
const char* dmuon_backend_string(void);

/* Device error word of the current device: 0 if no kernel reported a
 * problem, else a DMUON_ERR_* code.  Synchronises the device first.
 * clear != 0 resets the word to 0. */
int dmuon_device_status(int clear);

/* Frees the library's cached plans and scratch arenas and returns the pool's
 * memory (synchronises the device: the one call that does).  Safe to call at
 * any time from the host. */
void dmuon_release_cache(void);

/* Number of launch plans built in this process (a call with shapes seen
 * before builds none, whatever its tensor addresses). */
int64_t dmuon_plan_builds(void);

/* Test hook (host only, launches nothing): the stage kernels of the launch
 * plan used most recently (by the last call, or the plan it built).  Writes
 * one word per dtype group (at most max_groups; kernels may be NULL) and
 * returns the plan's number of groups, 0 when no plan exists.  Each word
 * ORs DMUON_PLAN_SYRK256 (the SYRK runs on 256 x 256 tiles, else 128 x 256)
 * DMUON_PLAN_GEMM_PAIR (the GEMM runs 256 x 256 tiles on two-CTA clusters,
 * else 128 x 256 tiles on single CTAs) and DMUON_PLAN_SQUARE256 (quintic
 * plans: the SQUARE stage runs on 256 x 256 tiles, else 128 x 256). */
#define DMUON_PLAN_SYRK256 1
#define DMUON_PLAN_GEMM_PAIR 2
#define DMUON_PLAN_SQUARE256 4
int dmuon_debug_last_plan(int* kernels, int max_groups);

/* Test hook (host only, launches nothing): the device-memory check the entry
 * points apply to every tensor address.  DMUON_OK for device or managed
 * memory, DMUON_ERR_INVALID_ARG for host memory (page-locked or not) and
 * NULL. */
int dmuon_debug_check_pointer(const void* p);

/*
 * dmuon_ns_orthogonalize_noalloc -- same result as dmuon_ns_orthogonalize
 * (bf16, in place), for callers that may not allocate device memory: code
 * running inside a framework that has already reserved the device's memory
 * for its own pool, sandboxed plugins that are not allowed to call
 * cudaMalloc, and latency-critical paths where cudaMalloc/cudaFree could
 * block or synchronise the device.  It calls no allocation routine.  (The
 * pages have no counterpart of this entry point; it is a property of this
 * library.)
 *   Scratch: a fixed 32 MiB device array inside the library.  The driver
 *   allocates it when the library's module is loaded on a device, i.e. at the
 *   first call of any entry point there, and it is held until the process
 *   exits; a caller that pre-reserves the device's memory should make one
 *   library call first.  Matrices whose scratch
 *   (dmuon_ns_workspace_bytes(m, n, DMUON_BF16) for steps >= 2) exceeds
 *   32 MiB - 16 KiB are rejected with DMUON_ERR_UNSUPPORTED; e.g. 2048 x 2048
 *   and 1024 x 4096 fit, 4096 x 4096 does not.
 *   Sharing: every call uses the same array, and nothing carries over from
 *   one call to the next: each call writes its own launch description
 *   (descriptor and tensor maps, passed as kernel parameters of a small
 *   upload kernel on `stream`) at the front of the array.  Calls that may
 *   overlap on the GPU (different streams without ordering between them) race
 *   on it; calls on one stream are ordered.
 *   Set-up: the first call on a device looks up the array's device address
 *   (once per device); make that first call before any stream capture.
 */
int dmuon_ns_orthogonalize_noalloc(void* X, int64_t m, int64_t n, int steps, dmuon_stream_t stream);

/* Kernel kinds reported by the timing and launch counters below. */
enum {
  DMUON_KERNEL_PROLOGUE = 0, /* momentum, Nesterov input, norm partials, copy into X */
  DMUON_KERNEL_FINALIZE = 1, /* per-matrix norm and scale */
  DMUON_KERNEL_SYRK = 2,     /* A = X X^T (upper tiles) */
  DMUON_KERNEL_GEMM = 3,     /* X <- 1.5 X - 0.5 A X, last step fused with the update */
  DMUON_KERNEL_APPLY = 4,    /* update for ns_steps == 0 */
  DMUON_KERNEL_ADAMW = 5,    /* AdamW of the non-orthogonalised parameters */
  DMUON_KERNEL_CLIP = 6,     /* per-segment gradient clipping (norms, coefficients, scaling) */
  DMUON_KERNEL_SQUARE = 7,   /* quintic coefficients: P = b A + c A A (upper tiles) */
  DMUON_KERNEL_KINDS = 8
};

/* Per-kernel timing: while enabled, every launch is bracketed by CUDA events
 * recorded on the caller's stream (so the numbers are device time of that
 * stream).  dmuon_stage_times() synchronises the device, adds up the elapsed
 * time of every bracketed launch since the last reset, and fills ms[k] and
 * launches[k] for k < n (n <= DMUON_KERNEL_KINDS); reset != 0 clears them. */
int dmuon_stage_timing(int enable);
int dmuon_stage_times(double* ms, int64_t* launches, int n, int reset);

/* Number of kernels this library has launched in this process. */
int64_t dmuon_launch_count(void);

/* Test hook: the next `n` library allocations fail as if the device were out
 * of memory (host-side fault injection; 0 disables). */
void dmuon_debug_fail_allocations(int n);

/* Test hook (host only, no CUDA call): the grouping the library uses for these
 * shapes.  which = 0: the groups of a device call (dmuon_muon_step_batched
 * and friends, without clipping); which = 1: the automatic groups of
 * dmuon_muon_step_batched_host (by gradient bytes).  Writes the group
 * boundaries (bounds[0] = 0, ..., bounds[groups] = count) and returns the
 * number of groups, or DMUON_ERR_INVALID_ARG (bad shapes, cap < groups + 1). */
int dmuon_debug_partition(const dmuon_shape shapes[], int count, int which, int* bounds, int cap);

/* Test hook: launches one CTA that waits on a barrier nothing arrives at,
 * with a wait limit of `limit_us` microseconds, then records
 * DMUON_ERR_TIMEOUT in the device error word and returns.  Exercises the
 * bounded-wait path of the kernels without hanging the GPU. */
int dmuon_debug_wait_timeout(int limit_us, dmuon_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* DMUON_H_ */
