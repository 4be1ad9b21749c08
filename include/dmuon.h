/*
 * dmuon.h - C ABI of the B200 (sm_100a) Muon-step library.
 *
 * One Muon optimizer step over a list of 2D matrices, on one GPU:
 *   momentum -> Nesterov input -> Frobenius normalisation -> ns_steps quintic
 *   Gram Newton-Schulz iterations -> decoupled weight decay + shape-scaled update.
 *
 * The method is the per-owner step of DMuon (DMuon Training Guide, "Step 4:
 * Create Optimizer" and its "Hyperparameter Guide" table; DMuon FAQ, "Why isn't
 * DMuon just ZeRO-1?" - Newton-Schulz needs the whole (m, n) gradient - and
 * "What related work should I cite?" - the default "gram" backend follows Gram
 * Newton-Schulz).  Per matrix of shape R x C, with m = min(R,C), n = max(R,C):
 *
 *   buf' = mu*buf + g
 *   x0   = g + mu*buf'  (nesterov)   |   buf'  (otherwise)
 *   X    = orient(x0) / (||x0||_F + 1e-7)      orient = transpose when R > C
 *   repeat ns_steps:  G = X X^T ;  X = a X + (b G + c G G) X
 *   O    = orient^-1(X)
 *   p'   = p (1 - lr wd) - lr * 0.2 * sqrt(n) * O
 *
 * Conventions common to every call:
 *  - Pointers named "device" are CUDA device pointers owned by the caller; the
 *    library never frees them.  Matrices are row-major and contiguous unless a
 *    leading dimension is given.
 *  - Every call is asynchronous on `stream` (a cudaStream_t; NULL = legacy
 *    default stream).  Nothing synchronises the host except
 *    dmuon_stream_status().
 *  - Arguments are validated on the host before anything is launched; on an
 *    error nothing is modified and the status says why (dmuon_get_last_error()
 *    holds a message, per host thread).
 *  - A CUDA error after launches began (DMUON_ERR_CUDA) can leave a step
 *    partly done (some buffers or parameters updated); the call still returns
 *    with all of its work ordered before later work on `stream`, so the
 *    caller can synchronise and restore its own copy.  DMUON_FAULT_INJECT=
 *    launch makes dmuon_step report such a failure before its first chain
 *    (momentum of the first chunk done, no parameter touched), for tests.
 *  - Device waits inside the kernels are bounded; a wait that runs out sets a
 *    per-device status word read by dmuon_stream_status() (DMUON_ERR_TIMEOUT).
 *  - A debug build of the library (compiled with -DDMUON_DEBUG:
 *    `build.py --debug` writes libdmuon_b200_debug.so) checks every global
 *    access of its kernels against the extent of the buffer it belongs to,
 *    computed on the host; an access outside is skipped and the status word
 *    records DMUON_ERR_BOUNDS (no trap, no fault).  Release builds carry no
 *    checks.
 *  - Results do not depend on how matrices are batched: a matrix gives the
 *    same bits alone, inside its group, or in a permuted list.
 */
#ifndef DMUON_H
#define DMUON_H

#include <stdint.h>

#if defined(__GNUC__)
#define DMUON_API __attribute__((visibility("default")))
#else
#define DMUON_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t. */
typedef struct CUstream_st* dmuon_stream_t;

typedef enum {
    DMUON_OK = 0,
    DMUON_ERR_INVALID_ARG = 1, /* bad pointer, size, dtype, alignment or count */
    DMUON_ERR_UNSUPPORTED = 2, /* no sm_100 device, or a size beyond a limit  */
    DMUON_ERR_CUDA = 3,        /* a CUDA runtime/driver call failed             */
    DMUON_ERR_OOM = 4,         /* workspace allocation failed                   */
    DMUON_ERR_TIMEOUT = 5,     /* a bounded device-side wait ran out            */
    DMUON_ERR_BOUNDS = 6       /* debug builds: an access outside its buffer was
                                  caught and skipped (see dmuon_stream_status)  */
} dmuon_status_t;

typedef enum {
    DMUON_F32 = 0,  /* fp32 storage; FFMA Newton-Schulz (fp32 X, G, p(G))            */
    DMUON_BF16 = 1  /* bf16 storage; tcgen05 tensor-core chain with fp32 accumulation */
} dmuon_dtype_t;

/* Shape of one matrix of a Muon step. */
typedef struct {
    int64_t rows;
    int64_t cols;
    int32_t dtype;     /* dmuon_dtype_t of param, grad and momentum buffer */
    int32_t reserved;  /* must be 0 */
} dmuon_shape_t;

/* Default quintic coefficients used when `coeffs` is NULL (the pages print
 * none; this is the widely used Muon triple). */
#define DMUON_DEFAULT_A 3.4445f
#define DMUON_DEFAULT_B (-4.7750f)
#define DMUON_DEFAULT_C 2.0315f
#define DMUON_NORM_EPS 1e-7f

/* ------------------------------------------------------------------------ */
/* Whole-path calls                                                          */
/* ------------------------------------------------------------------------ */

/*
 * dmuon_ns - orthogonalise one bf16 matrix with the Gram Newton-Schulz
 * iteration (DMuon Training Guide, Hyperparameter Guide: ns_steps and the
 * "gram" ns_backend rows).
 *   X      device, rows x cols bf16, row-major contiguous (read only)
 *   out    device, rows x cols bf16; may not overlap X
 *   rows, cols  > 0; rows*cols < 2^31
 *   steps  >= 0; steps == 0 gives out = X / (||X||_F + eps)
 *   coeffs HOST array of 3*steps floats (a_k, b_k, c_k for iteration k), or
 *          NULL for the default triple at every iteration
 * Works over the smaller side (transposes internally when rows > cols).
 * Uses the library's cached workspace for this (device, stream).  The shape
 * decides the path as for dmuon_step (see there); on the tensor-core path the
 * last two iterations of wide matrices are carried out as one block in Gram
 * space (the same result in exact arithmetic, fewer flops); see
 * dmuon_gram_poly.
 */
DMUON_API dmuon_status_t dmuon_ns(const void* X, void* out, int64_t rows, int64_t cols, int32_t steps,
                        const float* coeffs, dmuon_stream_t stream);

/* dmuon_ns with an explicit dtype (DMUON_F32 selects the fp32 FFMA path). */
DMUON_API dmuon_status_t dmuon_ns_ex(const void* X, void* out, int64_t rows, int64_t cols, int32_t steps,
                           const float* coeffs, int32_t dtype, dmuon_stream_t stream);

/*
 * dmuon_step - one Muon step over `count` matrices (DMuon Training Guide,
 * "Step 4": group 0, "momentum + NS + update").
 *   params, grads, mom_bufs  HOST arrays of `count` DEVICE pointers; matrix i
 *          is shapes[i].rows x shapes[i].cols, row-major contiguous, in
 *          shapes[i].dtype.  params and mom_bufs are updated in place; grads
 *          are read only.  No two matrices may overlap.
 *   shapes HOST array of `count` shapes (reserved fields 0)
 *   count  >= 0 (0 is a no-op)
 *   lr     Muon learning rate; the update uses lr * 0.2 * sqrt(max(R, C))
 *          (Hyperparameter Guide, lr row), the decay uses lr
 *   momentum  mu (default 0.95 on the pages); nesterov 0/1 (default 1)
 *   ns_steps  >= 0 (default 5); coeffs as for dmuon_ns
 *   wd     decoupled weight decay: p <- p (1 - lr wd) - ...
 * Matrices are grouped by shape (dmuon_plan_groups) and each group runs as
 * batched launches.  The library's workspace (cached per device and stream,
 * at most DMUON_WS_CAP_MB, default 8 GiB, unless one matrix alone needs more:
 * it then runs as a chunk of its own and the step runs without the
 * double-buffered overlap) is allocated stream-ordered on
 * first use or growth; after one call with the same shapes on the same
 * stream, a call allocates nothing and can be captured in a CUDA graph (a
 * call that would grow the workspace while its stream is capturing returns
 * DMUON_ERR_INVALID_ARG instead).  On the bf16 tensor-core path the update
 * runs inside the chain's last product (its epilogue writes the parameters;
 * DMUON_FUSED_UPDATE=0 runs it as a separate pass, with the same bits).  With
 * several chunks the momentum stage (and any separate update) runs on an
 * internal least-priority stream underneath the Newton-Schulz chains, which
 * run on internal greatest-priority streams (two chunks whose chains are one
 * launch each may run at once); all fork from `stream` and are joined back
 * into it before the call returns, on error paths too.  The results do not
 * depend on that schedule.
 *
 * Routing by shape (m = min(R, C), n = max(R, C)), all in one call: fp32
 * matrices run an FFMA chain with fp32 X, G and p(G); bf16 matrices with
 * m <= 64 keep G and p(G) in fp32 (FFMA); bf16 matrices with m < 256 and
 * n < 3 m keep X in fp32 as well (FFMA; bf16 storage of X cannot resolve the
 * many small singular values of such near-square matrices within 2e-2); all
 * other bf16 matrices run the tcgen05 chain, whose last two iterations run
 * in Gram space when n >= 2 m, or n >= 1.25 m and m >= 512.
 */
DMUON_API dmuon_status_t dmuon_step(void* const* params, const void* const* grads, void* const* mom_bufs,
                          const dmuon_shape_t* shapes, int32_t count, float lr, float momentum,
                          int32_t nesterov, int32_t ns_steps, const float* coeffs, float wd,
                          dmuon_stream_t stream);

/*
 * dmuon_step_clipped - dmuon_step on globally clipped gradients (DMuon
 * Training Guide, "Gradient Clipping": clip after the reduce, before
 * momentum + Newton-Schulz).  One norm pass reads every gradient, one block
 * forms coef = min(1, max_norm / (total + 1e-6)); the momentum kernel then
 * uses fl_T(g * fl32(coef)) (fl_T: rounding to the gradient's own dtype) in
 * place of g.  The result equals dmuon_clip_grad_norm followed by dmuon_step,
 * bit for bit, but the gradients are NOT modified (read-only, as in
 * dmuon_step) and no scaled copy is written.  Arguments as dmuon_step, plus
 * max_norm / norm_type / total_norm as dmuon_clip_grad_norm.
 */
DMUON_API dmuon_status_t dmuon_step_clipped(void* const* params, const void* const* grads, void* const* mom_bufs,
                                            const dmuon_shape_t* shapes, int32_t count, float lr, float momentum,
                                            int32_t nesterov, int32_t ns_steps, const float* coeffs, float wd,
                                            float max_norm, float norm_type, double* total_norm,
                                            dmuon_stream_t stream);

/*
 * dmuon_clip_grad_norm - global p-norm clipping of the Muon gradients, in
 * place (DMuon Training Guide, "Gradient Clipping": the Muon-only clip runs
 * after the gradient reduce and before momentum + Newton-Schulz; the default
 * strategy is global p-norm clipping).  Read with PyTorch's clip_grad_norm_
 * formula: the section gives DMuon's clip that routine's name and max_norm
 * argument and uses the two side by side:
 *   total = (sum over every element of every matrix of |g|^p)^(1/p)
 *           (p = inf: max |g|)
 *   coef  = min(1, max_norm / (total + 1e-6)) (NaN if total is NaN),
 *   g <- fl(g * fl32(coef))
 * Every gradient is rewritten; with coef = 1 the values are unchanged.
 *   grads      HOST array of `count` DEVICE pointers (shapes[i], row-major)
 *   shapes     HOST array of `count` shapes; gradients must not overlap
 *   max_norm   finite, >= 0
 *   norm_type  1, 2 or INFINITY (others: DMUON_ERR_UNSUPPORTED)
 *   total_norm DEVICE double or NULL: receives `total`
 * Deterministic (fixed-order fp64 reduction of per-tile fp32 partials).
 * Non-finite gradients follow PyTorch's formula: a NaN anywhere makes `total`
 * NaN and coef NaN, so every gradient becomes NaN; an infinity (and no NaN)
 * makes `total` inf and coef 0 (finite values become 0, infinities NaN).
 * `total` is the value to check for non-finite gradients before a step.
 */
DMUON_API dmuon_status_t dmuon_clip_grad_norm(void* const* grads, const dmuon_shape_t* shapes, int32_t count,
                                              float max_norm, float norm_type, double* total_norm,
                                              dmuon_stream_t stream);

/*
 * dmuon_clip_grad_norm_buckets - several independent global-norm clips in one
 * set of launches (DMuon Training Guide, "Fused CUDA clip for regular / Muon /
 * AdamW": when several gradient groups are clipped together, the norms, the
 * clip coefficients and the in-place scaling of every bucket are computed
 * together, each bucket with the semantics of its own clip).  Bucket k is
 * clipped exactly as dmuon_clip_grad_norm would clip its gradients alone, with
 * max_norms[k] and norm_types[k]: the same formula, reduction order and bits.
 * A gradient of any rank is passed as rows x cols with rows * cols = its
 * element count (the clip reads every gradient as one flat array).
 *   grads, shapes, count  every bucket's gradients, as for dmuon_clip_grad_norm
 *                 (none may overlap another, in any bucket)
 *   bucket_of    HOST array of `count` ints in [0, num_buckets)
 *   num_buckets  1 .. 128
 *   max_norms    HOST array of num_buckets floats, each finite and >= 0
 *   norm_types   HOST array of num_buckets floats, each 1, 2 or INFINITY
 *   total_norms  DEVICE array of num_buckets doubles, or NULL: bucket k's
 *                total in total_norms[k] (0 for an empty bucket)
 * Launches on `stream`: the norm partials of every bucket's same-shape tables,
 * one launch computing every bucket's total and coefficient (one block per
 * bucket), the in-place scaling of every table.  A NaN in one bucket makes
 * that bucket's gradients NaN and leaves the others alone.  Errors: as
 * dmuon_clip_grad_norm, plus DMUON_ERR_INVALID_ARG for a bucket index out of
 * range or a bad count of buckets.
 */
DMUON_API dmuon_status_t dmuon_clip_grad_norm_buckets(void* const* grads, const dmuon_shape_t* shapes,
                                                      int32_t count, const int32_t* bucket_of,
                                                      int32_t num_buckets, const float* max_norms,
                                                      const float* norm_types, double* total_norms,
                                                      dmuon_stream_t stream);

/*
 * dmuon_plan_groups - the shape grouping dmuon_step uses (host only, no GPU).
 * Matrices with equal (rows, cols, dtype) form a group; group ids follow
 * first appearance; `order` lists the groups one after another, members in
 * ascending index.
 *   shapes    HOST array of `count` shapes
 *   group_of  HOST out, `count` ints (group id of matrix i)
 *   order     HOST out, `count` ints (execution order)
 *   num_groups HOST out, 1 int
 */
DMUON_API dmuon_status_t dmuon_plan_groups(const dmuon_shape_t* shapes, int32_t count, int32_t* group_of,
                                 int32_t* order, int32_t* num_groups);

/*
 * dmuon_assign_owners - dedicated ownership of the matrices over `world`
 * ranks (host only, no GPU).  DMuon FAQ, "Why isn't DMuon just ZeRO-1?": one
 * rank owns a whole matrix and runs its Muon step, the other ranks receive the
 * updated parameter; Training Guide, "Verify Parameter Assignment": the
 * assignment is load-balanced and reported with per-rank loads and an
 * imbalance.  The pages give no rule; this one: the load of a matrix is the
 * flops of one Newton-Schulz iteration, 3 m^2 n + m^3 (m = min side); matrices
 * go from the most expensive down (equal costs: lower index first), each to the
 * rank with the least load so far (equal loads: lower rank).  The same input
 * gives the same assignment on every rank.
 *   shapes     HOST array of `count` shapes
 *   world      number of ranks, >= 1
 *   owner_of   HOST out, `count` ints: the rank that owns matrix i
 *   loads      HOST out, `world` doubles: the flops each rank owns
 *   imbalance  HOST out, 1 double: max(loads) / mean(loads) - 1 (0 when empty)
 */
DMUON_API dmuon_status_t dmuon_assign_owners(const dmuon_shape_t* shapes, int32_t count, int32_t world,
                                             int32_t* owner_of, double* loads, double* imbalance);

/* ------------------------------------------------------------------------ */
/* Stage calls: the individual kernels of the path, over `batch` matrices    */
/* stored one after another (matrix b starts at b * rows * ld elements).     */
/* dtype DMUON_BF16 runs the tcgen05 tensor-core kernels (bf16 in and out,   */
/* fp32 accumulation; ld a multiple of 8, pointers 16-byte aligned);         */
/* DMUON_F32 runs the FFMA kernels (fp32 in and out).                        */
/* ------------------------------------------------------------------------ */

/*
 * dmuon_gram - G = alpha * X X^T (the Gram matrix of one Gram Newton-Schulz
 * iteration, over the smaller side).  Only one triangle is computed; the
 * other is written as its mirror, so G is exactly symmetric.
 *   X  device, batch x m x n (leading dimension ldx >= n)
 *   G  device, batch x m x m (leading dimension ldg >= m); may not overlap X
 */
DMUON_API dmuon_status_t dmuon_gram(const void* X, void* G, int64_t batch, int64_t m, int64_t n,
                          int64_t ldx, int64_t ldg, float alpha, int32_t dtype,
                          dmuon_stream_t stream);

/*
 * dmuon_gram_poly - P = b G + c G G for a symmetric G (so that
 * p(G) = a I + P).  One triangle computed, the other mirrored.  The kernel
 * behind it computes the general symmetric product p1 (A B) + p0 E + p2 I of
 * commuting symmetric A, B, which the Gram-space block uses internally.
 *   G  device, batch x m x m (ldg); P device, batch x m x m (ldp), no overlap
 */
DMUON_API dmuon_status_t dmuon_gram_poly(const void* G, void* P, int64_t batch, int64_t m, int64_t ldg,
                               int64_t ldp, float b, float c, int32_t dtype,
                               dmuon_stream_t stream);

/*
 * dmuon_poly_apply - Y = alpha * (a X + P X)  ( = alpha * p(G) X ).
 *   P  device, batch x m x m (ldp);  X device, batch x m x n (ldx)
 *   Y  device, batch x m x n (ldy); may not overlap X or P
 */
DMUON_API dmuon_status_t dmuon_poly_apply(const void* P, const void* X, void* Y, int64_t batch, int64_t m,
                                int64_t n, int64_t ldp, int64_t ldx, int64_t ldy, float a,
                                float alpha, int32_t dtype, dmuon_stream_t stream);

/*
 * dmuon_momentum - the momentum stage for one matrix, in place on `buf`:
 *   buf' = mu*buf + g ;  x0 = g + mu*buf' (nesterov) or buf'
 * in fp32 with each operation rounded (no fused multiply-add), stored in
 * `dtype` (bf16 round-to-nearest-even).  x0 uses the unrounded fp32 buf'.
 *   buf, grad, x0  device, rows x cols, row-major contiguous
 *   sumsq  device, 1 double, or NULL: receives sum of squares of stored x0
 */
DMUON_API dmuon_status_t dmuon_momentum(void* buf, const void* grad, void* x0, int64_t rows, int64_t cols,
                              float momentum, int32_t nesterov, int32_t dtype, double* sumsq,
                              dmuon_stream_t stream);

/*
 * dmuon_update - the update stage for one matrix, in place on `param`:
 *   p' = fl(p * fl(1 - lr*wd)) - fl(s * O),  s = fl32(lr * 0.2 * sqrt(max(rows,cols)))
 *   param, O  device, rows x cols in dtype, row-major contiguous
 */
DMUON_API dmuon_status_t dmuon_update(void* param, const void* O, int64_t rows, int64_t cols, float lr,
                            float wd, int32_t dtype, dmuon_stream_t stream);

/* ------------------------------------------------------------------------ */
/* Allocation-free variant                                                   */
/* ------------------------------------------------------------------------ */

/* Size of the fixed scratch array behind dmuon_ns_noalloc (32 MiB).  Every
 * GPU on which the library is loaded holds this array until the process
 * exits. */
#define DMUON_NOALLOC_SCRATCH_BYTES (32u << 20)

/*
 * dmuon_ns_noalloc - dmuon_ns_ex for callers that must not allocate device
 * memory.  The DMuon documentation has no counterpart: this entry point
 * exists for callers such as a framework that has handed the whole device to
 * its own caching allocator, or a loop that may not allocate after start-up
 * (cudaMalloc can synchronise the device and its cost is unpredictable).
 * Instead of the cached workspace of dmuon_ns_ex it uses one fixed
 * DMUON_NOALLOC_SCRATCH_BYTES array in device memory that the library
 * reserves when it is loaded; it never calls cudaMalloc or cudaFree.  It runs
 * the kernels of dmuon_ns_ex in the same order, so both give the same bits.
 *   X, out, rows, cols, steps, coeffs, dtype  as for dmuon_ns_ex
 *   status  device, 1 int32, or NULL: cleared at the start of the call, then
 *           set to DMUON_ERR_TIMEOUT if a bounded device wait ran out (with
 *           NULL the word lives in the scratch array and is not reported)
 * Limit: the problem must fit the array; a matrix whose workspace (two m x n
 * copies of X, the Gram-sized m x m matrices of its schedule - two, or five
 * for a wide bf16 matrix whose last iterations run in Gram space - and the
 * norm partials, m = min(rows, cols)) exceeds it is rejected with
 * DMUON_ERR_INVALID_ARG and a message naming both sizes.  Examples that fit:
 * bf16 4096 x 1024 and 2048 x 1024, fp32 2048 x 1024; bf16 2048 x 2048 does
 * not.
 * Set-up: the first call on each device, with that device current, looks up
 * the array's device address; make that first call before any stream
 * capture.  A set-up that fails is not remembered: the next call retries it.
 * Sharing: every call on a device uses the same array and leaves its
 * contents behind; calls that can overlap on the GPU (different streams
 * without ordering between them, or several host threads) race on it and
 * must be serialised by the caller.
 */
DMUON_API dmuon_status_t dmuon_ns_noalloc(const void* X, void* out, int64_t rows, int64_t cols,
                                          int32_t steps, const float* coeffs, int32_t dtype,
                                          int32_t* status, dmuon_stream_t stream);

/* ------------------------------------------------------------------------ */
/* Status, workspace, build information                                      */
/* ------------------------------------------------------------------------ */

/* Message for the last non-OK status returned on this host thread. */
DMUON_API const char* dmuon_get_last_error(void);

/* Synchronises `stream`, then reads and clears the device status word of the
 * current device: DMUON_ERR_TIMEOUT if a device-side wait ran out since the
 * last call, DMUON_ERR_BOUNDS if a debug build caught an access outside its
 * buffer, DMUON_ERR_CUDA if the stream reports an error, else DMUON_OK. */
DMUON_API dmuon_status_t dmuon_stream_status(dmuon_stream_t stream);

/* Self-test of failure detection: launches one thread that waits on a device
 * barrier nothing will arrive on, with the same bounded wait the tensor-core
 * kernels use, limited to limit_us (1..2000000) microseconds.  The wait gives
 * up, records DMUON_ERR_TIMEOUT in the device status word and the kernel
 * returns; the next dmuon_stream_status() reports DMUON_ERR_TIMEOUT and clears
 * the word, and the context stays usable. */
DMUON_API dmuon_status_t dmuon_selftest_timeout(int32_t limit_us, dmuon_stream_t stream);

/* Self-test of the debug build's bounds checks: launches one thread that
 * evaluates a single check of an element offset just past a one-element
 * extent, and touches no memory either way.  In a debug build the check fails
 * and records DMUON_ERR_BOUNDS, which the next dmuon_stream_status() reports
 * (and clears); in a release build there are no checks and the status stays
 * DMUON_OK.  dmuon_build_info() names the build ("debug bounds checks"). */
DMUON_API dmuon_status_t dmuon_selftest_bounds(dmuon_stream_t stream);

/* Frees every cached workspace of the calling thread's current device after
 * synchronising the device.  Safe to call at any time between calls. */
DMUON_API void dmuon_release_workspace(void);

/* Bytes of workspace dmuon_step would use for these shapes (host only). */
DMUON_API int64_t dmuon_workspace_bytes(const dmuon_shape_t* shapes, int32_t count, int32_t ns_steps);

/* Number of kernels dmuon_step launches for these shapes (host only). */
DMUON_API int64_t dmuon_step_launches(const dmuon_shape_t* shapes, int32_t count, int32_t ns_steps);

/*
 * Per-kernel timing.  Between dmuon_profile_start() and dmuon_profile_stop()
 * every kernel that the calling host thread's calls enqueue is bracketed by
 * two CUDA events on its stream.  dmuon_profile_stop() waits for the last
 * event, then fills up to max_stats entries (one per kernel kind) and returns
 * how many kinds were seen (or -1 on a CUDA error).  "flops" and "bytes" are
 * the algorithmic work of the launches: gram m^2 n, poly m^3, apply 2 m^2 n
 * flops per matrix; momentum 4, update 3 element accesses per element.
 */
typedef struct {
    char name[32];
    int64_t launches;
    double total_ms;
    double flops;
    double bytes;
} dmuon_kernel_stat_t;

DMUON_API dmuon_status_t dmuon_profile_start(void);
DMUON_API int32_t dmuon_profile_stop(dmuon_kernel_stat_t* stats, int32_t max_stats);

/*
 * dmuon_profile_stop_launches - ends the same profiling window as
 * dmuon_profile_stop (use one or the other), but reports every launch, in
 * the order the calls enqueued them: its kernel kind, its duration, its
 * start relative to the first launch's start (launches on two streams may
 * overlap), and its algorithmic work.  Fills up to max_recs records and
 * returns the number of launches (or -1 on a CUDA error).
 */
typedef struct {
    char name[32];
    double start_ms;
    double ms;
    double flops;
    double bytes;
} dmuon_launch_record_t;

DMUON_API int32_t dmuon_profile_stop_launches(dmuon_launch_record_t* recs, int32_t max_recs);

/* Static string: version, target architecture, tile configuration. */
DMUON_API const char* dmuon_build_info(void);

#ifdef __cplusplus
}
#endif
#endif /* DMUON_H */
