/*
 * muon.h -- C ABI of the B200 (sm_100a) Muon optimizer-step library.
 *
 * The library orthogonalises 2D momentum matrices with Newton-Schulz (NS)
 * iterations and applies the Muon update, entirely in CUDA kernels on the
 * bound stream.  Sources of the method (web pages, cited by title + section):
 *
 *  [Gram-NS]       "GPU เร่งความเร็วใหม่! อัลกอริทึม Gram Newton-Schulz ..."
 *                  (itsolotime.com): Muon = steepest descent under the spectral
 *                  norm with polar(X) = U V^T approximated by NS, three matrix
 *                  products per standard step ("ข้อได้เปรียบของอัลกอริทึม");
 *                  the Gram form iterates on R = X X^T via p(t) = t q(t^2) and
 *                  needs a restart in half precision
 *                  ("ความท้าทายด้านความเสถียรและแนวทางแก้ไข").
 *  [NanoGPT-Muon]  "2 分钟训练 124M 参数 NanoGPT：Muon 优化器与工程复现实践"
 *                  (blog.hotdry.top): coefficients (3.4445, -4.7750, 2.0315),
 *                  five steps, bfloat16 ("Newton-Schulz 迭代的系数调优与 FLOP
 *                  开销分析"); momentum 0.95 with Nesterov ("工程复现清单").
 *
 * Conventions common to every call
 *  - Matrices are dense row-major, rows x cols, element (i, j) at i*cols + j.
 *  - The iteration runs on the short side: a matrix with rows > cols is
 *    processed as its transpose and the result is written back in the
 *    caller's layout.
 *  - All tensor pointers are DEVICE pointers owned by the caller; arrays of
 *    pointers, shapes and coefficients are HOST arrays read during the call.
 *  - Work is enqueued asynchronously on the stream set by muon_set_stream
 *    (default: the legacy default stream).  No call synchronises the host
 *    except muon_device_status and muon_profile_read.
 *  - The library owns a cached device workspace sized for the last shape set
 *    (released by muon_release_workspace or at unload).  Calls are not
 *    thread-safe; use one thread per library instance.  Calls may switch
 *    streams: a call's use of the workspace is ordered after the previous
 *    call's, on whichever stream that ran (an event wait, not a host sync).
 *    The caller's own tensors are not synchronised across streams.
 *  - CUDA graphs: muon_step, muon_orthogonalize, muon_adamw_step and
 *    muon_hybrid_step may be captured (stream capture of the bound stream)
 *    once the same call has run before the capture: a capture never builds
 *    a plan or uploads a table (MUON_ERR_UNSUPPORTED, nothing enqueued, if it
 *    would have to).  Under capture the cross-stream workspace ordering is
 *    left to the capture and the graph's launches.  Scalars (mu, lr, the
 *    AdamW step count and its bias corrections) are launch arguments: a
 *    graph replays the values it was captured with.
 *  - Every call returns a status (< 0 on error) and never throws.  On an
 *    argument error nothing is enqueued; muon_last_error() describes it.
 *  - Every device-side wait (a CTA pair waiting for its operands, for another
 *    tile's results, or for its accumulator) is bounded: after the limit the
 *    kernel records MUON_ERR_TIMEOUT in the device status word, drains its own
 *    copies and tensor-core work, frees its tensor memory and exits.
 *  - Environment knobs, read when a plan is built (tests and debugging):
 *    MUON_WAIT_LIMIT_MS  bound of every device-side wait (1..10000, default 1000)
 *    MUON_FAULT          alloc | launch | timeout: fail the workspace
 *                        allocation (MUON_ERR_NO_MEMORY) or the first launch
 *                        (MUON_ERR_CUDA) of a call before anything is
 *                        enqueued, or give the first tile of a chained launch
 *                        a dependency that is never met (MUON_ERR_TIMEOUT
 *                        after the wait limit)
 *    MUON_CHAIN_LAUNCH / MUON_SLOT_LAUNCHES  force one launch for the whole
 *                        Newton-Schulz chain / one launch per chain slot
 *    MUON_TMA_STORE=0    plain per-lane stores in the GEMM epilogue
 *    MUON_TILE_N=256|512 per-slot launches use 256-wide tiles only / 512-wide
 *                        tiles always (default: chosen per launch)
 *    MUON_DEBUG_CANARY=1 every workspace region is followed by a 1 KB guard
 *                        of a fixed byte pattern; after each call's launches
 *                        a check kernel compares every guard with it (and
 *                        restores it), so muon_device_status returns
 *                        MUON_ERR_GUARD after a write past a region's end
 *    MUON_PROFILE_VERBOSE  print every traced launch to stderr
 */
#ifndef MUON_B200_H
#define MUON_B200_H

#if defined(__GNUC__)
#define MUON_API __attribute__((visibility("default")))
#else
#define MUON_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

#define MUON_VERSION 10000 /* 1.0.0 */

/* status codes */
#define MUON_OK 0
#define MUON_ERR_INVALID_ARG (-1) /* null pointer, non-positive size, bad steps/count */
#define MUON_ERR_UNSUPPORTED (-2) /* dtype / mode combination not provided */
#define MUON_ERR_CUDA (-3)        /* a CUDA runtime or driver call failed */
#define MUON_ERR_NO_MEMORY (-4)   /* workspace allocation failed */
#define MUON_ERR_TIMEOUT (-5)     /* a bounded device-side wait ran out */
#define MUON_ERR_NONFINITE (-6)   /* ||U||_F was not finite for some matrix */
#define MUON_ERR_GUARD     (-7)   /* debug canary mode: a workspace guard was overwritten */

/* mode bits of muon_orthogonalize and muon_config.mode */
#define MUON_NS_STANDARD 0  /* A = X X^T, B = bA + cA^2, X <- aX + BX          */
#define MUON_NS_GRAM 1      /* iterate on R = X X^T with restarts, O = Q X       */
#define MUON_NS_AUTO 2      /* per matrix: Gram iff its FLOP count is lower      */
#define MUON_NS_FORM_MASK 0xff
#define MUON_PREC_FP32 0x100 /* fp32 check path: X is fp32, all math fp32 SIMT */

/* element types */
#define MUON_DTYPE_BF16 0
#define MUON_DTYPE_F32 1

#define MUON_MAX_STEPS 16

typedef struct muon_config {
    int steps;                        /* NS steps T for muon_step, 0..MUON_MAX_STEPS (default 5) */
    float coeffs[3 * MUON_MAX_STEPS]; /* (a, b, c) of step k at [3k..3k+2] (default tuned set)  */
    int mode;                         /* NS form for muon_step (default MUON_NS_AUTO)           */
    unsigned restart_mask;            /* Gram form: bit k (k >= 1) restarts before step k;
                                         used by both entry points (default 1u << 2)            */
    float eps;                        /* added to the Frobenius norm (default 1e-7)             */
    int momentum_dtype;               /* MUON_DTYPE_BF16 (default) or MUON_DTYPE_F32            */
    int param_dtype;                  /* MUON_DTYPE_F32 (default) or MUON_DTYPE_BF16            */
    int grad_dtype;                   /* gradients of muon_step and muon_adamw_step:
                                         MUON_DTYPE_BF16 (default) or MUON_DTYPE_F32            */
    float soft_threshold;             /* muon_step only: lam of the soft-threshold split (ROOT
                                         page, "ROOT优化器的技术创新": min ||M - B - O||_F^2 +
                                         lam ||O||_1, only the robust part B is orthogonalised).
                                         The outliers O are the update soft-thresholded at
                                         lam / 2, so B is the update clipped elementwise to
                                         [-lam/2, lam/2]; the momentum buffer keeps the full
                                         momentum.  A non-finite update (+-Inf, NaN) still flags
                                         the matrix non-finite.  0 = off (default); finite, >= 0 */
} muon_config;

/* Library version (MUON_VERSION of the build). */
MUON_API int muon_version(void);

/* Fill *cfg with the defaults listed above.  Returns MUON_ERR_INVALID_ARG if cfg is NULL. */
MUON_API int muon_default_config(muon_config* cfg);

/* Validate and install *cfg for subsequent calls (copied). */
MUON_API int muon_set_config(const muon_config* cfg);

/* Copy the installed config into *cfg. */
MUON_API int muon_get_config(muon_config* cfg);

/* Bind the cudaStream_t (passed as void*) that all later work is enqueued on. NULL = default stream. */
MUON_API int muon_set_stream(void* stream);

/* Human-readable description of the last error of this thread ("" if none). */
MUON_API const char* muon_last_error(void);

/* Free the cached workspace and plans (waits for the bound stream first). */
MUON_API int muon_release_workspace(void);

/*
 * Synchronise the bound stream, then read and clear the device status word.
 * Returns MUON_OK, MUON_ERR_TIMEOUT (a kernel's bounded wait ran out; its
 * outputs are undefined) or MUON_ERR_NONFINITE (a matrix had a non-finite
 * Frobenius norm; that matrix's outputs were left untouched).  If bad_index
 * is not NULL it receives the index of the first non-finite matrix (or -1).
 */
MUON_API int muon_device_status(int* bad_index);

/*
 * muon_orthogonalize -- X <- NS_T(X / (||X||_F + eps)) for a batch of matrices.
 *   [Gram-NS] "ข้อได้เปรียบของอัลกอริทึม" (polar via NS, standard and Gram forms);
 *   [NanoGPT-Muon] "Newton-Schulz 迭代的系数调优" (coefficients, T = 5).
 * batch   number of matrices (>= 1), stored back to back in X
 * m, n    rows and columns of each matrix (>= 1); the iteration uses the
 *         shorter side (Gram matrix min(m,n) x min(m,n))
 * X       device pointer, in place; bf16 by default, fp32 with MUON_PREC_FP32.
 *         Any alignment: a 16-byte aligned X with n % 8 == 0 takes the
 *         vectorised loads and the TMA stores, any other X element-wise
 *         loads and plain stores
 * coeffs  host array of 3*steps floats, (a, b, c) of step k at [3k..3k+2]
 * steps   T in 0..MUON_MAX_STEPS; 0 returns the normalised X
 * mode    MUON_NS_STANDARD | MUON_NS_GRAM | MUON_NS_AUTO, optionally | MUON_PREC_FP32
 * eps and the Gram restart schedule come from the installed config.
 * A zero matrix returns zeros (also with eps = 0).
 */
MUON_API int muon_orthogonalize(int batch, int m, int n, void* X, const float* coeffs, int steps, int mode);

/*
 * muon_step -- one Muon step over count 2D parameters.
 *   [NanoGPT-Muon] "从 SGD 到 Muon", "工程复现清单"; [Gram-NS] "ข้อได้เปรียบของอัลกอริทึม":
 *     M <- mu*M + G;  U = G + mu*M (nesterov) or U = M;
 *     O = NS_T(U / (||U||_F + eps));  W <- W - lr*O.
 * params      host array of count device pointers, param_dtype, updated in place
 * grads       host array of count device pointers, grad_dtype (bf16 default), read only
 * momentum    host array of count device pointers, momentum_dtype, updated in place
 * shape_list  host int[2*count]: rows_i, cols_i of parameter i (>= 1)
 * With muon_config.soft_threshold = lam > 0, U is first clipped elementwise
 * to [-lam/2, lam/2] (its soft-thresholded outlier part is dropped; M keeps
 * it).  Coefficients and steps come from the shape's registered schedule
 * (muon_set_shape_coeffs) or else from the installed config; NS form,
 * restarts, eps, dtypes and the threshold from the installed config.  A
 * matrix whose U is zero (e.g. an expert that received no tokens) leaves its
 * parameter unchanged, also with eps = 0.  16-byte aligned pointers and
 * cols % 8 == 0 take the vectorised paths (otherwise element-wise ones).
 * Distinct parameters must not overlap.
 */
MUON_API int muon_step(void* const* params, const void* const* grads, void* const* momentum, float mu, int nesterov,
              float lr, const int* shape_list, int count);

/*
 * muon_adamw_step -- AdamW step of the parameters Muon does not handle
 * (embeddings, output head, 1-D parameters), the other lane of the hybrid
 * optimizer: [NanoGPT-Muon] "从 SGD 到 Muon" (AdamW for embedding and
 * classification head and for scalar/vector parameters) and "工程复现清单"
 * (lr 6e-4, betas (0.9, 0.95), weight decay 0.1).  Per element, in fp32:
 *     p <- p (1 - lr wd);  m <- beta1 m + (1 - beta1) g;  v <- beta2 v + (1 - beta2) g^2
 *     p <- p - lr (m / (1 - beta1^step)) / (sqrt(v / (1 - beta2^step)) + eps)
 * params      host array of count device pointers, installed param_dtype, updated in place
 * grads       host array of count device pointers, installed grad_dtype, read only
 * exp_avg     host array of count device pointers, fp32 first moments, updated in place
 * exp_avg_sq  host array of count device pointers, fp32 second moments, updated in place
 * numels      host array of count element counts (>= 1); tensors are treated as flat
 * step        the step being taken (>= 1) for the bias corrections
 * 0 <= beta1, beta2 < 1; lr, weight_decay, eps finite (eps >= 0).  One grouped
 * launch on the bound stream; 8-element vector access when every pointer of a
 * tensor is 16-byte aligned and its numel is a multiple of 8.
 */
MUON_API int muon_adamw_step(void* const* params, const void* const* grads, void* const* exp_avg,
                             void* const* exp_avg_sq, const long long* numels, int count, float lr, float beta1,
                             float beta2, float eps, float weight_decay, int step);

/*
 * muon_hybrid_step -- the whole hybrid optimizer step of a model: muon_step
 * over its 2-D hidden matrices and the AdamW step (as muon_adamw_step) over
 * the rest, with the AdamW lane's elements in the SAME grouped elementwise
 * launch as the Muon momentum pass (its chunks follow the Muon chunks in one
 * grid), followed by the Newton-Schulz launches.
 *   [NanoGPT-Muon] "从 SGD 到 Muon" (Muon for the 2-D hidden weights, AdamW
 *   for embeddings, the output head and 1-D parameters), "工程复现清单".
 * The Muon arguments are muon_step's; `adamw` describes the AdamW lane (host
 * struct, read during the call; its arrays as in muon_adamw_step).  Both lanes
 * use the installed config's param_dtype and grad_dtype.  Every argument of
 * both lanes is checked before anything is enqueued.  Results equal a
 * muon_step followed by a muon_adamw_step with the same arguments.
 */
typedef struct muon_adamw_lane {
    void* const* params;           /* count device pointers, updated in place      */
    const void* const* grads;      /* count device pointers, read only             */
    void* const* exp_avg;          /* count device pointers, fp32, updated         */
    void* const* exp_avg_sq;       /* count device pointers, fp32, updated         */
    const long long* numels;       /* count element counts (>= 1)                  */
    int count;                     /* >= 1                                          */
    float lr, beta1, beta2, eps, weight_decay;
    int step;                      /* >= 1, for the bias corrections               */
} muon_adamw_lane;

MUON_API int muon_hybrid_step(void* const* params, const void* const* grads, void* const* momentum, float mu,
                              int nesterov, float lr, const int* shape_list, int count,
                              const muon_adamw_lane* adamw);

/*
 * muon_step_offload -- muon_step for a training loop that keeps gradients
 * and/or the updated parameters in page-locked host memory, with the PCIe
 * copies overlapped with the step.  The count matrices are split into
 * min(chunks, count) groups of consecutive matrices with about equal copy
 * bytes (the grouping of muon_offload_chunks).  All groups' gradients are
 * copied in, in order, on a host-to-device copy stream; group k is stepped on
 * the bound stream once its gradients have landed, and its updated
 * parameters are copied out on a device-to-host copy stream as soon as its
 * step has finished.  While group k is stepped, group k + 1's gradients come in and
 * group k - 1's parameters go out, so both copy directions and the kernels
 * run at once.
 * params, grads, momentum, mu, nesterov, lr, shape_list, count: as muon_step
 *               (grads are the device buffers the gradients are copied into)
 * grads_host   host array of count page-locked host pointers (grad_dtype,
 *               rows x cols row-major each), copied into grads; NULL: the
 *               gradients are already in grads
 * params_host  host array of count page-locked host pointers (param_dtype)
 *               that receive the updated parameters; NULL: no copy out
 * chunks       >= 1 (1: copy in, step, copy out, with no overlap)
 * Each group is one muon_step with its own cached plan and workspace, so the
 * results equal muon_step's bit for bit.  Host pointers that are not
 * page-locked give MUON_ERR_INVALID_ARG (their copies could not overlap).
 * Every argument is checked before anything is enqueued.  The call ends by
 * making the bound stream wait for both copy streams: work enqueued on it
 * afterwards, or a synchronize of it, comes after every copy.  A non-finite
 * matrix is reported by muon_device_status in the caller's numbering.  If
 * group k fails to run, groups before it are stepped and copied, later ones
 * are not.  The copy streams and the per-group plans are the library's
 * (muon_release_workspace frees the plans).
 */
MUON_API int muon_step_offload(void* const* params, const void* const* grads_host, void* const* grads,
                               void* const* momentum, void* const* params_host, float mu, int nesterov, float lr,
                               const int* shape_list, int count, int chunks);

/*
 * muon_debug_corrupt_guard -- debug canary mode only: overwrite one byte of
 * workspace guard `index` of the current plan (a plain memset on the bound
 * stream, inside the library's own allocation), so that a test can see the
 * next call's check report MUON_ERR_GUARD.  MUON_ERR_INVALID_ARG when the
 * mode is off, no plan exists or the index is out of range.
 */
MUON_API int muon_debug_corrupt_guard(int index);

/*
 * muon_offload_chunks -- the grouping of muon_step_offload: with bytes[i] >= 0
 * the weight of matrix i, fills bounds (host int[g + 1]) with 0 = bounds[0] <
 * bounds[1] < ... < bounds[g] = count: g = min(chunks, count) groups of
 * consecutive matrices of about equal total weight.  Group k closes at the
 * first matrix that brings the running total to k/g of the whole, or earlier
 * when only one matrix remains for each later group; all-zero weights count
 * matrices.  Returns g, or MUON_ERR_INVALID_ARG.  Host only.
 */
MUON_API int muon_offload_chunks(const long long* bytes, int count, int chunks, int* bounds);

/* ---- per-shape coefficient schedules ----------------------------------------
 *
 * [ROOT] (staging.reportify.cn tag page, "ROOT优化器的技术创新"): the quintic
 * Newton-Schulz coefficients are adapted to each matrix size (m, n) instead of
 * one fixed set for all shapes ("现有优化器的核心局限": a fixed set leaves a
 * shape-dependent orthogonalisation error).  A schedule is one (a, b, c)
 * triple per step; matrices of different shapes in ONE muon_step each run
 * their own schedule inside the same grouped launches.
 *
 * muon_set_shape_coeffs -- register the schedule of muon_step for matrices of
 * rows x cols.  A matrix and its transpose share one entry (the key is the
 * short and the long side).  coeffs: host array of 3*steps floats, (a, b, c) of
 * step k at [3k..3k+2], copied; steps in 0..MUON_MAX_STEPS (0: the matrix is
 * only normalised).  Re-registering a shape replaces its schedule.  Matrices
 * whose shape has no entry use muon_config.coeffs / muon_config.steps.
 * MUON_ERR_INVALID_ARG for sizes < 1, steps out of range, NULL or non-finite
 * coeffs, or more than MUON_MAX_SHAPE_SCHEDULES shapes.  Host-only: enqueues
 * nothing.  muon_orthogonalize is unaffected (it takes its coefficients as an
 * argument).
 * muon_get_shape_coeffs -- *steps = the registered step count (-1 if the shape
 * has none) and, if coeffs is not NULL, the 3 * steps coefficients.
 * muon_clear_shape_coeffs -- remove every entry.
 */
#define MUON_MAX_SHAPE_SCHEDULES 64
MUON_API int muon_set_shape_coeffs(int rows, int cols, const float* coeffs, int steps);
MUON_API int muon_get_shape_coeffs(int rows, int cols, float* coeffs, int* steps);
MUON_API int muon_clear_shape_coeffs(void);

/* ---- allocation-free normalisation ---------------------------------------
 *
 * The pages have no counterpart to this call: it exists for callers that
 * cannot allocate device memory -- code whose device memory belongs to a
 * framework's allocator or to a fixed budget reserved up front, and
 * latency-critical paths where a cudaMalloc (which may synchronise the
 * device) is not acceptable.
 *
 * muon_normalize_noalloc -- Y_i = X_i / (||X_i||_F + eps) for batch matrices
 * of m x n, the same result as muon_orthogonalize with steps = 0.  It calls no
 * cudaMalloc, cudaFree or allocating library routine: its scratch (per-chunk
 * partial sums, per-matrix ticket counters and scales) is a file-scope device
 * array of fixed size, MUON_NOALLOC_MAX_CHUNKS * 4 + MUON_NOALLOC_MAX_MATRICES
 * * 8 bytes (about 264 KiB), which every GPU that loads the library holds
 * until the process exits.
 * batch, m, n  >= 1; batch <= MUON_NOALLOC_MAX_MATRICES and
 *              batch * ceil(m*n / 8192) <= MUON_NOALLOC_MAX_CHUNKS, else
 *              MUON_ERR_INVALID_ARG (nothing is enqueued)
 * X, Y         device pointers to batch contiguous row-major m x n matrices
 *              of `dtype` (MUON_DTYPE_BF16 or MUON_DTYPE_F32); Y may equal X
 * eps          finite, >= 0
 * Work is enqueued on the bound stream.  The first call on a device looks up
 * the array's device address on that device (once, with that device
 * current); make that first call before any stream capture.  Every call
 * shares the array and it keeps the last call's contents: each call clears
 * the counters it uses, and calls that overlap on the GPU (other streams,
 * other threads) race on it.  A matrix whose norm is not finite leaves its Y
 * untouched; a zero matrix gives a zero Y, also with eps = 0.  The device
 * addresses found at set-up are cached per device without a lock, like the
 * rest of the library's state (calls are not thread-safe).
 */
#define MUON_NOALLOC_MAX_MATRICES 1024
#define MUON_NOALLOC_MAX_CHUNKS 65536 /* chunks of 8192 elements: 512 Mi elements in one call */
MUON_API int muon_normalize_noalloc(int batch, int m, int n, const void* X, void* Y, int dtype, float eps);

/* ---- tracing ------------------------------------------------------------ */

typedef struct muon_kernel_stats {
    char name[32];    /* kernel kind: "momentum_norm", "gemm_tc", "gemm_f32", "scale_apply", "adamw" */
    long long launches;
    double total_ms;  /* sum of CUDA-event durations on the launching stream */
    double flops;     /* algorithmic FLOPs summed over launches (symmetric products at half cost) */
    double bytes;     /* algorithmic HBM bytes summed over launches */
} muon_kernel_stats;

/* When on, a CUDA event pair is recorded on the bound stream around every launch. */
MUON_API int muon_profile_enable(int on);

/* Synchronise, fold pending events, copy up to max entries; *count receives the number of kinds. */
MUON_API int muon_profile_read(muon_kernel_stats* out, int max, int* count);

/* Clear the accumulated statistics. */
MUON_API int muon_profile_reset(void);

/* Number of kernels this library has launched since load. */
MUON_API long long muon_launch_count(void);

#ifdef __cplusplus
}
#endif
#endif /* MUON_B200_H */
