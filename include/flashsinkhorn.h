/*
 * flashsinkhorn.h -- C ABI of the B200 (sm_100a) log-domain Sinkhorn library.
 *
 * The operation is the stabilised log-domain Sinkhorn iteration for entropic
 * optimal transport with squared-Euclidean cost, written in attention form
 * ("FlashSinkhorn: IO-aware EOT on GPU", Metodologia section 1, Proposition 1):
 *
 *   C_ij = |x_i|^2 + |y_j|^2 - 2 x_i.y_j
 *   f-update  f_i = |x_i|^2 - eps * LSE_j [ (2 x_i.y_j + g_j - |y_j|^2)/eps + log b_j ]
 *   g-update  g_j = |y_j|^2 - eps * LSE_i [ (2 x_i.y_j + f_i - |x_i|^2)/eps + log a_i ]
 *
 * i.e. a row (column) LogSumExp of the dot-product score matrix X Y^T shifted
 * by a per-column (per-row) bias.  The n x m cost or score matrix is never
 * stored anywhere (section 2 of the same page: streamed tiles, online LSE,
 * one fused pass per update).
 *
 * Conventions shared by every call
 *  - Pointers named "device" are CUDA device pointers on the device that was
 *    current at fs_create; "host" pointers are ordinary host memory.
 *  - Arrays are dense row-major: X [batch][n][d], Y [batch][m][d],
 *    a/f [batch][n], b/g [batch][m], float32 unless stated.
 *  - Every call is enqueued on the stream given to fs_create and returns
 *    without waiting, except the calls documented as synchronising
 *    (fs_create, fs_marginal_err, fs_ot_cost, fs_sync, fs_solve_host).
 *  - Errors are return codes; nothing aborts or exits.  fs_last_error gives
 *    a message.  After FS_ERR_CUDA the handle should be destroyed.
 *  - One handle per thread / stream.  The library never allocates anything
 *    of size n*m: handle memory is O(batch (n + m) d).
 */
#ifndef FLASHSINKHORN_H
#define FLASHSINKHORN_H

#include <stddef.h>

#if defined(__GNUC__)
#define FS_API __attribute__((visibility("default")))
#else
#define FS_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    FS_OK = 0,
    FS_ERR_INVALID_ARG = 1, /* bad sizes, eps, weights, null pointers           */
    FS_ERR_CUDA = 2,        /* a CUDA runtime call failed                        */
    FS_ERR_UNSUPPORTED = 3, /* device is not sm_100 (B200) or shape unsupported  */
    FS_ERR_NONFINITE = 4,   /* a non-finite input or result was detected         */
    FS_ERR_TIMEOUT = 5,     /* a bounded device-side wait ran out                */
    FS_ERR_OOM = 6          /* device allocation failed                          */
} fs_status;

typedef enum { FS_F32 = 0, FS_BF16 = 1 } fs_dtype; /* element type of X and Y */

/* Operand precision of the score product X Y^T (accumulation is always fp32).
 * The tensor-core modes need packed rows of at most 512 bytes: d <= 256 for
 * BF16, d <= 128 for TF32 and 3XF16, d <= 64 for 3XTF32 (FS_ERR_UNSUPPORTED
 * beyond). */
typedef enum {
    FS_PREC_AUTO = 0,     /* BF16 for bf16 inputs; 3XF16 for fp32 inputs with d <= 128,
                             else F32_SIMT (d <= 256)                                */
    FS_PREC_BF16 = 1,     /* one bf16 tensor-core pass (exact for bf16 inputs)        */
    FS_PREC_TF32 = 2,     /* one tf32 tensor-core pass                                */
    FS_PREC_3XTF32 = 3,   /* hi*hi + lo*hi + hi*lo tf32 passes (~fp32 accurate)       */
    FS_PREC_3XF16 = 4,    /* the same three passes on fp16 hi/lo planes, power-of-two
                             scaled per cloud (~fp32 accurate, half the MMAs)         */
    FS_PREC_F32_SIMT = 5  /* plain fp32 FMA on CUDA cores (validation path, d <= 256) */
} fs_precision;

typedef enum {
    FS_SCHED_ALTERNATING = 0, /* f from g, then g from the new f (Gauss-Seidel)   */
    FS_SCHED_SYMMETRIC = 1    /* f and g both from the previous pair (Jacobi)     */
} fs_schedule;

/*
 * Ground cost C_ij ("FlashSinkhorn: IO-aware EOT on GPU": the squared
 * Euclidean cost of Proposition 1, and the cosine distance after
 * normalisation that the closing remarks name as the other cost the method
 * covers).
 *   FS_COST_SQEUCLIDEAN  C_ij = |x_i - y_j|^2
 *   FS_COST_COSINE       C_ij = 1 - x_i.y_j / (|x_i| |y_j|); X and Y rows must
 *                        be non-zero (FS_ERR_INVALID_ARG otherwise).  Rows are
 *                        normalised in fp32 on the device; the default
 *                        precision is then 3xF16 for d <= 128 whatever the
 *                        input dtype (normalised bf16 rows are no longer bf16).
 */
typedef enum { FS_COST_SQEUCLIDEAN = 0, FS_COST_COSINE = 1 } fs_cost;

typedef struct {
    int batch;          /* independent problems sharing n, m, d, eps            */
    int n, m, d;        /* points in X, in Y, and their dimension               */
    fs_dtype dtype;     /* element type of X and Y                              */
    fs_precision prec;  /* score-product precision                              */
    float eps;          /* entropic regularisation, absolute units of C         */
    fs_cost cost;       /* ground cost (0 = squared Euclidean)                  */
} fs_desc;

typedef struct fs_handle fs_handle;

/* Resolved configuration of a handle (for logging and benchmarks). */
typedef struct {
    int prec;               /* resolved fs_precision                            */
    int d_pad;              /* padded feature dimension                         */
    int row_bytes;          /* bytes of one packed operand row                  */
    int swizzle_bytes;      /* shared-memory swizzle span of the operand tiles  */
    int stages;             /* column-tile pipeline depth                       */
    int block_rows, block_cols; /* rows per CTA (128, or 256 when two row blocks share
                                   every column tile; FS_ROW_BLOCKS=1 forces 128) x columns
                                   per streamed tile                               */
    int splits_f, splits_g; /* column splits of the f- and g-direction passes   */
    int launches_update;    /* kernel launches of one fs_update_f / fs_update_g */
    int launches_solve_iter;/* kernel launches per fs_solve iteration           */
    size_t device_bytes;    /* device memory owned by the handle                */
    int cta_pair;           /* 1: each MMA spans a pair of SMs (tcgen05 cta_group::2); chosen for
                               512-byte operand rows, or for every width when the environment
                               variable FS_CTA_PAIR=1 (FS_CTA_PAIR=0 forbids it) */
    int last_apply_path;    /* kernel of the handle's last transport application (fs_transport_apply
                               and the calls built on it): 4 tensor cores, one CTA per 256 rows (two
                               128-row blocks sharing every streamed tile; dv < 64, rows of up to
                               256 bytes, at least one such CTA per SM, or FS_ROW_BLOCKS=2 at any
                               size); 1 tensor cores, one CTA per 128 rows (dv over 128, or with
                               FS_ROW_BLOCKS=1); 3 tensor cores on CTA pairs
                               (512-byte operand rows, or any width with FS_APPLY_PAIR=1); 2 CUDA
                               cores (dv over 256, the f32_simt precision, or FS_APPLY_SIMT=1);
                               6 tensor cores, one CTA per 128 rows with both softmax groups on the
                               block, taking alternate tiles into their own TMEM columns (dv <= 128,
                               rows of up to 256 bytes, where mode 4 is not taken; FS_ROW_BLOCKS=3
                               at any size);
                               5 one column (dv = 1) through the streamed LSE pass with the column
                               vector as its weight (tensor-core handles; FS_APPLY_VEC=0 keeps the
                               kernels above); 0 none yet */
    int last_solve_graph;   /* how the handle's last fs_solve ran: 1 as a replay of its CUDA graph,
                               2 as direct launches (a large problem, FS_SOLVE_GRAPH=0, or a
                               failed capture), 0 none yet */
    int last_measure_fused; /* 1: the handle's last fs_marginal_err / fs_ot_cost reused the statistics
                               the last alternating fs_solve reduced in its final pass (f and g were
                               that solve's output, unchanged bit for bit); 0: it streamed its own
                               measure passes */
    int last_hvp_fused;     /* 1: the handle's last fs_hvp_x formed its transport-matrix term
                               sum_j P_ij (v_i.y_j) y_j in one tensor-core pass (bf16 operands, or the
                               3xF16 / 3xTF32 splits, rows up to 256 bytes); 0: as d / nq transport
                               applications of width nq d (other operands, FS_HVP_FUSED=0, or
                               FS_APPLY_SIMT=1) */
    int last_apply_parts;   /* column parts of the row blocks past the last full wave in the handle's
                               last transport application (path 6, batch 1: where those row blocks
                               fill at most half the SMs, each is split over its column tiles into
                               up to 8 parts of at least two tiles, and a merge kernel adds the
                               parts; FS_APPLY_TAIL=0 turns this off); 1: no row block split */
} fs_info;

/*
 * Source: "FlashSinkhorn: IO-aware EOT on GPU", Enunciato del Problema (the
 * problem's data: clouds X (n x d) and Y (m x d), weights a and b, eps) and
 * Metodologia section 1 (the squared norms and log-weight biases that
 * Proposition 1 precomputes, done here once per handle).
 * Create a solver for one (batched) problem: X and Y (device, dtype, row-major
 * [batch][n|m][d]), weights a (device [batch][n]) and b (device [batch][m]),
 * NULL meaning uniform 1/n (1/m).  Weights must be positive and sum to 1
 * within 1e-5 per problem.  X and Y are copied and packed into handle-owned
 * buffers (fp32 inputs are first shifted by a common per-problem centre,
 * which leaves every potential unchanged), so the caller may free them
 * afterwards.  Synchronises `stream` once to validate the inputs.
 * stream: a cudaStream_t (NULL = legacy default stream).
 * Errors: FS_ERR_INVALID_ARG (sizes < 1, eps <= 0 or non-finite, bad weights,
 * null X/Y/out), FS_ERR_NONFINITE (non-finite X or Y), FS_ERR_UNSUPPORTED
 * (device is not compute capability 10.x), FS_ERR_OOM, FS_ERR_CUDA.
 * On error *out is set to NULL and nothing is leaked.
 */
FS_API fs_status fs_create(const fs_desc *desc, const void *X, const void *Y, const float *a,
                    const float *b, void *stream, fs_handle **out);

/* Source: "FlashSinkhorn: IO-aware EOT on GPU", Metodologia section 1,
 * Proposition 1 (the f-update as a row LSE of the biased score matrix) and
 * section 2 (one fused streaming pass).
 * One f-update (device g [batch][m] -> device f [batch][n]).  Asynchronous.
 * f and g must not overlap.  Non-finite results are flagged for fs_sync. */
FS_API fs_status fs_update_f(fs_handle *h, const float *g, float *f);

/* Source: the same page and sections; the g-update is the transposed pass
 * (the column LSE, the page prints only the f-update and the roles of X and
 * Y are symmetric).
 * One g-update (device f [batch][n] -> device g [batch][m]).  Asynchronous. */
FS_API fs_status fs_update_g(fs_handle *h, const float *f, float *g);

/*
 * Source: "FlashSinkhorn: IO-aware EOT on GPU", Metodologia section 1 (the
 * alternating log-domain iterations; the algorithm itself is unchanged, only
 * its evaluation; "Significato e Affermazioni").  The page does not fix the schedule; the
 * alternating (Gauss-Seidel) order is the plain reading, the symmetric
 * (Jacobi) order is offered beside it.
 * `iters` Sinkhorn iterations in place (device f, g).  ALTERNATING: each
 * iteration is f <- update_f(g) then g <- update_g(f); the incoming f is not
 * read (the first half-step overwrites it), so only g is an initial value.
 * SYMMETRIC: (f, g) <- (update_f(g), update_g(f)) from the previous pair;
 * both are initial values.  iters = 0 is a no-op.  Asynchronous.
 * For small problems (batch * n * m up to 2^26, iters up to 1024), where launch
 * latency is a visible part of a pass, the loop is captured once as a CUDA graph on a
 * stream private to the handle and replayed there, ordered after the work
 * already on the handle's stream and before what follows it (events on both
 * streams).  The graph is kept for the next call with the same f, g, iters
 * and schedule.  FS_SOLVE_GRAPH=1 in the environment uses the graph at every
 * problem size (still up to 1024 iterations), FS_SOLVE_GRAPH=0 never.  Results
 * are identical either way.
 */
FS_API fs_status fs_solve(fs_handle *h, float *f, float *g, int iters, fs_schedule schedule);

/*
 * Source: not printed on the pages.  The convergence measure of the marginal
 * constraints that the entropic plan must meet (Enunciato del Problema: the
 * plan couples a and b); read as the L1 errors of the plan's row and column
 * sums at the given potentials.
 * Marginal errors of the plan P_ij = a_i b_j exp((f_i + g_j - C_ij)/eps) at
 * device potentials (f, g): err_row[k] = sum_i |r_i - a_i|, err_col[k] =
 * sum_j |c_j - b_j| for each problem k (host arrays [batch]; either may be
 * NULL).  Streams the score matrix once per requested direction.
 * Synchronises the stream.
 */
FS_API fs_status fs_marginal_err(fs_handle *h, const float *f, const float *g, double *err_row,
                          double *err_col);

/*
 * Source: not printed on the pages beyond "the EOT cost" (Enunciato del
 * Problema).  Read as the textbook entropic dual objective, with the
 * transport cost <P, C> of the plan beside it; they coincide at convergence.
 * Objectives at device potentials (f, g), host arrays [batch] (either may be
 * NULL):  dual[k]   = <a,f> + <b,g> - eps (sum_ij P_ij - 1)
 *         primal[k] = <P, C>  (transport cost of the plan)
 * Streams the score matrix once.  Synchronises the stream.
 */
FS_API fs_status fs_ot_cost(fs_handle *h, const float *f, const float *g, double *dual,
                     double *primal);

/* Source: no counterpart on the pages (error reporting of the bounded waits).
 * Wait for the handle's stream and report device-side flags raised since the
 * last check (FS_ERR_NONFINITE, FS_ERR_TIMEOUT). */
FS_API fs_status fs_sync(fs_handle *h);

/* Source: no counterpart on the pages.  Resolved configuration of the handle. */
FS_API fs_status fs_get_info(const fs_handle *h, fs_info *info);

/* Source: no counterpart on the pages (handle lifetime).
 * Free the handle.  Its device memory is released in stream order on the
 * handle's stream (no host wait), so the stream must still exist; work
 * already enqueued that uses the handle completes first.  NULL is accepted. */
FS_API fs_status fs_destroy(fs_handle *h);

/*
 * Transport application ("FlashSinkhorn: IO-aware EOT on GPU", Metodologia
 * section 3: the barycentric projection and the gradient as plan-weighted
 * averages, computed without forming the plan).  At device potentials (f, g),
 * with P_ij = a_i b_j exp((f_i + g_j - C_ij)/eps) of each problem k:
 *   out[k][i][c] = sum_j P_ij V[k][j][c]      (V: device fp32 [batch][m][dv])
 *   r[k][i]      = sum_j P_ij                 (device [batch][n]; may be NULL)
 * out: device fp32 [batch][n][dv].  Scores come from the handle's packed
 * operands (its precision); the exponent is formed in double and the sums in
 * fp32.  A single column (dv = 1) on a tensor-core handle runs as a streamed
 * LSE pass that weights each column by V_j (the plan-weighted average beside
 * the row's LSE state), at that pass's cost; it takes an fp32 scratch of the
 * column side's length from the device's memory pool for the call.
 * Asynchronous.  Errors: FS_ERR_INVALID_ARG (null pointer, dv < 1).
 */
FS_API fs_status fs_transport_apply(fs_handle *h, const float *f, const float *g, const float *V, int dv,
                                    float *out, float *r);

/* Barycentric map T(x_i) = sum_j P_ij y_j / sum_j P_ij: Y is the caller's
 * device [batch][m][d] cloud in the handle's dtype (the handle keeps only its
 * packed form); out: device fp32 [batch][n][d].  Asynchronous. */
FS_API fs_status fs_barycentric_map(fs_handle *h, const float *f, const float *g, const void *Y, float *out);

/* Gradient of the entropic OT cost with respect to the positions X at (f, g):
 * grad_i = sum_j P_ij dC_ij/dx_i (at optimal potentials, the gradient of the
 * optimal value).  Squared Euclidean cost: 2 (r_i x_i - sum_j P_ij y_j).
 * Cosine cost (dC/dx = -(y^ - (x^.y^) x^) / |x|, x^ = x / |x|):
 * -(b_i - (x^_i.b_i) x^_i) / |x_i| with b_i = sum_j P_ij y^_j, one transport
 * application of Y's unit rows (an fp32 copy of them is taken from the
 * device's memory pool for the call).  X, Y: the caller's device clouds in
 * the handle's dtype (the ones the handle was created from); grad: device
 * fp32 [batch][n][d].  Asynchronous. */
FS_API fs_status fs_grad_x(fs_handle *h, const float *f, const float *g, const void *X, const void *Y,
                           float *grad);

/* The transposed application: out[k][j][c] = sum_i P_ij U[k][i][c] (U: device
 * fp32 [batch][n][du]), c[k][j] = sum_i P_ij (device [batch][m]; may be NULL);
 * out: device fp32 [batch][m][du].  Same arithmetic as fs_transport_apply.
 * Asynchronous. */
FS_API fs_status fs_transport_apply_t(fs_handle *h, const float *f, const float *g, const float *U, int du,
                                      float *out, float *c);

/* Gradient of the entropic OT cost with respect to the positions Y at (f, g):
 * fs_grad_x with the clouds' roles exchanged (both costs are symmetric).
 * Squared Euclidean cost: 2 (c_j y_j - sum_i P_ij x_i); cosine cost:
 * -(b_j - (y^_j.b_j) y^_j) / |y_j| with b_j = sum_i P_ij x^_i.  With fs_grad_x
 * and the potentials themselves (the gradients with respect to the weights a
 * and b, up to the constant fixed by sum a = sum b = 1) this is the backward
 * pass of the EOT loss.  X, Y: the caller's device clouds in the handle's
 * dtype; grad: device fp32 [batch][m][d].  Asynchronous. */
FS_API fs_status fs_grad_y(fs_handle *h, const float *f, const float *g, const void *X, const void *Y,
                           float *grad);

/*
 * Hessian-vector product of the entropic OT cost with respect to the positions
 * X, at optimal device potentials (f, g), in the
 * direction V (device fp32 [batch][n][d]); out: device fp32 [batch][n][d].  Streaming
 * ("FlashSinkhorn: IO-aware EOT on GPU", Metodologia section 3): a sequence of
 * transport-vector and transport-matrix products, O((n + m) d) memory.  The
 * potentials' response solves
 *   [diag(c) - P^T diag(1/r) P] dg = w - P^T (u / r)
 * by conjugate gradients (each step one transport-vector product each way),
 * stopped after max_cg_iters steps or when the residual falls below
 * cg_rtol times its start.  Each problem of a batch runs its own CG (its own
 * scalars and stopping test; a problem that has converged takes no further
 * steps while the others continue); *cg_iters_done (may be NULL) receives the
 * most steps any problem took.  The cosine cost takes the same sequence on
 * Y's unit rows y^ and the direction's part orthogonal to each x_i, over |x_i|
 * (its change of C is -y^_j.v~_i), with the second derivative of the cosine
 * distance in the final combination; its transport-matrix term is always the
 * column-block form (fs_get_info's last_hvp_fused = 0).  X, Y: the caller's
 * device clouds in the handle's dtype.  The host reads the stopping test
 * back after every k steps (k = 1 for the first 16, then up to 8; the steps a
 * converged problem sits through leave its iterates unchanged), synchronising
 * the stream each time; blocks of 8 steps replay one CUDA graph captured on the
 * handle's graph stream.  Errors: FS_ERR_INVALID_ARG, FS_ERR_UNSUPPORTED
 * (batch > 65535).
 */
FS_API fs_status fs_hvp_x(fs_handle *h, const float *f, const float *g, const void *X, const void *Y,
                          const float *V, float *out, int max_cg_iters, double cg_rtol, int *cg_iters_done);

/* Source: no counterpart on the pages.
 * Failure-path self test: launches on the handle's stream a kernel whose one
 * bounded wait (the same wait every pass uses) can never complete, and waits
 * for it.  Returns FS_ERR_TIMEOUT after about timeout_ms; the handle and the
 * CUDA context stay usable.  FS_ERR_INVALID_ARG for timeout_ms < 1. */
FS_API fs_status fs_selftest_wait(fs_handle *h, int timeout_ms);

/* Source: no counterpart on the pages.
 * Number of CUDA kernels this library has launched in this process so far
 * (all handles, all threads).  Host-side counter; never synchronises. */
FS_API unsigned long long fs_kernel_launches(void);

/* Source: no counterpart on the pages.
 * Last error message of the handle; NULL handle -> the last error of any
 * call on this thread that had no handle to record it in. */
FS_API const char *fs_last_error(const fs_handle *h);

/*
 * Source: the calls above in sequence (fs_create, fs_solve, fs_marginal_err,
 * fs_ot_cost), with the host copies around them; no counterpart of its own.
 * One-call end-to-end solve from HOST arrays: copies X, Y (dtype), a, b
 * (NULL = uniform) and the initial g to the current device, creates a
 * handle, runs `iters` iterations, copies f and g back, and evaluates the
 * marginal errors and objectives (any of the four result arrays may be
 * NULL).  Host buffers may be pageable; pinned buffers make the copies
 * asynchronous.  g_host is read (initial g) and written (final g); f_host
 * is written.  Synchronises `stream`.  Errors as fs_create / fs_solve.
 */
FS_API fs_status fs_solve_host(const fs_desc *desc, const void *X_host, const void *Y_host,
                        const float *a_host, const float *b_host, float *f_host,
                        float *g_host, int iters, fs_schedule schedule, double *err_row,
                        double *err_col, double *dual, double *primal, void *stream);

/*
 * One f-update that allocates nothing.  No counterpart on the pages: it is an
 * interface for callers that cannot allocate device memory when they need an
 * update -- plug-ins whose host framework owns all device memory and forbids
 * allocations by third-party code, services that reserve a fixed memory
 * budget up front, and latency-critical loops where an allocation (and the
 * synchronisation it can imply) is not acceptable.  fs_create allocates and
 * synchronises, so the handle API cannot serve them.
 * Inputs: device X [n][d], Y [m][d] (fp32, row-major), b [m] (NULL = uniform
 * 1/m), g [m]; output: device f [n], with
 *   f_i = |x_i|^2 - eps LSE_j[(2 x_i.y_j + g_j - |y_j|^2)/eps + log b_j].
 * Computed in plain fp32 on CUDA cores on inputs shifted by the common centre
 * t = (mean X + mean Y)/2 (the cost is translation-invariant, and the shift
 * keeps the arithmetic accurate for clouds far from the origin); enqueued on
 * `stream` (a cudaStream_t, NULL = legacy default); returns without waiting.
 * Scratch (the centring sums, the squared norms and the column bias) is a
 * fixed 4 MiB device array inside the library, held by every GPU that loads
 * it until the process exits, so: d <= 256 and n_pad + m + m_pad <= 982784
 * (n_pad, m_pad = n, m rounded up to 128), else FS_ERR_INVALID_ARG.  All calls
 * on a device share the array and it keeps the last call's contents (each call
 * writes everything it reads), so calls that overlap on the GPU race -- order
 * them on one stream.  The first call on each device, with that device
 * current, looks up the array's device address and sets a kernel attribute.
 * The address is kept per device
 * for the life of the process; after cudaDeviceReset it is stale, so do not
 * call this entry point on a device that has been reset.  Errors: return
 * codes, message in fs_last_error(NULL).
 */
FS_API fs_status fs_update_f_noalloc(int n, int m, int d, float eps, const float *X, const float *Y,
                                     const float *b, const float *g, float *f, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* FLASHSINKHORN_H */
