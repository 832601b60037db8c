/*
 * CPU oracle for log-domain Sinkhorn with squared-Euclidean or cosine cost.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may link, load or
 * call this file; only the tests, the smoke check and the benchmark's CPU
 * baseline leg use it.  It shares no code, header or constant with the CUDA
 * library.
 *
 * Everything is plain double precision, written straight from the
 * definitions of "FlashSinkhorn: IO-aware EOT on GPU" (Metodologia, section 1,
 * the stabilised log-domain f-update):
 *
 *   C_ij = |x_i - y_j|^2                         (evaluated directly as a sum of
 *                                                 squared differences, never in
 *                                                 the dot-product form)
 *   or, for the cosine cost (the other cost whose structure the method covers,
 *   per the closing remarks of the same page, "cosine distance after
 *   normalisation"),
 *   C_ij = 1 - x_i.y_j / (|x_i| |y_j|)           (from the raw vectors, in
 *                                                 double; undefined for a zero
 *                                                 vector)
 *   f_i  = -eps * LSE_j [ (g_j - C_ij)/eps + log b_j ]          (f-update)
 *   g_j  = -eps * LSE_i [ (f_i - C_ij)/eps + log a_i ]          (g-update, the
 *                                                 transpose of the f-update)
 *   P_ij = a_i b_j exp((f_i + g_j - C_ij)/eps)   (the transport plan)
 *
 * LSE is taken in two passes (maximum, then the sum of shifted exponentials).
 * Rows are independent, so an OpenMP loop over rows is the only parallelism;
 * each row is reduced in index order, so results do not depend on the thread
 * count.  Nothing of size n*m is stored.
 */
#include <math.h>
#include <stdlib.h>
#include <string.h>
#include <omp.h>

#if defined(__GNUC__) && (defined(__x86_64__) || defined(__i386__))
#define SO_CLONES __attribute__((target_clones("avx512f", "avx2", "default")))
#else
#define SO_CLONES
#endif

/* |p - q|^2 over d coordinates, directly from the differences. */
static inline double sq_dist(const double *p, const double *q, int d)
{
    double s = 0.0;
#pragma omp simd reduction(+ : s)
    for (int k = 0; k < d; ++k) {
        double t = p[k] - q[k];
        s += t * t;
    }
    return s;
}

/* 1 - cos(p, q) over d coordinates, from the dot product and the two norms. */
static inline double cos_dist(const double *p, const double *q, int d)
{
    double pq = 0.0, pp = 0.0, qq = 0.0;
#pragma omp simd reduction(+ : pq, pp, qq)
    for (int k = 0; k < d; ++k) {
        pq += p[k] * q[k];
        pp += p[k] * p[k];
        qq += q[k] * q[k];
    }
    return 1.0 - pq / (sqrt(pp) * sqrt(qq));
}

/* The cost between two points: cost 0 = squared Euclidean, 1 = cosine. */
static inline double cost_ij(int cost, const double *p, const double *q, int d)
{
    return cost == 1 ? cos_dist(p, q, d) : sq_dist(p, q, d);
}

/*
 * One entry of a log-domain update seen from point p against the cloud pts:
 *   out = -eps * LSE_j [ (pot_j - |p - pts_j|^2)/eps + logw_j ]
 * buf holds cnt doubles of scratch.
 */
SO_CLONES
static double soft_c_transform(const double *p, const double *pts, long cnt, int d,
                               const double *logw, const double *pot, double eps,
                               double *buf, int cost)
{
    double mx = -INFINITY;
    for (long j = 0; j < cnt; ++j) {
        double v = (pot[j] - cost_ij(cost, p, pts + (size_t)j * d, d)) / eps + logw[j];
        buf[j] = v;
        if (v > mx)
            mx = v;
    }
    if (mx == -INFINITY)
        return INFINITY;
    double s = 0.0;
    for (long j = 0; j < cnt; ++j)
        s += exp(buf[j] - mx);
    return -eps * (mx + log(s));
}

/* out_i = -eps * LSE_j [ (pot_j - C(P_i, Q_j))/eps + logw_j ], i < np_. */
static int soft_transform_all(long np_, long nq, int d, const double *P, const double *Q,
                              const double *logw, const double *pot, double eps, double *out,
                              int cost)
{
    int fail = 0;
#pragma omp parallel
    {
        double *buf = (double *)malloc(sizeof(double) * (size_t)(nq > 0 ? nq : 1));
        if (!buf) {
#pragma omp atomic write
            fail = 1;
        } else {
#pragma omp for schedule(dynamic, 16)
            for (long i = 0; i < np_; ++i)
                out[i] = soft_c_transform(P + (size_t)i * d, Q, nq, d, logw, pot, eps, buf, cost);
            free(buf);
        }
    }
    return fail ? -1 : 0;
}

/* f-update: f_i = -eps LSE_j[(g_j - C_ij)/eps + log b_j]. */
int so_update_f(long n, long m, int d, const double *X, const double *Y, const double *logb,
                const double *g, double eps, double *f, int cost)
{
    return soft_transform_all(n, m, d, X, Y, logb, g, eps, f, cost);
}

/* g-update: g_j = -eps LSE_i[(f_i - C_ij)/eps + log a_i]  (C_ij = C_ji^T). */
int so_update_g(long n, long m, int d, const double *X, const double *Y, const double *loga,
                const double *f, double eps, double *g, int cost)
{
    return soft_transform_all(m, n, d, Y, X, loga, f, eps, g, cost);
}

/*
 * Alternating Sinkhorn: `iters` times { f <- update_f(g); g <- update_g(f) }.
 * g holds the initial column potential on entry (f on entry is not read, as
 * the first half-step overwrites it); both hold the final pair on exit.
 */
int so_solve(long n, long m, int d, const double *X, const double *Y, const double *loga,
             const double *logb, double eps, int iters, double *f, double *g, int cost)
{
    for (int t = 0; t < iters; ++t) {
        if (so_update_f(n, m, d, X, Y, logb, g, eps, f, cost))
            return -1;
        if (so_update_g(n, m, d, X, Y, loga, f, eps, g, cost))
            return -1;
    }
    return 0;
}

/*
 * Row sums of the plan, straight from its definition:
 *   out_i = sum_j exp(logwp_i + logwq_j + (potp_i + potq_j - C(P_i, Q_j))/eps)
 * With (P,Q)=(X,Y) this is the row marginal r_i; with (Y,X) the column
 * marginal c_j.
 */
SO_CLONES
static double plan_row_sum(const double *p, const double *Q, long nq, int d, double logwp_i,
                           const double *logwq, double potp_i, const double *potq, double eps,
                           int cost)
{
    double s = 0.0;
    for (long j = 0; j < nq; ++j) {
        double c = cost_ij(cost, p, Q + (size_t)j * d, d);
        s += exp(logwp_i + logwq[j] + (potp_i + potq[j] - c) / eps);
    }
    return s;
}

static void plan_sums(long np_, long nq, int d, const double *P, const double *Q,
                      const double *logwp, const double *logwq, const double *potp,
                      const double *potq, double eps, double *out, int cost)
{
#pragma omp parallel for schedule(dynamic, 16)
    for (long i = 0; i < np_; ++i)
        out[i] = plan_row_sum(P + (size_t)i * d, Q, nq, d, logwp[i], logwq, potp[i], potq, eps, cost);
}

/* r_i = sum_j P_ij and c_j = sum_i P_ij. */
void so_marginals(long n, long m, int d, const double *X, const double *Y, const double *loga,
                  const double *logb, const double *f, const double *g, double eps, double *r,
                  double *c, int cost)
{
    if (r)
        plan_sums(n, m, d, X, Y, loga, logb, f, g, eps, r, cost);
    if (c)
        plan_sums(m, n, d, Y, X, logb, loga, g, f, eps, c, cost);
}

/*
 * Per-row plan statistics (summed in row order afterwards, so deterministic):
 *   out[0] = sum_ij P_ij
 *   out[1] = sum_ij P_ij C_ij                          (primal transport cost <P,C>)
 *   out[2] = sum_ij P_ij log(P_ij / (a_i b_j))         (= sum P (f_i+g_j-C_ij)/eps)
 *   out[3] = max_ij C_ij
 *   out[4] = min_ij C_ij
 */
SO_CLONES
static void plan_row_stats(const double *p, const double *Q, long nq, int d, double loga_i,
                           const double *logb, double f_i, const double *g, double eps,
                           double *acc, int cost)
{
    double sp = 0.0, spc = 0.0, spl = 0.0, cmax = -INFINITY, cmin = INFINITY;
    for (long j = 0; j < nq; ++j) {
        double c = cost_ij(cost, p, Q + (size_t)j * d, d);
        double lr = (f_i + g[j] - c) / eps;
        double pij = exp(loga_i + logb[j] + lr);
        sp += pij;
        spc += pij * c;
        spl += pij * lr;
        if (c > cmax)
            cmax = c;
        if (c < cmin)
            cmin = c;
    }
    acc[0] = sp;
    acc[1] = spc;
    acc[2] = spl;
    acc[3] = cmax;
    acc[4] = cmin;
}

int so_plan_stats(long n, long m, int d, const double *X, const double *Y, const double *loga,
                  const double *logb, const double *f, const double *g, double eps,
                  double *out, int cost)
{
    double *rows = (double *)malloc(sizeof(double) * 5 * (size_t)(n > 0 ? n : 1));
    if (!rows)
        return -1;
#pragma omp parallel for schedule(dynamic, 16)
    for (long i = 0; i < n; ++i)
        plan_row_stats(X + (size_t)i * d, Y, m, d, loga[i], logb, f[i], g, eps, rows + 5 * i, cost);
    double sp = 0.0, spc = 0.0, spl = 0.0, cmax = -INFINITY, cmin = INFINITY;
    for (long i = 0; i < n; ++i) {
        sp += rows[5 * i + 0];
        spc += rows[5 * i + 1];
        spl += rows[5 * i + 2];
        if (rows[5 * i + 3] > cmax)
            cmax = rows[5 * i + 3];
        if (rows[5 * i + 4] < cmin)
            cmin = rows[5 * i + 4];
    }
    free(rows);
    out[0] = sp;
    out[1] = spc;
    out[2] = spl;
    out[3] = cmax;
    out[4] = cmin;
    return 0;
}

/* Exact max_ij C_ij and, per row, min_j (C_ij - pot_j) and min_j (C_ij - pot_j - eps log w_j)
 * (the two sides of the c-transform sandwich for the f-update). */
SO_CLONES
static void row_minplus(const double *p, const double *Q, long nq, int d, const double *logw,
                        const double *pot, double eps, double *lo, double *hi, double *cmax, int cost)
{
    double l = INFINITY, h = INFINITY, cm = -INFINITY;
    for (long j = 0; j < nq; ++j) {
        double c = cost_ij(cost, p, Q + (size_t)j * d, d);
        double v = c - pot[j];
        if (v < l)
            l = v;
        double w = v - eps * logw[j];
        if (w < h)
            h = w;
        if (c > cm)
            cm = c;
    }
    *lo = l;
    *hi = h;
    *cmax = cm;
}

void so_minplus_bounds(long np_, long nq, int d, const double *P, const double *Q,
                       const double *logw, const double *pot, double eps, double *lo,
                       double *hi, double *cmax_row, int cost)
{
#pragma omp parallel for schedule(dynamic, 16)
    for (long i = 0; i < np_; ++i)
        row_minplus(P + (size_t)i * d, Q, nq, d, logw, pot, eps, lo + i, hi + i, cmax_row + i, cost);
}

/* Selected rows of the f-update (sampled parity at sizes where a full pass is too slow). */
int so_update_f_rows(long nrows, const long *rows, long m, int d, const double *X,
                     const double *Y, const double *logb, const double *g, double eps,
                     double *f_rows, int cost)
{
    int fail = 0;
#pragma omp parallel
    {
        double *buf = (double *)malloc(sizeof(double) * (size_t)(m > 0 ? m : 1));
        if (!buf) {
#pragma omp atomic write
            fail = 1;
        } else {
#pragma omp for schedule(dynamic, 1)
            for (long k = 0; k < nrows; ++k)
                f_rows[k] =
                    soft_c_transform(X + (size_t)rows[k] * d, Y, m, d, logb, g, eps, buf, cost);
            free(buf);
        }
    }
    return fail ? -1 : 0;
}

/*
 * Transport application ("FlashSinkhorn: IO-aware EOT on GPU", Metodologia
 * section 3: barycentric projection and gradient as weighted averages under
 * the plan), straight from the plan's definition:
 *   out_i = sum_j P_ij V_j   (V: [m][dv]),   r_i = sum_j P_ij,
 *   P_ij  = a_i b_j exp((f_i + g_j - C_ij)/eps).
 * Each row is summed in column order.
 */
int so_transport_apply(long n, long m, int d, const double *X, const double *Y, const double *loga,
                       const double *logb, const double *f, const double *g, double eps, int dv,
                       const double *V, double *out, double *r, int cost)
{
#pragma omp parallel for schedule(dynamic, 16)
    for (long i = 0; i < n; ++i) {
        double *o = out + (size_t)i * dv;
        for (int c = 0; c < dv; ++c)
            o[c] = 0.0;
        double s = 0.0;
        for (long j = 0; j < m; ++j) {
            double cij = cost_ij(cost, X + (size_t)i * d, Y + (size_t)j * d, d);
            double p = exp(loga[i] + logb[j] + (f[i] + g[j] - cij) / eps);
            s += p;
            const double *v = V + (size_t)j * dv;
            for (int c = 0; c < dv; ++c)
                o[c] += p * v[c];
        }
        r[i] = s;
    }
    return 0;
}

int so_num_threads(void)
{
    int t = 1;
#pragma omp parallel
    {
#pragma omp single
        t = omp_get_num_threads();
    }
    return t;
}
