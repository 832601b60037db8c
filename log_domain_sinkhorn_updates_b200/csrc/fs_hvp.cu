// Element-wise and reduction kernels of the streaming Hessian-vector product
// of the entropic OT cost with respect to X (squared Euclidean cost;
// "FlashSinkhorn: IO-aware EOT on GPU", Metodologia section 3: the HVP as a
// sequence of transport-vector and transport-matrix products).  The transport
// products themselves are the transport-application kernels; these kernels
// combine their outputs, all O((n + m) d).
//
// With P at optimal potentials, r = P 1, c = P^T 1, a direction V [n][d] and
// dC_ij = 2 (x_i - y_j).v_i:
//   u_i = sum_j P_ij dC_ij = 2 (r_i x_i - (P Y)_i).v_i
//   w_j = sum_i P_ij dC_ij = 2 ((P^T (x.v))_j - y_j.(P^T V)_j)
//   [diag(c) - P^T diag(1/r) P] dg = w - P^T (u / r),   df = (u - P dg) / r
//   (H V)_i = 2 r_i v_i + (2/eps) [ df_i (r_i x_i - (P Y)_i) + (P dg)_i x_i - (P (dg o Y))_i
//             - 2 ( (x_i.v_i)(r_i x_i - (P Y)_i) - x_i ((P Y)_i.v_i) + sum_j P_ij (y_j.v_i) y_j ) ]
//
// A batch of independent problems is laid out problem after problem ([batch][n]
// and [batch][n][d]), so the row-wise kernels run over batch x n rows as they
// are; the reductions and the conjugate-gradient updates take one problem per
// blockIdx.y, each with its own scalars.
#include <cuda_bf16.h>

#include "fs_internal.cuh"

namespace fs {
namespace {

template <typename T>
__device__ __forceinline__ float ldv(const T *p, size_t i);
template <>
__device__ __forceinline__ float ldv<float>(const float *p, size_t i) {
    return p[i];
}
template <>
__device__ __forceinline__ float ldv<__nv_bfloat16>(const __nv_bfloat16 *p, size_t i) {
    return __bfloat162float(p[i]);
}

__host__ __device__ inline int blocks_for(size_t n) {
    const size_t b = (n + 255) / 256;
    return (int)(b < 4096 ? (b > 0 ? b : 1) : 4096);
}

#define GRID_LOOP(i, n) for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < (n); i += (size_t)gridDim.x * blockDim.x)

// u_i = 2 (r_i x_i - PY_i).v_i;  W1_i = [v_i | x_i.v_i | u_i / r_i]  ([n][d+2])
template <typename T>
__global__ void prep_kernel(const T *X, const float *V, const float *PY, const float *r, int n, int d, float *u,
                            float *W1) {
    GRID_LOOP(i, (size_t)n) {
        float su = 0.f, sxv = 0.f;
        for (int k = 0; k < d; ++k) {
            const float x = ldv(X, i * d + k), v = V[i * d + k];
            su = fmaf(r[i] * x - PY[i * d + k], v, su);
            sxv = fmaf(x, v, sxv);
            W1[i * (d + 2) + k] = v;
        }
        u[i] = 2.f * su;
        W1[i * (d + 2) + d] = sxv;
        W1[i * (d + 2) + d + 1] = u[i] / r[i];
    }
}

// z_j = alpha (T_j[d] - y_j . T_j[0:d]) - T_j[d+1],  T = P^T W1  ([m][d+2]): the right-hand
// side w - P^T (u / r) of the potentials' response.  alpha = 2 for the squared Euclidean
// cost (W1 = [v | x.v | u/r]), 1 for the cosine cost (W1 = [v~ | 0 | u/r], Y = Y^)
template <typename T>
__global__ void w_kernel(const T *Y, const float *Tm, int m, int d, float alpha, float *z) {
    GRID_LOOP(j, (size_t)m) {
        float s = 0.f;
        for (int k = 0; k < d; ++k) s = fmaf(ldv(Y, j * d + k), Tm[j * (d + 2) + k], s);
        z[j] = alpha * (Tm[j * (d + 2) + d] - s) - Tm[j * (d + 2) + d + 1];
    }
}

// out = alpha * x o a + beta * y  (a or y may be null: treated as 1 / 0); or out = x / a when div
__global__ void vec_kernel(size_t n, const float *x, const float *a, float alpha, const float *y, float beta,
                           bool div, float *out) {
    GRID_LOOP(i, n) {
        const float av = a ? a[i] : 1.f;
        const float t = div ? x[i] / av : alpha * x[i] * av;
        out[i] = t + (y ? beta * y[i] : 0.f);
    }
}

// Problem b = blockIdx.y owns the segment [b len, (b + 1) len) of every vector.
#define SEG_LOOP(i, len) for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < (len); i += (size_t)gridDim.x * blockDim.x)

// Deterministic per-problem dot products: fixed-order block trees over each
// problem's segment (part[b][blockIdx.x]), then one block per problem over its partials.
__global__ void dot_partial_kernel(size_t len, const float *x, const float *y, double *part) {
    __shared__ double sh[256];
    const size_t base = (size_t)blockIdx.y * len;
    double s = 0.0;
    SEG_LOOP(i, len) s += (double)x[base + i] * (double)(y ? y[base + i] : 1.f);
    sh[threadIdx.x] = s;
    __syncthreads();
    for (int k = 128; k > 0; k >>= 1) {
        if ((int)threadIdx.x < k) sh[threadIdx.x] += sh[threadIdx.x + k];
        __syncthreads();
    }
    if (threadIdx.x == 0) part[(size_t)blockIdx.y * gridDim.x + blockIdx.x] = sh[0];
}
__global__ void dot_final_kernel(int nb, const double *part, double *out) {
    __shared__ double sh[256];
    const double *pb = part + (size_t)blockIdx.x * nb;
    double s = 0.0;
    for (int i = threadIdx.x; i < nb; i += 256) s += pb[i];
    sh[threadIdx.x] = s;
    __syncthreads();
    for (int k = 128; k > 0; k >>= 1) {
        if ((int)threadIdx.x < k) sh[threadIdx.x] += sh[threadIdx.x + k];
        __syncthreads();
    }
    if (threadIdx.x == 0) out[blockIdx.x] = sh[0];
}

// x_b -= s_b / len (s: device doubles, one per problem), keeping each problem's
// CG iterates orthogonal to the constant vector
__global__ void center_vec_kernel(size_t len, const double *s, float *x) {
    const size_t base = (size_t)blockIdx.y * len;
    const float mean = (float)(s[blockIdx.y] / (double)len);
    SEG_LOOP(i, len) x[base + i] -= mean;
}

// A problem's CG is still running while rr > tol2 zz (zz = z.z, the right-hand
// side's square norm); the host's loop test is the same comparison.
__device__ __forceinline__ bool cg_active(const double *rr, const double *zz, double tol2, int b) {
    return rr[b] > tol2 * zz[b] && zz[b] > 0.0;
}

// CG update on the device, from device scalars rr (r.r) and pap (p.Ap):
//   alpha = rr / pap;  x += alpha p;  res -= alpha Ap   (problems still running,
// each of which counts the step in steps[b])
__global__ void cg_step_kernel(size_t len, const double *rr, const double *pap, const double *zz, double tol2,
                               const float *p, const float *Ap, float *x, float *res, int *steps) {
    const int b = blockIdx.y;
    if (!cg_active(rr, zz, tol2, b)) return;
    if (blockIdx.x == 0 && threadIdx.x == 0) steps[b] += 1;
    const size_t base = (size_t)b * len;
    const float alpha = (float)(rr[b] / pap[b]);
    SEG_LOOP(i, len) {
        x[base + i] = fmaf(alpha, p[base + i], x[base + i]);
        res[base + i] = fmaf(-alpha, Ap[base + i], res[base + i]);
    }
}
// p = res + (rr_new / rr) p   (problems still running, judged on rr before the step)
__global__ void cg_dir_kernel(size_t len, const double *rr_new, const double *rr, const double *zz, double tol2,
                              const float *res, float *p) {
    const int b = blockIdx.y;
    if (!cg_active(rr, zz, tol2, b)) return;
    const size_t base = (size_t)b * len;
    const float beta = (float)(rr_new[b] / rr[b]);
    SEG_LOOP(i, len) p[base + i] = fmaf(beta, p[base + i], res[base + i]);
}

// out_j = [dg_j y_j | dg_j]  ([m][d+1]): one application gives P (dg o Y) and P dg
template <typename T>
__global__ void dgy_kernel(const T *Y, const float *dg, int m, int d, float *out) {
    GRID_LOOP(i, (size_t)m * (d + 1)) {
        const size_t j = i / (d + 1);
        const int k = (int)(i % (d + 1));
        out[i] = k < d ? dg[j] * ldv(Y, j * d + k) : dg[j];
    }
}

// df_i = (u_i - (P dg)_i) / r_i, (P dg)_i the last column of Q = P [dg o Y | dg] ([n][d+1])
__global__ void df_kernel(size_t n, int d, const float *u, const float *Q, const float *r, float *df) {
    GRID_LOOP(i, n) df[i] = (u[i] - Q[i * (d + 1) + d]) / r[i];
}

// Vc_j[q d + k] = y_j[k0 + q] y_jk for q < nq  ([m][nq d])
template <typename T>
__global__ void ychunk_kernel(const T *Y, int m, int d, int k0, int nq, float *Vc) {
    GRID_LOOP(i, (size_t)m * nq * d) {
        const size_t j = i / ((size_t)nq * d);
        const int q = (int)((i / d) % nq), k = (int)(i % d);
        Vc[i] = ldv(Y, j * d + k0 + q) * ldv(Y, j * d + k);
    }
}

// MV_ik += sum_q v_i[k0 + q] Oc_i[q d + k]
__global__ void mv_acc_kernel(const float *V, const float *Oc, int n, int d, int k0, int nq, float *MV) {
    GRID_LOOP(i, (size_t)n * d) {
        const size_t row = i / d;
        const int k = (int)(i % d);
        float s = MV[i];
        for (int q = 0; q < nq; ++q) s = fmaf(V[row * d + k0 + q], Oc[(row * nq + q) * d + k], s);
        MV[i] = s;
    }
}

// Q1: P [dg o Y | dg] ([n][d+1]; column d is P dg)
template <typename T>
__global__ void final_kernel(const T *X, const float *V, const float *PY, const float *r, const float *df,
                             const float *Q1, const float *MV, int n, int d, float eps, float *out) {
    GRID_LOOP(i, (size_t)n) {
        const float pdg = Q1[i * (d + 1) + d];
        float xv = 0.f, pyv = 0.f;
        for (int k = 0; k < d; ++k) {
            const float v = V[i * d + k];
            xv = fmaf(ldv(X, i * d + k), v, xv);
            pyv = fmaf(PY[i * d + k], v, pyv);
        }
        for (int k = 0; k < d; ++k) {
            const float x = ldv(X, i * d + k);
            const float gk = r[i] * x - PY[i * d + k];  // sum_j P_ij (x_i - y_j), component k
            const float inner = df[i] * gk + pdg * x - Q1[i * (d + 1) + k] -
                                2.f * (xv * gk - x * pyv + MV[i * d + k]);
            out[i * d + k] = 2.f * r[i] * V[i * d + k] + (2.f / eps) * inner;
        }
    }
}

}  // namespace

cudaError_t hvp_prep(const void *X, bool bf16, const float *V, const float *PY, const float *r, int n, int d,
                     float *u, float *W1, cudaStream_t s) {
    if (bf16)
        prep_kernel<<<blocks_for(n), 256, 0, s>>>(static_cast<const __nv_bfloat16 *>(X), V, PY, r, n, d, u, W1);
    else
        prep_kernel<<<blocks_for(n), 256, 0, s>>>(static_cast<const float *>(X), V, PY, r, n, d, u, W1);
    return cudaGetLastError();
}
cudaError_t hvp_w(const void *Y, bool bf16, const float *Tm, int m, int d, float alpha, float *z, cudaStream_t s) {
    if (bf16)
        w_kernel<<<blocks_for(m), 256, 0, s>>>(static_cast<const __nv_bfloat16 *>(Y), Tm, m, d, alpha, z);
    else
        w_kernel<<<blocks_for(m), 256, 0, s>>>(static_cast<const float *>(Y), Tm, m, d, alpha, z);
    return cudaGetLastError();
}
cudaError_t hvp_vec(size_t n, const float *x, const float *a, float alpha, const float *y, float beta, bool div,
                    float *out, cudaStream_t s) {
    vec_kernel<<<blocks_for(n), 256, 0, s>>>(n, x, a, alpha, y, beta, div, out);
    return cudaGetLastError();
}
// out[b] = x_b.y_b (y null: sum of x_b) for the batch problems' segments of
// length len; part holds at least batch x 4096 doubles.
cudaError_t hvp_dot(int batch, size_t len, const float *x, const float *y, double *part, double *out,
                    cudaStream_t s) {
    const int nb = blocks_for(len);
    dot_partial_kernel<<<dim3(nb, batch), 256, 0, s>>>(len, x, y, part);
    dot_final_kernel<<<batch, 256, 0, s>>>(nb, part, out);
    count_launches(1);  // the caller's launch macro counts the first
    return cudaGetLastError();
}
cudaError_t hvp_center(int batch, size_t len, const double *sum, float *x, cudaStream_t s) {
    center_vec_kernel<<<dim3(blocks_for(len), batch), 256, 0, s>>>(len, sum, x);
    return cudaGetLastError();
}
cudaError_t hvp_cg_step(int batch, size_t len, const double *rr, const double *pap, const double *zz, double tol2,
                        const float *p, const float *Ap, float *x, float *res, int *steps, cudaStream_t s) {
    cg_step_kernel<<<dim3(blocks_for(len), batch), 256, 0, s>>>(len, rr, pap, zz, tol2, p, Ap, x, res, steps);
    return cudaGetLastError();
}
cudaError_t hvp_cg_dir(int batch, size_t len, const double *rr_new, const double *rr, const double *zz, double tol2,
                       const float *res, float *p, cudaStream_t s) {
    cg_dir_kernel<<<dim3(blocks_for(len), batch), 256, 0, s>>>(len, rr_new, rr, zz, tol2, res, p);
    return cudaGetLastError();
}
cudaError_t hvp_dgy(const void *Y, bool bf16, const float *dg, int m, int d, float *out, cudaStream_t s) {
    if (bf16)
        dgy_kernel<<<blocks_for((size_t)m * (d + 1)), 256, 0, s>>>(static_cast<const __nv_bfloat16 *>(Y), dg, m, d,
                                                                   out);
    else
        dgy_kernel<<<blocks_for((size_t)m * (d + 1)), 256, 0, s>>>(static_cast<const float *>(Y), dg, m, d, out);
    return cudaGetLastError();
}
cudaError_t hvp_df(size_t n, int d, const float *u, const float *Q, const float *r, float *df, cudaStream_t s) {
    df_kernel<<<blocks_for(n), 256, 0, s>>>(n, d, u, Q, r, df);
    return cudaGetLastError();
}
cudaError_t hvp_ychunk(const void *Y, bool bf16, int m, int d, int k0, int nq, float *Vc, cudaStream_t s) {
    if (bf16)
        ychunk_kernel<<<blocks_for((size_t)m * nq * d), 256, 0, s>>>(static_cast<const __nv_bfloat16 *>(Y), m, d, k0,
                                                                     nq, Vc);
    else
        ychunk_kernel<<<blocks_for((size_t)m * nq * d), 256, 0, s>>>(static_cast<const float *>(Y), m, d, k0, nq, Vc);
    return cudaGetLastError();
}
cudaError_t hvp_mv_acc(const float *V, const float *Oc, int n, int d, int k0, int nq, float *MV, cudaStream_t s) {
    mv_acc_kernel<<<blocks_for((size_t)n * d), 256, 0, s>>>(V, Oc, n, d, k0, nq, MV);
    return cudaGetLastError();
}
cudaError_t hvp_final(const void *X, bool bf16, const float *V, const float *PY, const float *r, const float *df,
                      const float *Q1, const float *MV, int n, int d, float eps, float *out, cudaStream_t s) {
    if (bf16)
        final_kernel<<<blocks_for(n), 256, 0, s>>>(static_cast<const __nv_bfloat16 *>(X), V, PY, r, df, Q1, MV, n, d,
                                                   eps, out);
    else
        final_kernel<<<blocks_for(n), 256, 0, s>>>(static_cast<const float *>(X), V, PY, r, df, Q1, MV, n, d, eps,
                                                   out);
    return cudaGetLastError();
}

}  // namespace fs
