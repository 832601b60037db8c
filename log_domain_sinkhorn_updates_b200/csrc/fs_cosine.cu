// Derivatives of the cosine cost C(x, y) = 1 - x.y / (|x| |y|) with respect to
// the positions, for the gradient and the streaming Hessian-vector product of
// the entropic OT cost ("FlashSinkhorn: IO-aware EOT on GPU": Metodologia
// section 3 for the gradient and the HVP as transport products, and the
// closing remarks for the cosine distance after normalisation).
//
// With x^ = x / |x|, y^ = y / |y|, s = x^.y^ and rho = |x|:
//   dC/dx            = -(y^ - s x^) / rho                        (linear in y^)
//   (d^2 C/dx^2) v   = [ (y^.v) x^ + s v + (x^.v) y^ - 3 s (x^.v) x^ ] / rho^2
// Both are linear in y^, so every plan-weighted sum over j needs only
// b_i = sum_j P_ij y^_j (a transport application of the unit rows Y^):
//   grad_i = -(b_i - (x^_i.b_i) x^_i) / rho_i.
// The HVP's first-order change of C along v_i is dC_ij = -y^_j.v~_i with
// v~_i = (v_i - (x^_i.v_i) x^_i) / rho_i, so the potentials' response and the
// transport-matrix term are those of the squared Euclidean path with Y^ in
// place of Y and v~ in place of v; only the first and last steps differ (here).
// All kernels are row-wise, O((n + m) d); one thread per point.
#include <cuda_bf16.h>

#include "fs_internal.cuh"

namespace fs {
namespace {

template <typename T>
__device__ __forceinline__ float ldc(const T *p, size_t i);
template <>
__device__ __forceinline__ float ldc<float>(const float *p, size_t i) {
    return p[i];
}
template <>
__device__ __forceinline__ float ldc<__nv_bfloat16>(const __nv_bfloat16 *p, size_t i) {
    return __bfloat162float(p[i]);
}

inline int grid_rows(size_t rows) {
    const size_t b = (rows + 255) / 256;
    return (int)(b < 4096 ? (b > 0 ? b : 1) : 4096);
}

#define ROW_LOOP(i, n) for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < (n); i += (size_t)gridDim.x * blockDim.x)

// |p_i| in fp32, from a double sum of squares of the row's fp32 or bf16 values
template <typename T>
__device__ __forceinline__ float row_norm(const T *P, size_t i, int d) {
    double s = 0.0;
    for (int k = 0; k < d; ++k) {
        const double v = ldc(P, i * d + k);
        s += v * v;
    }
    return (float)sqrt(s);
}

// out_i = p_i / |p_i|  (fp32)
template <typename T>
__global__ void unit_rows_kernel(const T *P, size_t rows, int d, float *out) {
    ROW_LOOP(i, rows) {
        const float inv = 1.f / row_norm(P, i, d);
        for (int k = 0; k < d; ++k) out[i * d + k] = ldc(P, i * d + k) * inv;
    }
}

// grad_i = -(b_i - (x^_i.b_i) x^_i) / rho_i, in place over b (grad may alias b)
template <typename T>
__global__ void grad_kernel(const T *X, const float *b, size_t rows, int d, float *grad) {
    ROW_LOOP(i, rows) {
        const float rho = row_norm(X, i, d), inv = 1.f / rho;
        float s = 0.f;
        for (int k = 0; k < d; ++k) s = fmaf(ldc(X, i * d + k) * inv, b[i * d + k], s);
        for (int k = 0; k < d; ++k) {
            const float xh = ldc(X, i * d + k) * inv;
            grad[i * d + k] = -(b[i * d + k] - s * xh) * inv;
        }
    }
}

// v~_i = (v_i - (x^_i.v_i) x^_i) / rho_i  -> Vt [n][d] and W1 = [v~_i | 0 | u_i / r_i] [n][d+2];
// u_i = sum_j P_ij dC_ij = -b_i.v~_i  (b = P Y^, r = P 1)
template <typename T>
__global__ void hvp_prep_kernel(const T *X, const float *V, const float *b, const float *r, size_t rows, int d,
                                float *u, float *W1, float *Vt) {
    ROW_LOOP(i, rows) {
        const float rho = row_norm(X, i, d), inv = 1.f / rho;
        float xv = 0.f;
        for (int k = 0; k < d; ++k) xv = fmaf(ldc(X, i * d + k) * inv, V[i * d + k], xv);
        float su = 0.f;
        for (int k = 0; k < d; ++k) {
            const float vt = (V[i * d + k] - xv * (ldc(X, i * d + k) * inv)) * inv;
            Vt[i * d + k] = vt;
            W1[i * (d + 2) + k] = vt;
            su = fmaf(b[i * d + k], vt, su);
        }
        u[i] = -su;
        W1[i * (d + 2) + d] = 0.f;
        W1[i * (d + 2) + d + 1] = u[i] / r[i];
    }
}

// (H V)_i = [ (b_i.v_i) x^_i + s_i v_i + (x^_i.v_i) b_i - 3 s_i (x^_i.v_i) x^_i ] / rho_i^2
//           - (1/eps) (T_i - (x^_i.T_i) x^_i) / rho_i,
// s_i = x^_i.b_i,  T_i = df_i b_i + (P (dg o Y^))_i + sum_j P_ij (v~_i.y^_j) y^_j
// (Q1: P [dg o Y^ | dg], [n][d+1])
template <typename T>
__global__ void hvp_final_kernel(const T *X, const float *V, const float *b, const float *df, const float *Q1,
                                 const float *MV, size_t rows, int d, float eps, float *out) {
    ROW_LOOP(i, rows) {
        const float rho = row_norm(X, i, d), inv = 1.f / rho;
        float s = 0.f, bv = 0.f, xv = 0.f, xt = 0.f;
        for (int k = 0; k < d; ++k) {
            const float xh = ldc(X, i * d + k) * inv, v = V[i * d + k], bk = b[i * d + k];
            const float t = fmaf(df[i], bk, Q1[i * (d + 1) + k] + MV[i * d + k]);
            s = fmaf(xh, bk, s);
            bv = fmaf(bk, v, bv);
            xv = fmaf(xh, v, xv);
            xt = fmaf(xh, t, xt);
        }
        const float inv2 = inv * inv, ie = 1.f / eps;
        for (int k = 0; k < d; ++k) {
            const float xh = ldc(X, i * d + k) * inv, v = V[i * d + k], bk = b[i * d + k];
            const float t = fmaf(df[i], bk, Q1[i * (d + 1) + k] + MV[i * d + k]);
            const float second = (bv * xh + s * v + xv * bk - 3.f * s * xv * xh) * inv2;
            out[i * d + k] = second - ie * (t - xt * xh) * inv;
        }
    }
}

}  // namespace

cudaError_t cos_unit_rows(const void *P, bool bf16, size_t rows, int d, float *out, cudaStream_t s) {
    if (bf16)
        unit_rows_kernel<<<grid_rows(rows), 256, 0, s>>>(static_cast<const __nv_bfloat16 *>(P), rows, d, out);
    else
        unit_rows_kernel<<<grid_rows(rows), 256, 0, s>>>(static_cast<const float *>(P), rows, d, out);
    return cudaGetLastError();
}

cudaError_t cos_grad(const void *X, bool bf16, const float *b, size_t rows, int d, float *grad, cudaStream_t s) {
    if (bf16)
        grad_kernel<<<grid_rows(rows), 256, 0, s>>>(static_cast<const __nv_bfloat16 *>(X), b, rows, d, grad);
    else
        grad_kernel<<<grid_rows(rows), 256, 0, s>>>(static_cast<const float *>(X), b, rows, d, grad);
    return cudaGetLastError();
}

cudaError_t cos_hvp_prep(const void *X, bool bf16, const float *V, const float *b, const float *r, size_t rows, int d,
                         float *u, float *W1, float *Vt, cudaStream_t s) {
    if (bf16)
        hvp_prep_kernel<<<grid_rows(rows), 256, 0, s>>>(static_cast<const __nv_bfloat16 *>(X), V, b, r, rows, d, u,
                                                        W1, Vt);
    else
        hvp_prep_kernel<<<grid_rows(rows), 256, 0, s>>>(static_cast<const float *>(X), V, b, r, rows, d, u, W1, Vt);
    return cudaGetLastError();
}

cudaError_t cos_hvp_final(const void *X, bool bf16, const float *V, const float *b, const float *df, const float *Q1,
                          const float *MV, size_t rows, int d, float eps, float *out, cudaStream_t s) {
    if (bf16)
        hvp_final_kernel<<<grid_rows(rows), 256, 0, s>>>(static_cast<const __nv_bfloat16 *>(X), V, b, df, Q1, MV,
                                                         rows, d, eps, out);
    else
        hvp_final_kernel<<<grid_rows(rows), 256, 0, s>>>(static_cast<const float *>(X), V, b, df, Q1, MV, rows, d,
                                                         eps, out);
    return cudaGetLastError();
}

}  // namespace fs
