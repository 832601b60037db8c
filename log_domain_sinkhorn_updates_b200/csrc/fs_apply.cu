// Transport application on CUDA cores: out_i = sum_j P_ij V_j (and r_i =
// sum_j P_ij) for the plan P_ij = a_i b_j exp((f_i + g_j - C_ij)/eps) at given
// potentials, without forming P ("FlashSinkhorn: IO-aware EOT on GPU",
// Metodologia section 3: the barycentric projection and the gradient as
// plan-weighted averages over the same streamed tiles).
//
// In the f-direction orientation of the streamed passes, with S_ij = q_i.k_j
// the score of the packed operands (2 (x_i - t).(y_j - t), or x^.y^ for the
// cosine cost),
//   log2 P_ij = alpha_i + beta_j + S_ij log2(e)/eps,
//   alpha_i   = log2 a_i + (f_i - |x_i|^2) log2(e)/eps,
//   beta_j    = the column bias of the LSE pass (from g).
// The exponent is summed in double (its terms are large and of both signs),
// the dot product and the weighted sums in fp32.  One thread per row, 128
// rows per CTA; columns stream through shared memory in tiles of 32 with the
// packed operand rows turned back into fp32 values.  A CTA covers kChunk
// columns of V (blockIdx.y picks which), so dv of any size is covered by
// recomputing the scores once per chunk.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "fs_prep.cuh"

namespace fs {
namespace {

constexpr int kApplyRows = 128;
constexpr int kApplyCols = 32;
constexpr int kChunk = 32;  // columns of V per CTA

// Element k (< d) of a packed operand row, as the true fp32 value.
__device__ __forceinline__ float unpack_elem(const void *row, int mode, int d_p, int k, float unscale) {
    if (mode == kPackBf16) return __bfloat162float(static_cast<const __nv_bfloat16 *>(row)[k]);
    if (mode == kPack3xF16) {
        const __half *h = static_cast<const __half *>(row);
        return (__half2float(h[k]) + __half2float(h[d_p + k])) * unscale;
    }
    const float *f = static_cast<const float *>(row);
    if (mode == kPack3xTf32) return f[k] + f[d_p + k];
    return f[k];  // tf32-rounded or plain fp32
}

__device__ __forceinline__ size_t elem_bytes(int mode) {
    return (mode == kPackBf16 || mode == kPack3xF16) ? 2 : 4;
}

__global__ void __launch_bounds__(kApplyRows) apply_simt_kernel(const ApplyParams p) {
    extern __shared__ float sm[];
    const int d = p.d;
    const int ld = d + 1;
    float *srow = sm;                                    // [128][d+1]
    float *scol = srow + kApplyRows * ld;                // [32][d]
    float *sv = scol + kApplyCols * d;                   // [32][kChunk]
    float *sb = sv + kApplyCols * kChunk;                // [32]

    const int rl = threadIdx.x;
    const int rb = blockIdx.x, chunk = blockIdx.y, bz = blockIdx.z;
    const int row = rb * kApplyRows + rl;
    const int c0 = chunk * kChunk;
    const int nc = min(kChunk, p.dv - c0);
    const size_t eb = elem_bytes(p.pack_mode);
    const uint8_t *qbase = static_cast<const uint8_t *>(p.packQ) +
                           ((size_t)bz * p.rows_pad + (size_t)rb * kApplyRows) * p.row_elems * eb;
    const uint8_t *kbase = static_cast<const uint8_t *>(p.packK) + (size_t)bz * p.cols_rows * p.row_elems * eb;

    for (int e = rl; e < kApplyRows * d; e += kApplyRows) {
        const int r = e / d, k = e % d;
        srow[r * ld + k] = unpack_elem(qbase + (size_t)r * p.row_elems * eb, p.pack_mode, p.d_p, k, p.q_unscale);
    }
    const bool valid = row < p.rows;
    const size_t prow = (size_t)bz * p.rows_stride + row;
    const double alpha = valid ? (double)p.row_logw2[prow] +
                                     ((double)p.pot_row[(size_t)bz * p.rows + row] - (double)p.row_norm[prow]) * p.scale
                               : 0.0;
    float acc[kChunk];
#pragma unroll
    for (int c = 0; c < kChunk; ++c) acc[c] = 0.f;
    float rs = 0.f;

    for (int j0 = 0; j0 < p.cols; j0 += kApplyCols) {
        __syncthreads();
        for (int e = rl; e < kApplyCols * d; e += kApplyRows) {
            const int j = e / d, k = e % d;
            scol[e] = j0 + j < p.cols ? unpack_elem(kbase + (size_t)(j0 + j) * p.row_elems * eb, p.pack_mode, p.d_p,
                                                    k, p.k_unscale)
                                      : 0.f;
        }
        for (int e = rl; e < kApplyCols * kChunk; e += kApplyRows) {
            const int j = e / kChunk, c = e % kChunk;
            float v = 0.f;
            if (j0 + j < p.cols && c < nc) {
                const size_t vi = ((size_t)bz * p.cols + j0 + j) * p.dv + c0 + c;
                v = p.v_bf16 ? __bfloat162float(static_cast<const __nv_bfloat16 *>(p.V)[vi])
                             : static_cast<const float *>(p.V)[vi];
            }
            sv[e] = v;
        }
        if (rl < kApplyCols)
            sb[rl] = j0 + rl < p.cols ? p.col_bias[(size_t)bz * p.cols_stride + j0 + rl] : -INFINITY;
        __syncthreads();
        if (!valid) continue;
        const int jn = min(kApplyCols, p.cols - j0);
        for (int j = 0; j < jn; ++j) {
            float s = 0.f;
            for (int k = 0; k < d; ++k) s = fmaf(srow[rl * ld + k], scol[j * d + k], s);
            const double arg = alpha + (double)sb[j] + (double)s * p.scale;
            const float e = exp2f((float)arg);
            rs += e;
#pragma unroll
            for (int c = 0; c < kChunk; ++c) acc[c] = fmaf(e, sv[j * kChunk + c], acc[c]);
        }
    }
    if (!valid) return;
    const float inv = p.divide ? 1.f / rs : 1.f;
    for (int c = 0; c < nc; ++c) p.out[((size_t)bz * p.rows + row) * p.dv + c0 + c] = acc[c] * inv;
    if (p.rsum && chunk == 0) p.rsum[(size_t)bz * p.rows + row] = rs;
}

template <typename T>
__device__ __forceinline__ float ld_val(const T *p, size_t i);
template <>
__device__ __forceinline__ float ld_val<float>(const float *p, size_t i) {
    return p[i];
}
template <>
__device__ __forceinline__ float ld_val<__nv_bfloat16>(const __nv_bfloat16 *p, size_t i) {
    return __bfloat162float(p[i]);
}

template <typename T>
__global__ void grad_combine_kernel(const T *X, const float *r, const float *pv, size_t total, int d, float *grad) {
    for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < total; i += (size_t)gridDim.x * blockDim.x)
        grad[i] = 2.f * fmaf(r[i / d], ld_val(X, i), -pv[i]);
}

}  // namespace

cudaError_t launch_apply_simt(const ApplyParams &p, int batch, cudaStream_t s) {
    const size_t smem = sizeof(float) * ((size_t)kApplyRows * (p.d + 1) + (size_t)kApplyCols * p.d +
                                         (size_t)kApplyCols * kChunk + kApplyCols);
    cudaError_t e = cudaFuncSetAttribute(apply_simt_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    dim3 grid(p.rows_pad / kApplyRows, (p.dv + kChunk - 1) / kChunk, batch);
    apply_simt_kernel<<<grid, kApplyRows, smem, s>>>(p);
    return cudaGetLastError();
}

cudaError_t launch_grad_combine(const void *X, bool bf16, const float *r, const float *pv, int batch, int rows,
                                int d, float *grad, cudaStream_t s) {
    const size_t total = (size_t)batch * rows * d;
    const size_t want = (total + 255) / 256;
    const int blocks = (int)(want < 148 * 16 ? want : 148 * 16);
    if (bf16)
        grad_combine_kernel<<<blocks, 256, 0, s>>>(static_cast<const __nv_bfloat16 *>(X), r, pv, total, d, grad);
    else
        grad_combine_kernel<<<blocks, 256, 0, s>>>(static_cast<const float *>(X), r, pv, total, d, grad);
    return cudaGetLastError();
}

}  // namespace fs
