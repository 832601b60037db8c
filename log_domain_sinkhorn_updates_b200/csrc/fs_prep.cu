// O((n+m)d) set-up and per-pass helper kernels: centring, operand packing
// with squared norms, log-weights, column/row biases, and the final
// deterministic reduction of measure-pass statistics.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "fs_prep.cuh"

namespace fs {
namespace {

template <typename T>
__device__ __forceinline__ float load_val(const T *p, size_t i);
template <>
__device__ __forceinline__ float load_val<float>(const float *p, size_t i) {
    return p[i];
}
template <>
__device__ __forceinline__ float load_val<__nv_bfloat16>(const __nv_bfloat16 *p, size_t i) {
    return __bfloat162float(p[i]);
}

// Deterministic 256-thread block sum of one double per thread (fixed tree).
__device__ double block_sum_256(double v, double *sh) {
    sh[threadIdx.x] = v;
    __syncthreads();
    for (int s = 128; s > 0; s >>= 1) {
        if ((int)threadIdx.x < s) sh[threadIdx.x] += sh[threadIdx.x + s];
        __syncthreads();
    }
    double r = sh[0];
    __syncthreads();
    return r;
}

// t_k = (mean_i x_ik + mean_j y_jk) / 2, one block per (k, problem).
template <typename T>
__global__ void center_kernel(const T *X, const T *Y, int n, int m, int d, float *t) {
    __shared__ double sh[256];
    const int k = blockIdx.x, bz = blockIdx.y;
    double sx = 0.0, sy = 0.0;
    for (int i = threadIdx.x; i < n; i += 256) sx += load_val(X, ((size_t)bz * n + i) * d + k);
    for (int j = threadIdx.x; j < m; j += 256) sy += load_val(Y, ((size_t)bz * m + j) * d + k);
    sx = block_sum_256(sx, sh);
    sy = block_sum_256(sy, sh);
    if (threadIdx.x == 0) t[(size_t)bz * d + k] = (float)(0.5 * (sx / n + sy / m));
}

__device__ __forceinline__ float round_tf32(float x) {
    uint32_t r;
    asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
    return __uint_as_float(r);
}

// One warp per padded row: v = src - t (fp32), packed = scale * v in the
// layout of `mode`, norm = |v|^2 (double accumulation, fixed shuffle tree).
// With `normalize`, v = src / |src| instead and norm = 1/2 (cosine cost).
template <typename T>
__global__ void pack_kernel(const T *src, int rows, int rows_pad, int d, int batch, const float *t, float scale,
                            int mode, int d_p, int row_elems, void *dst, float *norm, int norm_stride, int *err,
                            bool normalize) {
    const int lane = threadIdx.x & 31;
    const long long gw = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const long long nw = ((long long)gridDim.x * blockDim.x) >> 5;
    for (long long wr = gw; wr < (long long)batch * rows_pad; wr += nw) {
        const int bz = (int)(wr / rows_pad), r = (int)(wr % rows_pad);
        const bool valid = r < rows;
        double acc = 0.0;
        bool bad = false;
        float inv = 1.f;
        if (normalize) {
            double ss = 0.0;
            if (valid)
                for (int k = lane; k < d; k += 32) {
                    const double x = load_val(src, ((size_t)bz * rows + r) * d + k);
                    ss += x * x;
                }
            for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
            if (valid && !(ss > 0.0)) {
                if (lane == 0) atomicOr(err, kDevErrZeroRow);
            } else if (valid) {
                inv = (float)(1.0 / sqrt(ss));
            }
        }
        for (int e = lane; e < row_elems; e += 32) {
            float v = 0.f;
            int k = e;
            int plane = 0;
            if (mode == kPack3xTf32 || mode == kPack3xF16) {
                plane = e / d_p;
                k = e % d_p;
                if (plane > 1) k = d;  // padding beyond the two planes
            }
            if (valid && k < d) {
                float x = load_val(src, ((size_t)bz * rows + r) * d + k);
                if (!isfinite(x)) bad = true;
                v = normalize ? x * inv : x - (t ? t[(size_t)bz * d + k] : 0.f);
            }
            float out;
            if (mode == kPackBf16) {
                const __nv_bfloat16 q = __float2bfloat16_rn(v);
                const float vq = __bfloat162float(q);
                if (k < d) acc += (double)vq * vq;
                static_cast<__nv_bfloat16 *>(dst)[wr * row_elems + e] = __float2bfloat16_rn(scale * vq);
                continue;
            } else if (mode == kPackTf32) {
                out = round_tf32(scale * v);
                if (k < d) acc += (double)v * v;
            } else if (mode == kPack3xF16) {
                // scale is a power of two chosen so that |scale * v| <= 2^14: exact,
                // and far inside the fp16 range.
                const float sv = scale * v;
                const __half hi = __float2half_rn(sv);
                const __half lo = __float2half_rn(sv - __half2float(hi));
                if (plane == 0 && k < d) acc += (double)v * v;
                static_cast<__half *>(dst)[wr * row_elems + e] =
                    plane == 0 ? hi : (plane == 1 ? lo : __float2half_rn(0.f));
                continue;
            } else if (mode == kPack3xTf32) {
                const float sv = scale * v;
                const float hi = round_tf32(sv);
                out = plane == 0 ? hi : (plane == 1 ? sv - hi : 0.f);
                if (plane == 0 && k < d) acc += (double)v * v;
            } else {  // plain fp32
                out = scale * v;
                if (k < d) acc += (double)v * v;
            }
            static_cast<float *>(dst)[wr * row_elems + e] = out;
        }
        for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
        if (bad) atomicOr(err, kDevErrNonfinite);
        if (lane == 0) norm[(size_t)bz * norm_stride + r] = valid ? (normalize ? 0.5f : (float)acc) : 0.f;
    }
}

// max |src - t| over every element of every problem (one block per problem,
// fixed-order tree; the per-problem maxima are folded with atomicMax on the
// float bits, which orders like the values for non-negative floats).
template <typename T>
__global__ void maxabs_kernel(const T *src, int rows, int d, const float *t, unsigned *out) {
    __shared__ float sh[256];
    const int bz = blockIdx.x;
    float mx = 0.f;
    for (size_t e = threadIdx.x; e < (size_t)rows * d; e += 256) {
        const int k = (int)(e % d);
        const float v = load_val(src, (size_t)bz * rows * d + e) - (t ? t[(size_t)bz * d + k] : 0.f);
        mx = fmaxf(mx, fabsf(v));
    }
    sh[threadIdx.x] = mx;
    __syncthreads();
    for (int s = 128; s > 0; s >>= 1) {
        if ((int)threadIdx.x < s) sh[threadIdx.x] = fmaxf(sh[threadIdx.x], sh[threadIdx.x + s]);
        __syncthreads();
    }
    if (threadIdx.x == 0) atomicMax(out, __float_as_uint(sh[0]));
}

// log2 of the weights (uniform when w == null), -inf on padding; per-problem
// sum (for the |sum - 1| check) and count of non-positive / non-finite entries.
__global__ void weights_kernel(const float *w, int cnt, int cnt_pad, float *lw2, double *wstat) {
    __shared__ double sh[256];
    const int bz = blockIdx.x;
    double s = 0.0, bad = 0.0;
    const double ulog = -log2((double)cnt);
    for (int i = threadIdx.x; i < cnt_pad; i += 256) {
        float out = -INFINITY;
        if (i < cnt) {
            if (w) {
                const float v = w[(size_t)bz * cnt + i];
                if (!(v > 0.f) || !isfinite(v)) bad += 1.0;
                s += (double)v;
                out = (float)log2((double)v);
            } else {
                s += 1.0 / cnt;
                out = (float)ulog;
            }
        }
        lw2[(size_t)bz * cnt_pad + i] = out;
    }
    s = block_sum_256(s, sh);
    bad = block_sum_256(bad, sh);
    if (threadIdx.x == 0) {
        wstat[2 * bz + 0] = s;
        wstat[2 * bz + 1] = bad;
    }
}

__global__ void fill_kernel(float *p, size_t count, float v) {
    for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < count; i += (size_t)gridDim.x * blockDim.x)
        p[i] = v;
}

// out_j = ((pot_j - |col_j|^2) log2(e)/eps + log2 w_j), -inf on padding.
__global__ void bias_kernel(const float *pot, int cnt, int cnt_pad, int batch, const float *norm, const float *lw2,
                            double scale2, float *out, void *mm, float mm_inv_c, int mm_tf32) {
    const size_t total = (size_t)batch * cnt_pad;
    for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < total; i += (size_t)gridDim.x * blockDim.x) {
        const int bz = (int)(i / cnt_pad), j = (int)(i % cnt_pad);
        float v = -INFINITY;
        if (j < cnt) v = (float)__fma_rn((double)pot[(size_t)bz * cnt + j] - (double)norm[i], scale2, (double)lw2[i]);
        out[i] = v;
        if (mm) store_bias_mm(mm, i, v, mm_inv_c, mm_tf32);
    }
}

// Every bias row of a side as a padding column's: (-inf, 0, 0, ...).
__global__ void fill_bias_mm_kernel(void *mm, size_t count, int tf32) {
    for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < count; i += (size_t)gridDim.x * blockDim.x)
        store_bias_mm(mm, i, -INFINITY, 1.f, tf32);
}

// out[bz][0..3] = sum over row blocks of the measure statistics (fixed order);
// out[bz][4] = sum_j w_j pot_j over the column side (when pot != null).
__global__ void finalize_kernel(const double *stats, int row_blocks, const float *col_pot, const float *col_lw2,
                                int cols, int cols_pad, double *out) {
    __shared__ double sh[256];
    const int bz = blockIdx.x;
    if (threadIdx.x < 4) {
        double s = 0.0;
        for (int r = 0; r < row_blocks; ++r) s += stats[((size_t)bz * row_blocks + r) * 4 + threadIdx.x];
        out[(size_t)bz * 8 + threadIdx.x] = s;
    }
    double acc = 0.0;
    if (col_pot)
        for (int j = threadIdx.x; j < cols; j += 256)
            acc += exp2((double)col_lw2[(size_t)bz * cols_pad + j]) * (double)col_pot[(size_t)bz * cols + j];
    acc = block_sum_256(acc, sh);
    if (threadIdx.x == 0) out[(size_t)bz * 8 + 4] = acc;
}

// flag |= 1 where a and b differ in any bit (a potential and its snapshot).
__global__ void differs_kernel(const float *a, const float *b, size_t count, int *flag) {
    const uint32_t *ua = reinterpret_cast<const uint32_t *>(a);
    const uint32_t *ub = reinterpret_cast<const uint32_t *>(b);
    int any = 0;
    for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < count; i += (size_t)gridDim.x * blockDim.x)
        any |= ua[i] != ub[i];
    if (__syncthreads_or(any) && threadIdx.x == 0) atomicOr(flag, 1);
}

int grid_for(size_t work, int per_block) {
    size_t g = (work + per_block - 1) / per_block;
    if (g > 148 * 32) g = 148 * 32;
    return (int)(g < 1 ? 1 : g);
}

}  // namespace

cudaError_t launch_center(const void *X, const void *Y, bool bf16, int batch, int n, int m, int d, float *t,
                          cudaStream_t s) {
    dim3 grid(d, batch);
    if (bf16)
        center_kernel<<<grid, 256, 0, s>>>(static_cast<const __nv_bfloat16 *>(X),
                                          static_cast<const __nv_bfloat16 *>(Y), n, m, d, t);
    else
        center_kernel<<<grid, 256, 0, s>>>(static_cast<const float *>(X), static_cast<const float *>(Y), n, m,
                                          d, t);
    return cudaGetLastError();
}

cudaError_t launch_pack(const void *src, bool bf16, int rows, int rows_pad, int d, int batch, const float *t,
                        float scale, int mode, int d_p, int row_elems, void *dst, float *norm, int norm_stride,
                        int *err, cudaStream_t s, bool normalize) {
    const size_t warps = (size_t)batch * rows_pad;
    const int grid = grid_for(warps * 32, 256);
    if (bf16)
        pack_kernel<<<grid, 256, 0, s>>>(static_cast<const __nv_bfloat16 *>(src), rows, rows_pad, d, batch, t,
                                        scale, mode, d_p, row_elems, dst, norm, norm_stride, err, normalize);
    else
        pack_kernel<<<grid, 256, 0, s>>>(static_cast<const float *>(src), rows, rows_pad, d, batch, t, scale,
                                        mode, d_p, row_elems, dst, norm, norm_stride, err, normalize);
    return cudaGetLastError();
}

cudaError_t launch_maxabs(const void *src, bool bf16, int rows, int d, int batch, const float *t, float *out,
                          cudaStream_t s) {
    cudaError_t e = cudaMemsetAsync(out, 0, sizeof(float), s);
    if (e != cudaSuccess) return e;
    unsigned *o = reinterpret_cast<unsigned *>(out);
    if (bf16)
        maxabs_kernel<<<batch, 256, 0, s>>>(static_cast<const __nv_bfloat16 *>(src), rows, d, t, o);
    else
        maxabs_kernel<<<batch, 256, 0, s>>>(static_cast<const float *>(src), rows, d, t, o);
    return cudaGetLastError();
}

cudaError_t launch_weights(const float *w, int batch, int cnt, int cnt_pad, float *lw2, double *wstat,
                           cudaStream_t s) {
    weights_kernel<<<batch, 256, 0, s>>>(w, cnt, cnt_pad, lw2, wstat);
    return cudaGetLastError();
}

// out[b][j] = v[b][j] for j < cnt, 0 up to stride: a per-point vector in the
// padded per-point layout the streamed passes read
__global__ void pad_vec_kernel(const float *v, int batch, int cnt, int stride, float *out) {
    const size_t total = (size_t)batch * stride;
    for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < total; i += (size_t)gridDim.x * blockDim.x) {
        const size_t b = i / stride;
        const int j = (int)(i % stride);
        out[i] = j < cnt ? v[b * cnt + j] : 0.f;
    }
}

cudaError_t launch_pad_vec(const float *v, int batch, int cnt, int stride, float *out, cudaStream_t s) {
    pad_vec_kernel<<<grid_for((size_t)batch * stride, 256), 256, 0, s>>>(v, batch, cnt, stride, out);
    return cudaGetLastError();
}

cudaError_t launch_fill(float *p, size_t count, float v, cudaStream_t s) {
    fill_kernel<<<grid_for(count, 256), 256, 0, s>>>(p, count, v);
    return cudaGetLastError();
}

cudaError_t launch_bias(const float *pot, int batch, int cnt, int cnt_pad, const float *norm, const float *lw2,
                        double scale2, float *out, void *mm, float mm_inv_c, int mm_tf32, cudaStream_t s) {
    bias_kernel<<<grid_for((size_t)batch * cnt_pad, 256), 256, 0, s>>>(pot, cnt, cnt_pad, batch, norm, lw2, scale2,
                                                                      out, mm, mm_inv_c, mm_tf32);
    return cudaGetLastError();
}

cudaError_t launch_fill_bias_mm(void *mm, size_t count, int tf32, cudaStream_t s) {
    fill_bias_mm_kernel<<<grid_for(count, 256), 256, 0, s>>>(mm, count, tf32);
    return cudaGetLastError();
}

cudaError_t launch_differs(const float *a, const float *b, size_t count, int *flag, cudaStream_t s) {
    differs_kernel<<<grid_for(count, 256), 256, 0, s>>>(a, b, count, flag);
    return cudaGetLastError();
}

cudaError_t launch_finalize(const double *stats, int batch, int row_blocks, const float *col_pot,
                            const float *col_lw2, int cols, int cols_pad, double *out, cudaStream_t s) {
    finalize_kernel<<<batch, 256, 0, s>>>(stats, row_blocks, col_pot, col_lw2, cols, cols_pad, out);
    return cudaGetLastError();
}

}  // namespace fs
