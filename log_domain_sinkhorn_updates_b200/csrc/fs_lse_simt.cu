// Streamed LSE pass on CUDA cores (plain fp32 FMA dot products).
//
// The validation path of the library (FS_PREC_F32_SIMT): the same pass as the
// tensor-core kernel -- row-stationary traversal, online max / sum-exp per
// row, nothing of size n*m stored -- with the score product computed by FMA
// in fp32 and the exponentials by the accurate exp2f.  One thread owns one
// row; column tiles of 32 points are staged in shared memory.
#include "fs_finish.cuh"

namespace fs {
namespace {

constexpr int kSimtCols = 32;

template <bool MEASURE>
__global__ void __launch_bounds__(kBlockRows) lse_simt_kernel(const PassParams p) {
    extern __shared__ float sm[];
    const int d = p.d;
    const int ld = d + 1;  // odd stride: conflict-free per-thread row reads
    float *srow = sm;                              // [128][d+1]
    float *scol = srow + kBlockRows * ld;          // [32][d]
    float *sbias = scol + kSimtCols * d;           // [32]
    float *scn = sbias + kSimtCols;                // [32]
    double *red = reinterpret_cast<double *>(scn + kSimtCols + (kSimtCols & 1));  // [4][128]
    int *flag = reinterpret_cast<int *>(red + 4 * kBlockRows);

    const int rl = threadIdx.x;
    const int rb = blockIdx.x, split = blockIdx.y, bz = blockIdx.z;
    const float *rows = static_cast<const float *>(p.plain_rows) + ((size_t)bz * p.rows_pad + (size_t)rb * kBlockRows) * d;
    const float *cols = static_cast<const float *>(p.plain_cols) + (size_t)bz * p.cols_rows * d;
    const float *bias = p.col_bias + (size_t)bz * p.cols_stride;
    const float *cnorm = MEASURE ? p.col_norm + (size_t)bz * p.cols_stride : nullptr;

    for (int e = rl; e < kBlockRows * d; e += kBlockRows) srow[(e / d) * ld + (e % d)] = rows[e];

    const int c_begin = split * p.tiles_per_split * kBlockCols;
    const int c_end = min(p.cols_rows, c_begin + p.tiles_per_split * kBlockCols);
    const float c = p.scale2;
    const float xn = MEASURE ? p.row_norm[(size_t)bz * p.rows_stride + rb * kBlockRows + rl] : 0.f;
    float m = -INFINITY, l = 0.f, w = 0.f;

    for (int c0 = c_begin; c0 < c_end; c0 += kSimtCols) {
        __syncthreads();
        for (int e = rl; e < kSimtCols * d; e += kBlockRows) scol[e] = cols[(size_t)c0 * d + e];
        if (rl < kSimtCols) {
            sbias[rl] = bias[c0 + rl];
            if (MEASURE) scn[rl] = cnorm[c0 + rl];
        }
        __syncthreads();
        float z[kSimtCols], sc[kSimtCols];
        float tmax = -INFINITY;
#pragma unroll 4
        for (int j = 0; j < kSimtCols; ++j) {
            float s = 0.f;
            for (int k = 0; k < d; ++k) s = fmaf(srow[rl * ld + k], scol[j * d + k], s);
            sc[j] = s;
            z[j] = fmaf(s, c, sbias[j]);
            tmax = fmaxf(tmax, z[j]);
        }
        const float mnew = fmaxf(m, tmax);
        if (mnew == -INFINITY) continue;
        const float scale = exp2f(m - mnew);
        float acc = 0.f, accw = 0.f;
#pragma unroll
        for (int j = 0; j < kSimtCols; ++j) {
            const float e = exp2f(z[j] - mnew);
            acc += e;
            if (MEASURE) accw = fmaf(e, xn + scn[j] - sc[j], accw);
        }
        l = l * scale + acc;
        if (MEASURE) w = w * scale + accw;
        m = mnew;
    }
    finish_rows<MEASURE>(p, blockIdx.x, rl, m, l, w, 0, red, flag);
}

size_t simt_smem_bytes(int d) {
    return sizeof(float) * ((size_t)kBlockRows * (d + 1) + (size_t)kSimtCols * d + 2 * kSimtCols + 1) +
           sizeof(double) * 4 * kBlockRows + 16 + 8;
}

}  // namespace

cudaError_t launch_lse_simt(const PassParams &p, int batch, bool measure, cudaStream_t s) {
    const size_t smem = simt_smem_bytes(p.d);
    dim3 grid(p.rows_pad / kBlockRows, p.splits, batch);
    if (measure) {
        cudaFuncSetAttribute(lse_simt_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        lse_simt_kernel<true><<<grid, kBlockRows, smem, s>>>(p);
    } else {
        cudaFuncSetAttribute(lse_simt_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        lse_simt_kernel<false><<<grid, kBlockRows, smem, s>>>(p);
    }
    return cudaGetLastError();
}

}  // namespace fs
