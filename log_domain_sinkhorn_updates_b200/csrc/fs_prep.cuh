// Launchers of the set-up and helper kernels (fs_prep.cu).
#pragma once

#include "fs_internal.cuh"

namespace fs {

// Operand packing modes.
constexpr int kPackBf16 = 0;    // one bf16 plane
constexpr int kPackTf32 = 1;    // one fp32 plane rounded to tf32
constexpr int kPack3xTf32 = 2;  // [hi | lo] fp32 planes, hi = tf32(v), lo = v - hi
constexpr int kPackPlain = 3;   // plain fp32 rows of d values (SIMT path)
constexpr int kPack3xF16 = 4;   // [hi | lo] fp16 planes of the scaled value, hi = f16(v), lo = f16(v - hi)

cudaError_t launch_center(const void *X, const void *Y, bool bf16, int batch, int n, int m, int d, float *t,
                          cudaStream_t s);
// normalize: divide each row by its Euclidean norm first (cosine cost; t must
// be null) and store 1/2 as its squared norm: with the column side packed at
// scale 1 instead of 2, |q|^2 + |k|^2 - q.k = 1/2 + 1/2 - cos = 1 - cos.
// A zero row raises kDevErrZeroRow.
cudaError_t launch_pack(const void *src, bool bf16, int rows, int rows_pad, int d, int batch, const float *t,
                        float scale, int mode, int d_p, int row_elems, void *dst, float *norm, int norm_stride,
                        int *err, cudaStream_t s, bool normalize = false);
// out[0] = max over every problem of |src - t| (fp32), for the 3xF16 scaling.
cudaError_t launch_maxabs(const void *src, bool bf16, int rows, int d, int batch, const float *t, float *out,
                          cudaStream_t s);
cudaError_t launch_weights(const float *w, int batch, int cnt, int cnt_pad, float *lw2, double *wstat,
                           cudaStream_t s);
cudaError_t launch_fill(float *p, size_t count, float v, cudaStream_t s);
// v [batch][cnt] -> out [batch][stride], zero beyond cnt.
cudaError_t launch_pad_vec(const float *v, int batch, int cnt, int stride, float *out, cudaStream_t s);
// out [batch][cnt_pad]: the base-2 bias of the pass whose columns are this side,
// -inf beyond cnt; mm (may be null): the same as score-product rows
// (store_bias_mm, 32 bytes per column).
cudaError_t launch_bias(const float *pot, int batch, int cnt, int cnt_pad, const float *norm, const float *lw2,
                        double scale2, float *out, void *mm, float mm_inv_c, int mm_tf32, cudaStream_t s);
// count bias rows (32 bytes each) set to a padding column's.
cudaError_t launch_fill_bias_mm(void *mm, size_t count, int tf32, cudaStream_t s);
// *flag |= 1 if the count floats at a and b differ in any bit.
cudaError_t launch_differs(const float *a, const float *b, size_t count, int *flag, cudaStream_t s);
cudaError_t launch_finalize(const double *stats, int batch, int row_blocks, const float *col_pot,
                            const float *col_lw2, int cols, int cols_pad, double *out, cudaStream_t s);

}  // namespace fs
