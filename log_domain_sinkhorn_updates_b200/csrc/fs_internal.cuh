// Internal declarations of the sm_100a log-domain Sinkhorn library.
//
// Notation follows "FlashSinkhorn: IO-aware EOT on GPU" (Metodologia,
// Proposition 1): a pass computes, for every row i of its "row side",
//
//   LSE2_i = log2 sum_j 2^( S_ij * log2(e)/eps + beta_j ),   S_ij = <q_i, k_j>
//
// where the packed operands are q = x - t and k = 2 (y - t) (t a common
// centre, zero for bf16 inputs), so S_ij = 2 (x_i - t).(y_j - t), and beta_j
// is the column bias ((g_j - |y_j - t|^2)/eps + log b_j) * log2(e) in base-2
// units (-inf on padding columns).  The f-update is then
//   f_i = |x_i - t|^2 - eps ln2 LSE2_i.
// The g-update is the same pass with the two sides exchanged (the product is
// symmetric in q and k: S_ji^T = <k_j, q_i>).  For the cosine cost the rows
// are normalised instead of centred, k = y^ (no factor 2) and every norm term
// is 1/2, so the same pass computes C_ij = 1 - x^_i.y^_j.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

namespace fs {

constexpr int kBlockRows = 128;   // rows of one CTA (one TMEM lane per row)
constexpr int kBlockCols = 256;   // columns of one streamed tile (the MMA's N)
constexpr float kLog2e = 1.4426950408889634f;
constexpr double kLn2d = 0.69314718055994530942;
constexpr double kLog2ed = 1.44269504088896340736;

// device error bits (fs_handle::err)
constexpr int kDevErrNonfinite = 1;
constexpr int kDevErrTimeout = 2;
constexpr int kDevErrBadWeights = 4;
constexpr int kDevErrZeroRow = 8;  // a zero row under the cosine cost

// Parameters of one streamed LSE pass (row side R against column side C).
struct PassParams {
    int rows, rows_pad;        // valid rows of the row side; packed operand rows per problem
    int rows_stride;           // per-problem stride of the row side's per-point arrays
    int cols, cols_rows;       // valid columns; packed operand rows per problem of the column side
    int cols_stride;           // per-problem stride of the column side's per-point arrays
    int row_bytes;             // bytes of a packed operand row (tensor-core paths)
    int swz;                   // swizzle span in bytes (32, 64 or 128)
    int plane_bytes;           // bytes of one operand plane (multiple of 32)
    int d;                     // feature dim of the plain fp32 layout (SIMT path)
    int splits;                // column splits (grid.y)
    int tiles_per_split;       // column tiles handled by one split
    int col_tiles;             // 256-column tiles covering cols
    int stages;                // pipeline depth (tensor-core path)
    int issuers;               // MMA-issuing threads of the one-CTA tensor-core pass: 1, or 2 (one per TMEM
                               // buffer, so the two softmax groups' score chains do not wait on each other)
    float scale2;              // log2(e)/eps, times sscale
    float sscale;              // factor from the MMA's raw score to S_ij (1 unless operands were scaled)
    double eps;
    const float *col_bias;     // [batch][cols_stride], base-2, -inf beyond cols
    const float *row_norm;     // [batch][rows_stride] |row - t|^2
    const float *row_logw2;    // [batch][rows_stride] log2 of the row weights
    const float *col_norm;     // [batch][cols_stride] (measure passes only)
    const float *pot_in;       // [batch][rows] current row potential (measure passes)
    float *pot_out;            // [batch][rows] new row potential (update passes)
    float *next_bias;          // [batch][rows_stride] base-2 bias for the opposite pass, or null
    void *next_bias_mm;        // with next_bias, or null: the same bias as score-product rows (store_bias_mm)
    float mm_inv_c;            // 1 / scale2: base-2 bias -> raw score units
    int mm_tf32;               // score-product rows in tf32 (else bf16)
    float4 *part;              // [batch][splits][rows_pad] split partials (m, l, w, -)
    unsigned *counters;        // [batch][row_blocks] arrival counters (self-resetting)
    double *stats;             // [batch][row_blocks][4] measure partial sums
    double *tail_stats;        // update passes, or null: [batch][row_blocks][4] marginal statistics of the
                               // potential this pass writes (the plan's row sums at that potential)
    // Measure passes with col_vec set take the plan-weighted average of a column
    // vector instead of the cost: vec_out_i = sum_j P_ij v_j, vec_rsum_i = sum_j P_ij
    // (may be null); no statistics.  Tensor-core passes only.
    const float *col_vec;      // [batch][cols_stride], zero beyond cols
    float *vec_out;            // [batch][rows]
    float *vec_rsum;           // [batch][rows] or null
    const void *plain_rows;    // SIMT path: [batch][rows_pad][d] fp32
    const void *plain_cols;    // SIMT path: [batch][cols_rows][d] fp32
    unsigned long long timeout_ns;
    int *err;
};

// ---------------------------------------------------------------------------
// small device helpers
// ---------------------------------------------------------------------------
__device__ __forceinline__ float ex2_approx(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// Packed pairs of fp32 (sm_100 f32x2 arithmetic: one instruction, two lanes).
__device__ __forceinline__ uint64_t pack2(float a, float b) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
    return r;
}
__device__ __forceinline__ void unpack2(uint64_t v, float &a, float &b) {
    asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(v));
}
__device__ __forceinline__ uint64_t fma2(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t r;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
    return r;
}
__device__ __forceinline__ uint64_t add2(uint64_t a, uint64_t b) {
    uint64_t r;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}
__device__ __forceinline__ float max3(float a, float b, float c) {
    float r;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}

// The column bias beta_j as the tensor-core pass adds it to the score: the
// update pass takes S'_ij = S_ij + beta_j / c from one more K step of its S
// product, against a tile whose rows are (1, 1, 1, 0, ...), so that
// z_ij = S'_ij c (c = scale2) needs no per-column load or add in the softmax.
// A column's 32-byte row holds beta_j / c split into three parts exact in the
// operand type, (hi, mid, lo, 0, ...): bf16 parts (8 significant bits each),
// or tf32 parts (fp32 values with the low 13 mantissa bits clear, which the
// tf32 product reads exactly); -inf (padding) is (-inf, 0, 0).
__device__ __forceinline__ float tf32_trunc(float x) { return __uint_as_float(__float_as_uint(x) & 0xFFFFE000u); }
__device__ __forceinline__ void store_bias_mm(void *mm, size_t j, float beta, float inv_c, int tf32) {
    const float v = beta * inv_c;
    uint4 w = make_uint4(0u, 0u, 0u, 0u);
    if (tf32) {
        float p0 = v, p1 = 0.f, p2 = 0.f;
        if (isfinite(v)) {
            p0 = tf32_trunc(v);
            const float r = v - p0;
            p1 = tf32_trunc(r);
            p2 = tf32_trunc(r - p1);
        }
        w = make_uint4(__float_as_uint(p0), __float_as_uint(p1), __float_as_uint(p2), 0u);
    } else {
        __nv_bfloat16 h0 = __float2bfloat16_rn(v), h1 = __float2bfloat16_rn(0.f), h2 = h1;
        if (isfinite(v)) {
            const float r = v - __bfloat162float(h0);
            h1 = __float2bfloat16_rn(r);
            h2 = __float2bfloat16_rn(r - __bfloat162float(h1));
        }
        w.x = (uint32_t)__bfloat16_as_ushort(h0) | ((uint32_t)__bfloat16_as_ushort(h1) << 16);
        w.y = (uint32_t)__bfloat16_as_ushort(h2);
    }
    uint4 *dst = reinterpret_cast<uint4 *>(static_cast<char *>(mm) + j * 32);
    dst[0] = w;
    dst[1] = make_uint4(0u, 0u, 0u, 0u);
}

__device__ __forceinline__ unsigned long long globaltimer_ns() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
    return t;
}

// Merge two online-LSE states (max m, sum l, weighted sum w) in base 2.
__device__ __forceinline__ void lse_merge(float &m, float &l, float &w, float m2, float l2, float w2) {
    float M = fmaxf(m, m2);
    if (M == -INFINITY) { m = -INFINITY; l = 0.f; w = 0.f; return; }
    float s1 = exp2f(m - M), s2 = exp2f(m2 - M);
    l = l * s1 + l2 * s2;
    w = w * s1 + w2 * s2;
    m = M;
}

// Finish 128 rows of a pass.  Called by exactly 128 threads (one per row,
// row_local = 0..127) that hold the final online state of their row over the
// CTA's column range.  bar_id/bar_threads name a barrier covering exactly
// these 128 threads.  Handles the split merge (the last CTA of a row block to
// arrive merges all splits in fixed order, so results are deterministic),
// the potential write, the next pass's bias, and measure-mode statistics.
template <bool MEASURE>
__device__ void finish_rows(const PassParams &p, int row_local, float m, float l, float w,
                            int bar_id, double *red_smem /* >= 4*128 doubles */,
                            int *flag_smem);

}  // namespace fs

namespace fs {
// Parameters of a transport application (P V with P_ij = a_i b_j exp((f_i + g_j - C_ij)/eps)
// at given potentials), in the orientation of the f-direction pass.
struct ApplyParams {
    int rows, rows_pad, rows_stride;  // row side (X): valid, padded, per-point stride
    int cols, cols_rows, cols_stride; // column side (Y)
    int d, d_p, row_elems, pack_mode, dv;
    float q_unscale, k_unscale;       // packed value x this = the operand's true value
    double scale;                     // log2(e)/eps
    const void *packQ, *packK;        // packed operand rows ([batch][rows_pad|cols_rows][row_elems])
    const float *row_norm, *row_logw2, *pot_row;  // |x_i|^2 term, log2 a_i, f
    const float *col_bias;            // ((g_j - |y_j|^2)/eps + ln b_j) log2 e, -inf padding
    const void *V;                    // [batch][cols][dv], fp32 or bf16 (v_bf16)
    int v_bf16;
    float *out;                       // [batch][rows][dv]
    float *rsum;                      // [batch][rows] or null
    int divide;                       // 1: out = P V / r (barycentric map)
    // tensor-core path only
    int row_bytes, swz, plane_bytes, dv_pad, kslots, stages;
    float sscale;                     // raw MMA score -> S_ij (3xF16 operand scaling)
    unsigned long long timeout_ns;
    int *err;
    // one-row-block two-group kernel (fs_apply_tc_q2.cu, batch 1): row blocks from
    // main_blocks on are split over their column tiles into tail_k parts, one CTA
    // each; a part leaves its raw O and row sum in tail_o [tail_k][tail rows][dv]
    // and tail_rs [tail_k][tail rows], and a merge kernel adds them.  tail_k = 1:
    // no split (main_blocks = every row block).
    int main_blocks, tail_k;
    float *tail_o, *tail_rs;
};

// Launchers (defined in the .cu files); all return cudaGetLastError().
cudaError_t launch_lse_simt(const PassParams &p, int batch, bool measure, cudaStream_t s);
// Single-CTA pass; qt = 128-row blocks resident per CTA (1 or 2; rows_pad / 128
// must be a multiple of qt).
cudaError_t launch_lse_tc(const PassParams &p, int batch, bool measure, int prec, int qt,
                          const void *map_rows, const void *map_cols, const void *map_bias, size_t smem_bytes,
                          cudaStream_t s);
size_t tc_smem_bytes(int row_bytes, int qt, int stages, bool measure);
int tc_max_stages(int row_bytes, int qt, bool measure);
// Transport application on CUDA cores (fp32): out = P V (or P V / r), rsum = P 1.
cudaError_t launch_apply_simt(const ApplyParams &p, int batch, cudaStream_t s);
// Tensor-core transport application (fs_apply_tc.cu): shared memory, K-ring
// depth and P~/V~ stage count for operand rows of row_bytes, dv_pad output
// columns and vpl planes of V~ (0 if it does not fit); V~ packing; the launch
// (prec as the LSE pass).
size_t apply_tc_plan(int row_bytes, int dv_pad, int vpl, int *kslots, int *stages);
cudaError_t launch_vt_pack(const void *V, bool bf16, int batch, int m, int dv, int m_pad, int dv_pad, int vpl,
                           void *out, cudaStream_t s);
cudaError_t launch_apply_tc(const ApplyParams &p, int batch, int prec, int vpl, const void *map_q, const void *map_k,
                            const void *map_v, size_t smem, cudaStream_t s);
// The CTA-pair transport application (fs_apply_tc2.cu): plan for dv_pad a
// multiple of 32 (at most 256), and the launch (map_k: 64-row boxes; rows_pad /
// 128 must be even).
size_t apply_tc2_plan(int row_bytes, int dv_pad, int vpl, int *kslots, int *stages);
// Two 128-row blocks per CTA sharing every streamed K tile and V~ quarter
// (fs_apply_tc_q2.cu; dv_pad <= 128, rows of up to 256 bytes).
// qb: 128-row blocks per CTA, 2 (each group its own block) or 1 (both groups on one
// block, alternate tiles).
size_t apply_q2_plan(int row_bytes, int dv_pad, int vpl, int qb, int *kslots, int *stages);
// With qb = 1 and p.tail_k > 1: the whole row blocks (if main_blocks > 0), the
// split ones' column parts, then the merge kernel.
cudaError_t launch_apply_q2(const ApplyParams &p, int batch, int prec, int vpl, int qb, const void *map_q,
                            const void *map_k, const void *map_v, size_t smem, cudaStream_t s);
cudaError_t launch_apply_tc2(const ApplyParams &p, int batch, int prec, int vpl, const void *map_q, const void *map_k,
                             const void *map_v, size_t smem, cudaStream_t s);
// A kernel whose one bounded mbarrier wait nothing ever completes: after
// timeout_ns it raises kDevErrTimeout and returns (fs_tc_common usage check).
cudaError_t launch_wait_probe(unsigned long long timeout_ns, int *err, cudaStream_t s);
// Element-wise pieces of the streaming Hessian-vector product (fs_hvp.cu).
cudaError_t hvp_prep(const void *X, bool bf16, const float *V, const float *PY, const float *r, int n, int d,
                     float *u, float *W1, cudaStream_t s);
cudaError_t hvp_w(const void *Y, bool bf16, const float *Tm, int m, int d, float alpha, float *z, cudaStream_t s);
cudaError_t hvp_vec(size_t n, const float *x, const float *a, float alpha, const float *y, float beta, bool div,
                    float *out, cudaStream_t s);
cudaError_t hvp_dot(int batch, size_t len, const float *x, const float *y, double *part, double *out,
                    cudaStream_t s);
cudaError_t hvp_center(int batch, size_t len, const double *sum, float *x, cudaStream_t s);
// steps[b] += 1 for each problem still running (its CG step count)
cudaError_t hvp_cg_step(int batch, size_t len, const double *rr, const double *pap, const double *zz, double tol2,
                        const float *p, const float *Ap, float *x, float *res, int *steps, cudaStream_t s);
cudaError_t hvp_cg_dir(int batch, size_t len, const double *rr_new, const double *rr, const double *zz, double tol2,
                       const float *res, float *p, cudaStream_t s);
cudaError_t hvp_dgy(const void *Y, bool bf16, const float *dg, int m, int d, float *out, cudaStream_t s);
cudaError_t hvp_df(size_t n, int d, const float *u, const float *Q, const float *r, float *df, cudaStream_t s);
cudaError_t hvp_ychunk(const void *Y, bool bf16, int m, int d, int k0, int nq, float *Vc, cudaStream_t s);
cudaError_t hvp_mv_acc(const float *V, const float *Oc, int n, int d, int k0, int nq, float *MV, cudaStream_t s);
cudaError_t hvp_final(const void *X, bool bf16, const float *V, const float *PY, const float *r, const float *df,
                      const float *Q1, const float *MV, int n, int d, float eps, float *out, cudaStream_t s);
// grad[bz][i][k] = 2 (r_i x_ik - pv[bz][i][k]) from the caller's X (fp32 or bf16).
cudaError_t launch_grad_combine(const void *X, bool bf16, const float *r, const float *pv, int batch, int rows,
                                int d, float *grad, cudaStream_t s);
// The CTA-pair variant (one MMA over two SMs; rows_pad / 128 must be even).
cudaError_t launch_lse_tc2(const PassParams &p, int batch, bool measure, int prec, const void *map_rows,
                           const void *map_cols, size_t smem_bytes, cudaStream_t s);
size_t tc2_smem_bytes(int row_bytes, int stages, bool measure);
int tc2_max_stages(int row_bytes, bool measure);
// The fused transport-matrix term of the HVP (fs_hvp_tc.cu): which U packing the
// handle's precision takes (0: none), the plan, the bf16 hi/lo split of U, the launch.
int hvp_w_mode(int prec, int plane_bytes, int row_bytes);
size_t hvp_w_plan(int row_bytes, int umode, int dv_pad, int vpl, int *kslots, int *stages);
cudaError_t launch_u_split(const float *V, int batch, int rows, int rows_pad, int d, int row_elems, void *out,
                           cudaStream_t s);
cudaError_t launch_hvp_w(const ApplyParams &p, int batch, int prec, int umode, int vpl, float cw, const float *dirv,
                         const float *center, const void *map_q, const void *map_u, const void *map_k,
                         const void *map_v, size_t smem, cudaStream_t s);
// Cosine-cost derivatives (fs_cosine.cu): unit rows p / |p| (fp32), the gradient
// -(b - (x^.b) x^) / |x| from b = P Y^, and the HVP's first and last steps.
cudaError_t cos_unit_rows(const void *P, bool bf16, size_t rows, int d, float *out, cudaStream_t s);
cudaError_t cos_grad(const void *X, bool bf16, const float *b, size_t rows, int d, float *grad, cudaStream_t s);
cudaError_t cos_hvp_prep(const void *X, bool bf16, const float *V, const float *b, const float *r, size_t rows, int d,
                         float *u, float *W1, float *Vt, cudaStream_t s);
cudaError_t cos_hvp_final(const void *X, bool bf16, const float *V, const float *b, const float *df, const float *Q1,
                          const float *MV, size_t rows, int d, float eps, float *out, cudaStream_t s);
// Record msg as this thread's handle-less error (what fs_last_error(NULL) returns).
void set_thread_error(const char *msg);
// Add `count` kernels launched outside fs_api.cu to what fs_kernel_launches reports.
void count_launches(unsigned count);
}  // namespace fs
