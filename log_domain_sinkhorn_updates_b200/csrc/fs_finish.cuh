// Row epilogue shared by the streamed LSE passes: column-split merge,
// potential write, next-pass bias, and measure-mode statistics.
#pragma once

#include "fs_internal.cuh"

namespace fs {

__device__ __forceinline__ void named_barrier(int id, int nthreads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// rb: the 128-row block this CTA's rows belong to; the CTA's 128 threads of
// that block call this together (named barrier bar_id).
template <bool MEASURE>
__device__ void finish_rows(const PassParams &p, int rb, int rl, float m, float l, float w, int bar_id,
                            double *red, int *flag) {
    const int split = blockIdx.y, bz = blockIdx.z;
    const int row_blocks = p.rows_pad / kBlockRows;
    const int row = rb * kBlockRows + rl;
    const size_t prow = (size_t)bz * p.rows_stride + row;  // per-point arrays of the row side

    if (p.splits > 1) {
        // Publish this split's partial state, then let the last CTA of the row
        // block (in arrival order) merge all splits in split order.
        float4 *mine = p.part + ((size_t)bz * p.splits + split) * p.rows_pad;
        mine[row] = make_float4(m, l, w, 0.f);
        __threadfence();
        named_barrier(bar_id, kBlockRows);
        if (rl == 0) {
            unsigned *ctr = p.counters + (size_t)bz * row_blocks + rb;
            unsigned old = atomicAdd(ctr, 1u);
            int last = (old == (unsigned)(p.splits - 1));
            if (last) *ctr = 0u;  // every split has arrived: reset for the next pass
            *flag = last;
        }
        named_barrier(bar_id, kBlockRows);
        if (!*flag) return;
        __threadfence();
        const float4 *base = p.part + (size_t)bz * p.splits * p.rows_pad;
        float4 v = __ldcg(base + row);
        m = v.x;
        l = v.y;
        w = v.z;
        for (int s = 1; s < p.splits; ++s) {
            float4 u = __ldcg(base + (size_t)s * p.rows_pad + row);
            lse_merge(m, l, w, u.x, u.y, u.z);
        }
    }

    const bool valid = row < p.rows;
    const double lse2 = (l > 0.f) ? (double)m + log2((double)l) : -INFINITY;

    double c0 = 0.0, c1 = 0.0, c2 = 0.0, c3 = 0.0;
    if (!MEASURE) {
        if (valid) {
            const double pot = (double)p.row_norm[prow] - p.eps * kLn2d * lse2;
            const float pot32 = (float)pot;
            p.pot_out[(size_t)bz * p.rows + row] = pot32;
            if (!isfinite(pot)) atomicOr(p.err, kDevErrNonfinite);
            // The opposite pass's bias, computed from the stored float potential
            // exactly as the standalone bias kernel does, so a fused solve equals
            // the same sequence of single updates bit for bit.
            if (p.next_bias) {
                const float nb =
                    (float)__fma_rn((double)pot32 - (double)p.row_norm[prow], kLog2ed / p.eps, (double)p.row_logw2[prow]);
                p.next_bias[prow] = nb;
                if (p.next_bias_mm) store_bias_mm(p.next_bias_mm, prow, nb, p.mm_inv_c, p.mm_tf32);
            }
            if (p.tail_stats) {
                // The plan's row sum at the stored potential: the exact update is
                // pot, the stored value pot32, so r_i = a_i exp((pot32 - pot)/eps)
                // (what a measure pass at the same potentials computes).
                const double a = exp2((double)p.row_logw2[prow]);
                const double r = a * exp2(((double)pot32 - pot) * (kLog2ed / p.eps));
                c0 = fabs(r - a);
                c1 = r;
                c3 = a * (double)pot32;
            }
        }
        if (!p.tail_stats) return;  // uniform over the kernel: a launch parameter
    } else if (p.col_vec) {
        // Vector pass: w / l is the plan-weighted average of v over row i, and the
        // row sum r_i is that of a measure pass (below), so sum_j P_ij v_j = r_i w_i / l_i.
        if (valid) {
            const double lw2 = (double)p.row_logw2[prow];
            const double pot = (double)p.pot_in[(size_t)bz * p.rows + row];
            const double r = exp2(lw2 + (pot - (double)p.row_norm[prow]) * (kLog2ed / p.eps) + lse2);
            const double avg = (l > 0.f) ? (double)w / (double)l : 0.0;
            p.vec_out[(size_t)bz * p.rows + row] = (float)(r * avg);
            if (p.vec_rsum) p.vec_rsum[(size_t)bz * p.rows + row] = (float)r;
            if (!isfinite(r) || !isfinite(avg)) atomicOr(p.err, kDevErrNonfinite);
        }
        return;  // uniform over the kernel: a launch parameter
    } else if (valid) {
        // Measure mode: with the current row potential pot_in, the plan's row sum is
        //   r_i = a_i exp((pot_i - pot~_i)/eps),  pot~_i = |row|^2 - eps ln2 LSE2_i,
        // i.e. log2 r_i = log2 a_i + (pot_i - |row|^2) log2(e)/eps + LSE2_i, and
        // sum_j P_ij C_ij = r_i * (w_i / l_i).
        const double lw2 = (double)p.row_logw2[prow];
        const double pot = (double)p.pot_in[(size_t)bz * p.rows + row];
        const double a = exp2(lw2);
        const double r = exp2(lw2 + (pot - (double)p.row_norm[prow]) * (kLog2ed / p.eps) + lse2);
        const double mc = (l > 0.f) ? (double)w / (double)l : 0.0;
        c0 = fabs(r - a);
        c1 = r;
        c2 = r * mc;
        c3 = a * pot;
        if (!isfinite(r) || !isfinite(mc)) atomicOr(p.err, kDevErrNonfinite);
    }

    red[0 * kBlockRows + rl] = c0;
    red[1 * kBlockRows + rl] = c1;
    red[2 * kBlockRows + rl] = c2;
    red[3 * kBlockRows + rl] = c3;
    named_barrier(bar_id, kBlockRows);
    for (int stride = kBlockRows / 2; stride > 0; stride >>= 1) {
        if (rl < stride) {
#pragma unroll
            for (int k = 0; k < 4; ++k) red[k * kBlockRows + rl] += red[k * kBlockRows + rl + stride];
        }
        named_barrier(bar_id, kBlockRows);
    }
    double *out = MEASURE ? p.stats : p.tail_stats;
    if (rl < 4) out[((size_t)bz * row_blocks + rb) * 4 + rl] = red[rl * kBlockRows];
}

}  // namespace fs
