// The transport-matrix term of the streaming Hessian-vector product,
//   MV_i = sum_j P_ij (v_i . y_j) y_j,
// in one pass over the plan ("FlashSinkhorn: IO-aware EOT on GPU", Metodologia
// section 3: the HVP as a sequence of transport-vector and transport-matrix
// products, O((n + m) d) memory).  Written as d transport applications of
// width d (one per column k of y, weighted by v_ik) this term costs d / nq
// full passes; here one pass forms the weight v_i . y_j with a second
// tensor-core score against the same K tile:
//   S  = Q K^T   (the plan's score, the handle's operands),
//   S' = U K^T   (U = the direction V packed as an MMA operand),
//   p~'_ij = p~_ij w_ij,  w_ij = v_i . y_j = S'_ij cw + v_i . t,
//   O' += P~' Y~ (Y~ = Y transposed into bf16 planes),   MV_i = a_i O'_i,
// with p~_ij = P_ij / a_i = 2^(alpha_i + beta_j + S_ij c) as in the transport
// application.  K holds 2 kscale (y - t), so cw = 1 / (2 kscale uscale).
//
// U: for bf16 operands (one plane, exact bf16 clouds) the fp32 direction is
// split into bf16 hi and lo tiles and S' = U_hi K^T + U_lo K^T (UMODE 2); for
// the split modes (3xF16, 3xTF32) U is packed like X, with its own
// power-of-two scale, and S' takes the same three passes as S (UMODE 1).
//
// A job is 64 columns of one 128-column K tile: S and S' of the job land side
// by side in one 128-column TMEM accumulator (two of them, one per softmax
// group; group g takes the g-th half of every tile), O' from column 256.
// Warp roles as in the transport kernel: warp 0 lane 0 streams Q, U, K and
// the bias slices, lane 1 the Y~ halves; warp 1 allocates TMEM and issues the
// MMAs; warps 2..9 are the two softmax groups.  Every wait is bounded.
//
// A batch of independent problems runs as blockIdx.z: problem bz's rows of
// Q and U start at bz rows_pad (U's hi and lo tiles are each batch x rows_pad
// rows), its K rows at bz cols_rows, its Y~ planes at bz vpl dv_pad, its
// centre at bz d.
#include <cuda_bf16.h>

#include "fs_tc_common.cuh"

namespace fs {
namespace {

using namespace tc;

constexpr int kWThreads = 320;
constexpr int kWTS = 128;   // columns per K tile
constexpr int kWJ = 64;     // columns per job
constexpr int kWBias = 2;   // bias-slice ring (tiles)
constexpr uint32_t kWPBytes = kBlockRows * 128;  // one bf16 plane of P~': 128 rows x 64 values

struct WLayout {
    uint32_t q, u, k, st, stage, bias, bars, misc, total;
};

__host__ __device__ inline WLayout w_layout(int row_bytes, int utiles, int kslots, int dv_pad, int vpl, int stages) {
    WLayout L;
    const uint32_t swz = (uint32_t)(row_bytes <= 32 ? 32 : (row_bytes <= 64 ? 64 : 128));
    L.q = 0;
    L.u = L.q + (uint32_t)kBlockRows * row_bytes;
    L.k = L.u + (uint32_t)utiles * kBlockRows * row_bytes;
    L.st = L.k + (uint32_t)kslots * kWTS * swz;
    L.stage = 2 * kWPBytes + (uint32_t)vpl * dv_pad * 128;
    L.bias = L.st + (uint32_t)stages * L.stage;
    L.bars = L.bias + kWBias * kWTS * 4;
    L.misc = L.bars + (2 * kslots + 2 * kWBias + 3 * stages + 6) * 8;
    L.total = L.misc + 16;
    return L;
}

// UMODE 1: U packed like X (utiles = 1); UMODE 2: U = bf16 hi and lo tiles.
template <int KIND, int NPASS, int KS, int UMODE, int VPL>
__global__ void __launch_bounds__(kWThreads, 1)
    hvp_w_kernel(const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_u,
                 const __grid_constant__ CUtensorMap map_k, const __grid_constant__ CUtensorMap map_v,
                 const ApplyParams p, const float cw, const float *__restrict__ dirv,
                 const float *__restrict__ center) {
    using G = RowGeom<NPASS, KS>;
    constexpr int kSwz = G::kSwz, kAtoms = G::kAtoms, kRowBytes = G::kRowBytes;
    constexpr int kUTiles = UMODE == 2 ? 2 : 1;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = smem_raw + ((1024u - (saddr(smem_raw) & 1023u)) & 1023u);
    const int KSL = p.kslots, NS = p.stages;
    const int box_inner = kSwz / (KIND == 1 ? 4 : 2);
    const uint32_t kslot_bytes = (uint32_t)kWTS * kSwz;
    const uint32_t vplane_bytes = (uint32_t)p.dv_pad * 128u;
    const WLayout L = w_layout(kRowBytes, kUTiles, KSL, p.dv_pad, VPL, NS);

    uint8_t *sQ = smem + L.q;
    uint8_t *sU = smem + L.u;
    uint8_t *sK = smem + L.k;
    uint8_t *sSt = smem + L.st;
    float *sBias = reinterpret_cast<float *>(smem + L.bias);
    uint64_t *kfull = reinterpret_cast<uint64_t *>(smem + L.bars);
    uint64_t *kempty = kfull + KSL;
    uint64_t *bfull = kempty + KSL;
    uint64_t *bempty = bfull + kWBias;
    uint64_t *pfull = bempty + kWBias;  // [NS]
    uint64_t *vfull = pfull + NS;       // [NS]
    uint64_t *stfree = vfull + NS;      // [NS]
    uint64_t *qfull = stfree + NS;
    uint64_t *sfull = qfull + 1;   // [2]
    uint64_t *sempty = sfull + 2;  // [2]
    uint64_t *ofull = sempty + 2;
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(smem + L.misc);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + L.misc + 8);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int rb = blockIdx.x, bz = blockIdx.z;
    const int ntiles = (p.cols + kWTS - 1) / kWTS;
    const int njobs = 2 * ntiles;
    const uint32_t tmem_cols = 512u;  // [S | S'] x 2 jobs in [0, 256), O' from 256

    if (threadIdx.x == 0) {
        for (int s = 0; s < KSL; ++s) {
            mbar_init(kfull + s, 1);
            mbar_init(kempty + s, 1);
        }
        for (int j = 0; j < kWBias; ++j) {
            mbar_init(bfull + j, 1);
            mbar_init(bempty + j, 8);  // both groups read every tile's slice
        }
        for (int s = 0; s < NS; ++s) {
            mbar_init(pfull + s, 4);
            mbar_init(vfull + s, 1);
            mbar_init(stfree + s, 1);
        }
        mbar_init(qfull, 1);
        for (int b = 0; b < 2; ++b) {
            mbar_init(sfull + b, 1);
            mbar_init(sempty + b, 4);
        }
        mbar_init(ofull, 1);
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(saddr(tmem_holder)),
                     "r"(tmem_cols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_holder;
    const uint32_t tmem_o = tmem_base + 256u;

    if (warp == 0) {
        // ---------------- TMA producers ----------------
        if (lane == 0) {  // Q, U, K tiles, bias slices
            bool ok = true;
            int k_issued = 0, b_issued = 0;
            mbar_expect_tx(qfull, (uint32_t)(1 + kUTiles) * kBlockRows * kRowBytes);
            for (int a = 0; a < kAtoms; ++a) {
                tma_load_2d(saddr(sQ) + a * kBlockRows * kSwz, &map_q, saddr(qfull), a * box_inner,
                            bz * p.rows_pad + rb * kBlockRows);
                for (int u = 0; u < kUTiles; ++u)
                    tma_load_2d(saddr(sU) + (u * kAtoms + a) * kBlockRows * kSwz, &map_u, saddr(qfull), a * box_inner,
                                (u * (int)gridDim.z + bz) * p.rows_pad + rb * kBlockRows);
            }
            for (int t = 0; ok && t < ntiles; ++t) {
                const int col0 = t * kWTS;
                if (*abort_flag) break;
                for (int a = 0; a < kAtoms && ok; ++a) {
                    const int i = t * kAtoms + a, s = i % KSL;
                    if (i >= KSL && !mbar_wait(kempty + s, ((uint32_t)(i / KSL) & 1u) ^ 1u, p.timeout_ns)) {
                        ok = false;
                        break;
                    }
                    mbar_expect_tx(kfull + s, kslot_bytes);
                    tma_load_2d(saddr(sK + (size_t)s * kslot_bytes), &map_k, saddr(kfull + s), a * box_inner,
                                bz * p.cols_rows + col0);
                    k_issued = i + 1;
                }
                if (!ok) break;
                const int j = t % kWBias;
                if (t >= kWBias && !mbar_wait(bempty + j, ((uint32_t)(t / kWBias) & 1u) ^ 1u, p.timeout_ns)) {
                    ok = false;
                    break;
                }
                mbar_expect_tx(bfull + j, kWTS * 4);
                bulk_load(saddr(sBias + j * kWTS), p.col_bias + (size_t)bz * p.cols_stride + col0, kWTS * 4,
                          saddr(bfull + j));
                b_issued = t + 1;
            }
            if (!ok) {
                atomicOr(p.err, kDevErrTimeout);
                *abort_flag = 1;
            }
            mbar_wait(qfull, 0, p.timeout_ns);
            for (int i = max(0, k_issued - KSL); i < k_issued; ++i)
                mbar_wait(kfull + (i % KSL), (uint32_t)(i / KSL) & 1u, p.timeout_ns);
            for (int t = max(0, b_issued - kWBias); t < b_issued; ++t)
                mbar_wait(bfull + (t % kWBias), (uint32_t)(t / kWBias) & 1u, p.timeout_ns);
        } else if (lane == 1) {  // Y~ of every job
            bool ok = true;
            int v_issued = 0;
            for (int jb = 0; ok && jb < njobs; ++jb) {
                if (*abort_flag) break;
                const int s = jb % NS;
                if (jb >= NS && !mbar_wait(stfree + s, ((uint32_t)(jb / NS) & 1u) ^ 1u, p.timeout_ns)) {
                    ok = false;
                    break;
                }
                uint8_t *sv = sSt + (size_t)s * L.stage + 2 * kWPBytes;
                mbar_expect_tx(vfull + s, (uint32_t)VPL * vplane_bytes);
                for (int pl = 0; pl < VPL; ++pl)
                    tma_load_2d(saddr(sv + pl * vplane_bytes), &map_v, saddr(vfull + s), jb * kWJ,
                                (bz * VPL + pl) * p.dv_pad);
                v_issued = jb + 1;
            }
            if (!ok) {
                atomicOr(p.err, kDevErrTimeout);
                *abort_flag = 1;
            }
            for (int i = max(0, v_issued - NS); i < v_issued; ++i)
                mbar_wait(vfull + (i % NS), (uint32_t)(i / NS) & 1u, p.timeout_ns);
        }
        __syncwarp();
    } else if (warp == 1) {
        // ---------------- MMA issuer ----------------
        if (lane == 0) {
            const uint32_t idesc_s = make_idesc<KIND, kBlockRows, kWJ>();
            const uint32_t idesc_u = make_idesc<UMODE == 2 ? 0 : KIND, kBlockRows, kWJ>();
            const uint32_t idesc_o = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(p.dv_pad >> 3) << 17) |
                                     ((uint32_t)(kBlockRows >> 4) << 24);
            const uint64_t adesc_q = make_sdesc(saddr(sQ), kSwz);
            const uint64_t adesc_u0 = make_sdesc(saddr(sU), kSwz);
            const uint64_t adesc_u1 = make_sdesc(saddr(sU) + kAtoms * kBlockRows * kSwz, kSwz);
            bool ok = mbar_wait(qfull, 0, p.timeout_ns);
            tc_fence_after();
            uint64_t bdesc[4] = {0ull, 0ull, 0ull, 0ull};
            for (int jb = 0; ok && jb <= njobs; ++jb) {
                if (jb < njobs) {  // S and S' of job jb: 64 columns, rows 64 h.. of every K slot
                    const int t = jb >> 1, hf = jb & 1, b = hf;
                    if (jb >= 2 && !mbar_wait(sempty + b, ((uint32_t)(jb >> 1) & 1u) ^ 1u, p.timeout_ns)) {
                        ok = false;
                        break;
                    }
                    if (hf == 0) {
#pragma unroll
                        for (int a = 0; a < kAtoms; ++a) {
                            const int i = t * kAtoms + a;
                            if (!mbar_wait(kfull + (i % KSL), (uint32_t)(i / KSL) & 1u, p.timeout_ns)) ok = false;
                            bdesc[a] = make_sdesc(saddr(sK + (size_t)(i % KSL) * kslot_bytes), kSwz);
                        }
                    }
                    if (!ok || *abort_flag) break;
                    tc_fence_after();
                    uint64_t bdh[4];
#pragma unroll
                    for (int a = 0; a < 4; ++a) bdh[a] = bdesc[a] + (uint64_t)(hf * ((kWJ * kSwz) >> 4));
                    const uint32_t dt = tmem_base + (uint32_t)(b * 2 * kWJ);
                    issue_s_tile<KIND, NPASS, KS, kBlockRows>(dt, adesc_q, bdh, idesc_s);
                    if constexpr (UMODE == 2) {
                        issue_s_tile<0, 1, KS, kBlockRows>(dt + kWJ, adesc_u0, bdh, idesc_u);
                        issue_s_tile<0, 1, KS, kBlockRows, false, true>(dt + kWJ, adesc_u1, bdh, idesc_u);
                    } else {
                        issue_s_tile<KIND, NPASS, KS, kBlockRows>(dt + kWJ, adesc_u0, bdh, idesc_u);
                    }
                    tc_commit(saddr(sfull + b));
                }
                if (jb >= 1) {  // O' += P~' Y~ of job jb - 1
                    const int jj = jb - 1, s = jj % NS;
                    const uint32_t ph = (uint32_t)(jj / NS) & 1u;
                    if (!mbar_wait(pfull + s, ph, p.timeout_ns) || !mbar_wait(vfull + s, ph, p.timeout_ns)) {
                        ok = false;
                        break;
                    }
                    if (*abort_flag) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t st = saddr(sSt + (size_t)s * L.stage);
                    const uint64_t phi = make_sdesc(st, 128u);
                    const uint64_t plo = make_sdesc(st + kWPBytes, 128u);
                    const uint64_t v0 = make_sdesc(st + 2 * kWPBytes, 128u);
                    const uint64_t v1 = make_sdesc(st + 2 * kWPBytes + (VPL - 1) * vplane_bytes, 128u);
                    auto pv = [&](const uint32_t first) {
#pragma unroll
                        for (int ks = 0; ks < kWJ / 16; ++ks) {
                            tc_mma<0>(tmem_o, phi + 2u * ks, v0 + 2u * ks, idesc_o, ks == 0 ? first : 1u);
                            tc_mma<0>(tmem_o, plo + 2u * ks, v0 + 2u * ks, idesc_o, 1u);
                            if (VPL == 2) tc_mma<0>(tmem_o, phi + 2u * ks, v1 + 2u * ks, idesc_o, 1u);
                        }
                    };
                    if (jj == 0)
                        pv(0u);
                    else
                        pv(1u);
                    tc_commit(saddr(stfree + s));
                }
            }
            if (!ok) {
                atomicOr(p.err, kDevErrTimeout);
                *abort_flag = 1;
            }
            tc_commit(saddr(ofull));
            mbar_wait(ofull, 0, p.timeout_ns);
        }
        __syncwarp();
    } else {
        // ---------------- softmax groups: group g takes half g of every tile ----------------
        const int q = warp & 3;
        const int grp = (warp - 2) >> 2;
        const int rl = q * 32 + lane;
        const int row = rb * kBlockRows + rl;
        const bool valid = row < p.rows;
        const size_t grow = (size_t)bz * p.rows + row;         // row in [batch][rows] arrays
        const size_t prow = (size_t)bz * p.rows_stride + row;  // row in the handle's padded per-point arrays
        const float alpha = valid ? (float)(((double)p.pot_row[grow] - (double)p.row_norm[prow]) * p.scale) : -INFINITY;
        const float c = (float)(p.scale * (double)p.sscale);
        // w_ij = S'_ij cw + v_i . t (t: the centre the operands are packed around)
        float bw = 0.f;
        if (valid && center)
            for (int k = 0; k < p.d; ++k) bw = fmaf(dirv[grow * p.d + k], center[(size_t)bz * p.d + k], bw);
        const uint64_t cc = pack2(c, c), aa = pack2(alpha, alpha), cwp = pack2(cw, cw), bwp = pack2(bw, bw);
        const uint32_t lane_base = tmem_base + ((uint32_t)(q * 32) << 16);
        const uint32_t prow_off = (uint32_t)((rl >> 3) * 1024 + (rl & 7) * 128);
        bool ok = true;
        for (int t = 0; ok && t < ntiles; ++t) {
            const int jb = 2 * t + grp, j = t % kWBias;
            if (!mbar_wait(sfull + grp, (uint32_t)t & 1u, p.timeout_ns) ||
                !mbar_wait(bfull + j, (uint32_t)(t / kWBias) & 1u, p.timeout_ns)) {
                ok = false;
                break;
            }
            tc_fence_after();
            if (grp == 1 && q == 2 && lane == 0)  // both jobs of tile t are complete: its K slots are free
                for (int a = 0; a < kAtoms; ++a) mbar_arrive(kempty + ((t * kAtoms + a) % KSL));
            uint32_t r[kWJ], r2[kWJ];
            const uint32_t ta = lane_base + (uint32_t)(grp * 2 * kWJ);
            tmem_ld32(ta + 0u, &r[0]);
            tmem_ld32(ta + 32u, &r[32]);
            tmem_ld32(ta + 64u, &r2[0]);
            tmem_ld32(ta + 96u, &r2[32]);
            tmem_ld_wait();
            tc_fence_before();  // S and S' are in registers: the accumulator may take the next job
            __syncwarp();
            if (lane == 0) mbar_arrive(sempty + grp);
            const float4 *bq = reinterpret_cast<const float4 *>(sBias + j * kWTS + grp * kWJ);
            uint32_t hi[kWJ / 2], lo[kWJ / 2];
#pragma unroll
            for (int k = 0; k < kWJ; k += 4) {
                const float4 bb = bq[k / 4];
                float e0, e1, e2, e3, w0, w1, w2, w3;
                unpack2(add2(fma2(pack2(__uint_as_float(r[k]), __uint_as_float(r[k + 1])), cc, pack2(bb.x, bb.y)), aa),
                        e0, e1);
                unpack2(add2(fma2(pack2(__uint_as_float(r[k + 2]), __uint_as_float(r[k + 3])), cc,
                                  pack2(bb.z, bb.w)),
                             aa),
                        e2, e3);
                unpack2(fma2(pack2(__uint_as_float(r2[k]), __uint_as_float(r2[k + 1])), cwp, bwp), w0, w1);
                unpack2(fma2(pack2(__uint_as_float(r2[k + 2]), __uint_as_float(r2[k + 3])), cwp, bwp), w2, w3);
                e0 = ex2_approx(e0) * w0;
                e1 = ex2_approx(e1) * w1;
                e2 = ex2_approx(e2) * w2;
                e3 = ex2_approx(e3) * w3;
                const __nv_bfloat162 h01 = __floats2bfloat162_rn(e0, e1);
                const __nv_bfloat162 h23 = __floats2bfloat162_rn(e2, e3);
                const float2 f01 = __bfloat1622float2(h01);
                const float2 f23 = __bfloat1622float2(h23);
                const __nv_bfloat162 l01 = __floats2bfloat162_rn(e0 - f01.x, e1 - f01.y);
                const __nv_bfloat162 l23 = __floats2bfloat162_rn(e2 - f23.x, e3 - f23.y);
                hi[k / 2] = *reinterpret_cast<const uint32_t *>(&h01);
                hi[k / 2 + 1] = *reinterpret_cast<const uint32_t *>(&h23);
                lo[k / 2] = *reinterpret_cast<const uint32_t *>(&l01);
                lo[k / 2 + 1] = *reinterpret_cast<const uint32_t *>(&l23);
            }
            const int s = jb % NS;
            if (jb >= NS && !mbar_wait(stfree + s, ((uint32_t)(jb / NS) & 1u) ^ 1u, p.timeout_ns)) {
                ok = false;
                break;
            }
            uint8_t *prow_hi = sSt + (size_t)s * L.stage + prow_off;
            uint8_t *prow_lo = prow_hi + kWPBytes;
#pragma unroll
            for (int ch = 0; ch < 8; ++ch) {
                const uint32_t off = (uint32_t)((ch ^ (rl & 7)) << 4);
                *reinterpret_cast<uint4 *>(prow_hi + off) =
                    make_uint4(hi[4 * ch], hi[4 * ch + 1], hi[4 * ch + 2], hi[4 * ch + 3]);
                *reinterpret_cast<uint4 *>(prow_lo + off) =
                    make_uint4(lo[4 * ch], lo[4 * ch + 1], lo[4 * ch + 2], lo[4 * ch + 3]);
            }
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(pfull + s);
                mbar_arrive(bempty + j);
            }
            if (*abort_flag) break;
        }
        if (!ok) {
            atomicOr(p.err, kDevErrTimeout);
            *abort_flag = 1;
        }
        if (grp == 0) {
            const bool done = mbar_wait(ofull, 0, p.timeout_ns) && !*abort_flag;
            tc_fence_after();
            const float a_i = valid ? (float)exp2((double)p.row_logw2[prow]) : 0.f;
            for (int c0 = 0; c0 < p.dv_pad; c0 += 32) {
                uint32_t o[32];
                tmem_ld32(lane_base + 256u + (uint32_t)c0, o);
                tmem_ld_wait();
                if (done && valid)
                    for (int k = 0; k < 32 && c0 + k < p.dv; ++k)
                        p.out[grow * p.dv + c0 + k] = __uint_as_float(o[k]) * a_i;
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(tmem_cols)
                     : "memory");
    }
}

// U = bf16 hi and lo tiles of the direction V [batch][rows][d]: out[0][bz][r][k] =
// bf16(v), out[1][bz][r][k] = bf16(v - hi), rows r < rows_pad, row_elems per row
// (zero beyond d and rows).
__global__ void u_split_kernel(const float *V, int batch, int rows, int rows_pad, int d, int row_elems,
                               __nv_bfloat16 *out) {
    const size_t total = (size_t)batch * rows_pad * row_elems;
    for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < total; i += (size_t)gridDim.x * blockDim.x) {
        const size_t rr = i / row_elems;
        const int bz = (int)(rr / rows_pad), r = (int)(rr % rows_pad), k = (int)(i % row_elems);
        const float v = (r < rows && k < d) ? V[((size_t)bz * rows + r) * d + k] : 0.f;
        const __nv_bfloat16 h = __float2bfloat16_rn(v);
        out[i] = h;
        out[total + i] = __float2bfloat16_rn(v - __bfloat162float(h));
    }
}

template <int KIND, int NPASS, int KS, int UMODE>
cudaError_t launch_w(const ApplyParams &p, int batch, int vpl, float cw, const float *dirv, const float *center,
                     const void *mq, const void *mu, const void *mk, const void *mv, size_t smem, cudaStream_t s) {
    if (vpl == 1) {
        auto kern = hvp_w_kernel<KIND, NPASS, KS, UMODE, 1>;
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        kern<<<dim3(p.rows_pad / kBlockRows, 1, batch), kWThreads, smem, s>>>(
            *static_cast<const CUtensorMap *>(mq), *static_cast<const CUtensorMap *>(mu),
            *static_cast<const CUtensorMap *>(mk), *static_cast<const CUtensorMap *>(mv), p, cw, dirv, center);
    } else {
        auto kern = hvp_w_kernel<KIND, NPASS, KS, UMODE, 2>;
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        kern<<<dim3(p.rows_pad / kBlockRows, 1, batch), kWThreads, smem, s>>>(
            *static_cast<const CUtensorMap *>(mq), *static_cast<const CUtensorMap *>(mu),
            *static_cast<const CUtensorMap *>(mk), *static_cast<const CUtensorMap *>(mv), p, cw, dirv, center);
    }
    return cudaGetLastError();
}

}  // namespace

// The operand geometries the fused term supports: one bf16 plane of 1, 2, 4 or
// 8 K-steps of 32 bytes, or hi/lo planes (3xF16, 3xTF32) of 1, 2 or 4, in rows of
// at most 256 bytes.  Returns the U mode (1: packed like X, 2: bf16 hi/lo
// tiles) or 0 where the fused term does not apply.
int hvp_w_mode(int prec, int plane_bytes, int row_bytes) {
    if (row_bytes > 256) return 0;
    const int ks = plane_bytes / 32;
    if (ks * 32 != plane_bytes) return 0;
    if (prec == 1) return (ks == 1 || ks == 2 || ks == 4 || ks == 8) ? 2 : 0;   // bf16
    if (prec == 3 || prec == 4) return (ks == 1 || ks == 2 || ks == 4) ? 1 : 0;  // 3xTF32, 3xF16
    return 0;
}

// Shared memory, K-ring depth and stage count of the fused term (0 if it does not fit).
size_t hvp_w_plan(int row_bytes, int umode, int dv_pad, int vpl, int *kslots, int *stages) {
    const size_t limit = 227 * 1024;
    const int swz = row_bytes <= 32 ? 32 : (row_bytes <= 64 ? 64 : 128);
    const int atoms = row_bytes / swz;
    const int utiles = umode == 2 ? 2 : 1;
    const int plans[4][2] = {{2, 3}, {1, 3}, {2, 2}, {1, 2}};  // {K tiles, stages}, best first
    for (const auto &pl : plans) {
        const size_t bytes = (size_t)w_layout(row_bytes, utiles, pl[0] * atoms, dv_pad, vpl, pl[1]).total + 1024;
        if (bytes <= limit) {
            *kslots = pl[0] * atoms;
            *stages = pl[1];
            return bytes < 120 * 1024 ? 120 * 1024 : bytes;
        }
    }
    return 0;
}

cudaError_t launch_u_split(const float *V, int batch, int rows, int rows_pad, int d, int row_elems, void *out,
                           cudaStream_t s) {
    const size_t total = (size_t)batch * rows_pad * row_elems;
    size_t g = (total + 255) / 256;
    if (g > 148 * 16) g = 148 * 16;
    u_split_kernel<<<(unsigned)g, 256, 0, s>>>(V, batch, rows, rows_pad, d, row_elems,
                                               static_cast<__nv_bfloat16 *>(out));
    return cudaGetLastError();
}

// prec: 1 = bf16 (umode 2), 3 = 3xTF32, 4 = 3xF16 (umode 1); p: the application's
// parameters in the f direction, p.dv = d, p.out = MV [batch][n][d].
cudaError_t launch_hvp_w(const ApplyParams &p, int batch, int prec, int umode, int vpl, float cw, const float *dirv,
                         const float *center, const void *map_q, const void *map_u, const void *map_k,
                         const void *map_v, size_t smem, cudaStream_t s) {
    const int ks = p.plane_bytes / 32;
    if (prec == 1 && umode == 2) {
        if (ks == 1) return launch_w<0, 1, 1, 2>(p, batch, vpl, cw, dirv, center, map_q, map_u, map_k, map_v, smem, s);
        if (ks == 2) return launch_w<0, 1, 2, 2>(p, batch, vpl, cw, dirv, center, map_q, map_u, map_k, map_v, smem, s);
        if (ks == 4) return launch_w<0, 1, 4, 2>(p, batch, vpl, cw, dirv, center, map_q, map_u, map_k, map_v, smem, s);
        if (ks == 8) return launch_w<0, 1, 8, 2>(p, batch, vpl, cw, dirv, center, map_q, map_u, map_k, map_v, smem, s);
    } else if (prec == 4 && umode == 1) {
        if (ks == 1) return launch_w<2, 3, 1, 1>(p, batch, vpl, cw, dirv, center, map_q, map_u, map_k, map_v, smem, s);
        if (ks == 2) return launch_w<2, 3, 2, 1>(p, batch, vpl, cw, dirv, center, map_q, map_u, map_k, map_v, smem, s);
        if (ks == 4) return launch_w<2, 3, 4, 1>(p, batch, vpl, cw, dirv, center, map_q, map_u, map_k, map_v, smem, s);
    } else if (prec == 3 && umode == 1) {
        if (ks == 1) return launch_w<1, 3, 1, 1>(p, batch, vpl, cw, dirv, center, map_q, map_u, map_k, map_v, smem, s);
        if (ks == 2) return launch_w<1, 3, 2, 1>(p, batch, vpl, cw, dirv, center, map_q, map_u, map_k, map_v, smem, s);
        if (ks == 4) return launch_w<1, 3, 4, 1>(p, batch, vpl, cw, dirv, center, map_q, map_u, map_k, map_v, smem, s);
    }
    return cudaErrorInvalidValue;
}

}  // namespace fs
