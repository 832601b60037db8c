// Transport application on the sm_100a tensor cores with two 128-row blocks per
// CTA and the plan tile kept in TMEM: out_i = sum_j P_ij V_j at given
// potentials, without forming P ("FlashSinkhorn: IO-aware EOT on GPU",
// Metodologia section 3: plan-weighted averages over the same streamed tiles,
// an attention-style "P V" product).
//
// The arithmetic is that of the one-block kernel (fs_apply_tc.cu): S = Q K^T
// per 128-column tile, p~_ij = P_ij / a_i = 2^(alpha'_i + beta_j + S_ij c)
// split into bf16 hi + lo, O += P~ V~ in TMEM, and at the end out_i = a_i O_i
// (or O_i / sum_j p~_ij) and r_i = a_i sum_j p~_ij.  Two things differ.
//  * Each CTA keeps 256 rows of Q (two blocks) resident, and every K tile and
//    every V~ half it streams serves both blocks: half the L2 -> SM stream of
//    K and V~ per cost entry.
//  * P~ never goes through shared memory.  The softmax warps write it back
//    into the TMEM columns of the S they have just read (hi and lo of a 64-
//    column half in that half's own 64 columns, two bf16 per column), and the
//    P V product takes its A operand from TMEM.  With both operands in shared
//    memory, every MMA of the P V product read 8 KB there and the P~ stores
//    competed with them; that shared-memory traffic, not the tensor pipe, set
//    the pace of the earlier designs.
//
// TMEM (512 columns): block g's S / P~ in [128 g, 128 g + 128), its O in
// [256 + 128 g, 256 + 128 g + dv_pad), so dv <= 128.  Shared memory: Q (both
// blocks), a ring of K slots (one operand atom of a 128-column tile each), a
// ring of V~ halves (64 columns, dv_pad rows per plane), the bias slices.
//
// Warps: 0 streams Q, the K tiles and the bias slices; 10 streams the V~
// halves; 1 allocates TMEM; 1 and 11 issue the MMAs of block 0 and of block 1
// (one thread each); 2..5 and 6..9 are the softmax groups of blocks 0 and 1,
// one warp per TMEM lane quadrant.  Each block's chain runs on its own:
// S_g(t), its softmax, its P V products, and S_g(t + 1) once those have
// completed (its P~ columns are free again); the tensor core interleaves the
// two chains.  A K slot and a V~ half are free once both issuing threads'
// commits after the products that read them have arrived.  (With one issuing
// thread the two chains were serialised through it: a clock64 trace at n = m
// = 65536, d = 128 showed 7900 clk per tile with both S products issued after
// both blocks' P V products, and 6740 with the blocks alternating.)
// Every wait is bounded; on expiry the kernel raises kDevErrTimeout, stops,
// drains its own copies and MMAs, frees TMEM and returns.
#include <cuda_bf16.h>

#include "fs_tc_common.cuh"

namespace fs {
namespace {

using namespace tc;

constexpr int kQ2Threads = 384;
constexpr int kQ2TS = 128;   // columns per tile (N of the S product)
constexpr int kQ2H = 64;     // columns per half (K of one P V product)
constexpr int kQ2Bias = 4;   // bias-slice ring (tiles)
constexpr int kQ2MaxKsteps = 64;

struct Q2Layout {
    uint32_t q, k, v, vstage, bias, koff, rs, bars, misc, total;
};

__host__ __device__ inline int q2swz(int row_bytes) { return row_bytes <= 32 ? 32 : (row_bytes <= 64 ? 64 : 128); }

// V~ stage = [plane 0 (| plane 1)], dv_pad rows of 64 bf16 (128 bytes, 128-byte swizzle).
__host__ __device__ inline Q2Layout q2_layout(int row_bytes, int kslots, int dv_pad, int vpl, int vstages,
                                              int qb) {
    Q2Layout L;
    const uint32_t swz = (uint32_t)q2swz(row_bytes);
    L.q = 0;
    L.k = L.q + (uint32_t)qb * kBlockRows * (uint32_t)row_bytes;
    L.v = L.k + (uint32_t)kslots * kQ2TS * swz;
    L.vstage = (uint32_t)vpl * dv_pad * 128;
    L.bias = L.v + (uint32_t)vstages * L.vstage;
    L.koff = L.bias + kQ2Bias * kQ2TS * 4;
    L.rs = L.koff + 3 * kQ2MaxKsteps * 4;  // one row block: group 1's row sums for group 0
    L.bars = L.rs + (qb == 1 ? kBlockRows * 4 : 0);
    L.misc = L.bars + (2 * kslots + 2 * kQ2Bias + 2 * vstages + 10) * 8;
    L.total = L.misc + 16;
    return L;
}

// PKS > 0: the K-step count of an operand plane, fixed at compile time (the S
// products are issued with immediate descriptor offsets); PKS = 0: any width.
// QB = 2: two row blocks, group g (and issuing thread g) owns block g and every
// tile.  QB = 1: one row block shared by both groups; group g takes the tiles of
// parity g into its own S / P~ columns and its own O, and group 0 adds the two O
// at the end.  TAIL (QB = 1): CTA x takes column part x % tail_k of row block
// main_blocks + x / tail_k and leaves its raw sums for the merge kernel.
template <int KIND, int NPASS, int VPL, int PKS, int QB, bool TAIL>
__global__ void __launch_bounds__(kQ2Threads, 1)
    apply_q2_kernel(const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_k,
                    const __grid_constant__ CUtensorMap map_v, const ApplyParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = smem_raw + ((1024u - (saddr(smem_raw) & 1023u)) & 1023u);
    const int KS = p.kslots, NV = p.stages;
    const uint32_t swz = (uint32_t)p.swz;
    const int atoms = p.row_bytes / p.swz;
    const int box_inner = p.swz / (KIND == 1 ? 4 : 2);
    const uint32_t kslot_bytes = (uint32_t)kQ2TS * swz;
    const uint32_t vplane_bytes = (uint32_t)p.dv_pad * 128u;
    const uint32_t qblock_bytes = (uint32_t)kBlockRows * p.row_bytes;
    const Q2Layout L = q2_layout(p.row_bytes, KS, p.dv_pad, VPL, NV, QB);

    uint8_t *sQ = smem + L.q;
    uint8_t *sK = smem + L.k;
    uint8_t *sV = smem + L.v;
    float *sBias = reinterpret_cast<float *>(smem + L.bias);
    uint32_t *koff = reinterpret_cast<uint32_t *>(smem + L.koff);
    float *sRs = reinterpret_cast<float *>(smem + L.rs);
    uint64_t *kfull = reinterpret_cast<uint64_t *>(smem + L.bars);
    uint64_t *kempty = kfull + KS;
    uint64_t *bfull = kempty + KS;
    uint64_t *bempty = bfull + kQ2Bias;
    uint64_t *vfull = bempty + kQ2Bias;  // [NV] V~ half loaded
    uint64_t *vfree = vfull + NV;        // [NV] both blocks' P V products of the half complete
    uint64_t *qfull = vfree + NV;
    uint64_t *sfull = qfull + 1;   // [2] S of block g ready
    uint64_t *pready = sfull + 2;  // [2][2] P~ of block g, half h written to TMEM
    uint64_t *pfree = pready + 4;  // [2] block g's P V products complete: its S / P~ columns are free
    uint64_t *ofull = pfree + 2;
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(smem + L.misc);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + L.misc + 8);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int bz = blockIdx.z;
    const int ntiles = (p.cols + kQ2TS - 1) / kQ2TS;
    // rows [QB 128 rb, QB 128 (rb + 1)) of problem bz over the column tiles [tb, tb + nt)
    const int rb = TAIL ? p.main_blocks + (int)blockIdx.x / p.tail_k : (int)blockIdx.x;
    const int part = TAIL ? (int)blockIdx.x % p.tail_k : 0;
    const int tb = TAIL ? part * ntiles / p.tail_k : 0;
    const int nt = TAIL ? (part + 1) * ntiles / p.tail_k - tb : ntiles;
    const uint32_t tmem_cols = 512u;

    if (threadIdx.x == 0) {
        for (int s = 0; s < KS; ++s) {
            mbar_init(kfull + s, 1);
            mbar_init(kempty + s, QB);  // the S products that read the slot
        }
        for (int j = 0; j < kQ2Bias; ++j) {
            mbar_init(bfull + j, 1);
            mbar_init(bempty + j, 4 * QB);  // the softmax warps that read the slice
        }
        for (int s = 0; s < NV; ++s) {
            mbar_init(vfull + s, 1);
            mbar_init(vfree + s, QB);  // the P V products that read the half
        }
        mbar_init(qfull, 1);
        for (int g = 0; g < 2; ++g) {
            mbar_init(sfull + g, 1);
            mbar_init(pready + 2 * g, 4);
            mbar_init(pready + 2 * g + 1, 4);
            mbar_init(pfree + g, 1);
        }
        mbar_init(ofull, 2);  // both issuing threads' last commits
        if constexpr (PKS == 0) {  // descriptor offsets of the S products' K steps, for any width
            const uint32_t plane = (uint32_t)p.plane_bytes;
            const int ksteps = (int)(plane / 32u);
            for (int i = 0; i < NPASS * ksteps; ++i) {
                const int pass = i / ksteps, k = i % ksteps;
                const uint32_t ao = (pass == 1 ? plane : 0u) + 32u * k;
                const uint32_t bo = (pass == 2 ? plane : 0u) + 32u * k;
                koff[i] = ((ao / swz) * (kBlockRows * swz) + ao % swz) >> 4;
                koff[kQ2MaxKsteps + i] = bo / swz;
                koff[2 * kQ2MaxKsteps + i] = (bo % swz) >> 4;
            }
        }
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

    if (warp == 0) {
        // ---------------- TMA producer: Q (both blocks), K tiles, bias slices ----------------
        if (lane == 0) {
            bool ok = true;
            int k_issued = 0, b_issued = 0;
            mbar_expect_tx(qfull, (uint32_t)QB * qblock_bytes);
            for (int g = 0; g < QB; ++g)
                for (int a = 0; a < atoms; ++a)
                    tma_load_2d(saddr(sQ) + g * qblock_bytes + a * kBlockRows * swz, &map_q, saddr(qfull),
                                a * box_inner, bz * p.rows_pad + rb * QB * kBlockRows + g * kBlockRows);
            for (int t = 0; ok && t < nt; ++t) {
                const int col0 = (tb + t) * kQ2TS;
                if (*abort_flag) break;
                for (int a = 0; a < atoms && ok; ++a) {
                    const int i = t * atoms + a, s = i % KS;
                    if (i >= KS && !mbar_wait(kempty + s, ((uint32_t)(i / KS) & 1u) ^ 1u, p.timeout_ns)) {
                        ok = false;
                        break;
                    }
                    mbar_expect_tx(kfull + s, kslot_bytes);
                    tma_load_2d(saddr(sK + (size_t)s * kslot_bytes), &map_k, saddr(kfull + s), a * box_inner,
                                bz * p.cols_rows + col0);
                    k_issued = i + 1;
                }
                if (!ok) break;
                const int j = t % kQ2Bias;
                if (t >= kQ2Bias && !mbar_wait(bempty + j, ((uint32_t)(t / kQ2Bias) & 1u) ^ 1u, p.timeout_ns)) {
                    ok = false;
                    break;
                }
                mbar_expect_tx(bfull + j, kQ2TS * 4);
                bulk_load(saddr(sBias + j * kQ2TS), p.col_bias + (size_t)bz * p.cols_stride + col0, kQ2TS * 4,
                          saddr(bfull + j));
                b_issued = t + 1;
            }
            if (!ok) {
                atomicOr(p.err, kDevErrTimeout);
                *abort_flag = 1;
            }
            // never leave with copies in flight
            mbar_wait(qfull, 0, p.timeout_ns);
            for (int i = max(0, k_issued - KS); i < k_issued; ++i)
                mbar_wait(kfull + (i % KS), (uint32_t)(i / KS) & 1u, p.timeout_ns);
            for (int t = max(0, b_issued - kQ2Bias); t < b_issued; ++t)
                mbar_wait(bfull + (t % kQ2Bias), (uint32_t)(t / kQ2Bias) & 1u, p.timeout_ns);
        }
        __syncwarp();
    } else if (warp == 10) {
        // ---------------- TMA producer: V~ halves ----------------
        if (lane == 0) {
            bool ok = true;
            int v_issued = 0;
            for (int hh = 0; ok && hh < 2 * nt; ++hh) {
                if (*abort_flag) break;
                const int s = hh % NV;
                if (hh >= NV && !mbar_wait(vfree + s, ((uint32_t)(hh / NV) & 1u) ^ 1u, p.timeout_ns)) {
                    ok = false;
                    break;
                }
                uint8_t *sv = sV + (size_t)s * L.vstage;
                mbar_expect_tx(vfull + s, (uint32_t)VPL * vplane_bytes);
                for (int pl = 0; pl < VPL; ++pl)
                    tma_load_2d(saddr(sv + pl * vplane_bytes), &map_v, saddr(vfull + s), (2 * tb + hh) * kQ2H,
                                (bz * VPL + pl) * p.dv_pad);
                v_issued = hh + 1;
            }
            if (!ok) {
                atomicOr(p.err, kDevErrTimeout);
                *abort_flag = 1;
            }
            for (int i = max(0, v_issued - NV); i < v_issued; ++i)
                mbar_wait(vfull + (i % NV), (uint32_t)(i / NV) & 1u, p.timeout_ns);
        }
        __syncwarp();
    } else if (warp == 1 || warp == 11) {
        // ---------------- MMA issuers: warp 1 for group 0, warp 11 for group 1 ----------------
        if (lane == 0) {
            const int g = warp == 1 ? 0 : 1;
            // this group's tiles: every tile of its own block (QB = 2), or the tiles of parity g
            const int t_first = QB == 2 ? 0 : g, t_step = QB == 2 ? 1 : 2;
            const uint32_t idesc_s = make_idesc<KIND, kBlockRows, kQ2TS>();
            // P~ V~: bf16 x bf16 -> fp32, M = 128, N = dv_pad, A from TMEM
            const uint32_t idesc_o = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(p.dv_pad >> 3) << 17) |
                                     ((uint32_t)(kBlockRows >> 4) << 24);
            const int nk = NPASS * (p.plane_bytes / 32);
            const uint64_t adesc = make_sdesc(saddr(sQ) + (QB == 2 ? g : 0) * qblock_bytes, swz);
            // S_g(t) = Q_g K(t)^T into block g's columns
            auto s_product = [&](const uint64_t (&bdesc)[4]) {
                const uint32_t dt = tmem_base + (uint32_t)(g * kQ2TS);
                if constexpr (PKS > 0) {
                    issue_s_tile<KIND, NPASS, PKS, kBlockRows>(dt, adesc, bdesc, idesc_s);
                } else {
                    for (int i = 0; i < nk; ++i) {
                        const uint32_t ba = koff[kQ2MaxKsteps + i];
                        const uint64_t bd =
                            ba == 0 ? bdesc[0] : (ba == 1 ? bdesc[1] : (ba == 2 ? bdesc[2] : bdesc[3]));
                        tc_mma<KIND>(dt, adesc + koff[i], bd + koff[2 * kQ2MaxKsteps + i], idesc_s,
                                     i > 0 ? 1u : 0u);
                    }
                }
                tc_commit(saddr(sfull + g));
            };
            // the descriptors of tile t's K slots, once they have landed
            auto k_tile = [&](const int t, uint64_t (&bdesc)[4]) -> bool {
#pragma unroll
                for (int a = 0; a < 4; ++a) {
                    bdesc[a] = 0ull;
                    if (a < atoms) {
                        const int i = t * atoms + a;
                        if (!mbar_wait(kfull + (i % KS), (uint32_t)(i / KS) & 1u, p.timeout_ns)) return false;
                        bdesc[a] = make_sdesc(saddr(sK + (size_t)(i % KS) * kslot_bytes), swz);
                    }
                }
                return true;
            };
            // O_g += P~_g(t, h) V~(t, h): 4 K steps of 16 (8 TMEM columns of bf16 pairs each),
            // hi.hi + lo.hi (+ hi.lo); every offset and accumulate flag an immediate
            auto pv_half = [&](const uint32_t vs, const int h, const uint32_t first) {
                const uint32_t to = tmem_base + 256u + (uint32_t)(g * kQ2TS);
                const uint32_t phi = tmem_base + (uint32_t)(g * kQ2TS + h * kQ2H);
                const uint32_t plo = phi + 32u;
                const uint64_t v0 = make_sdesc(vs, 128u);
                const uint64_t v1 = make_sdesc(vs + (VPL - 1) * vplane_bytes, 128u);
#pragma unroll
                for (int ks = 0; ks < kQ2H / 16; ++ks) {
                    tc_mma_ts(to, phi + 8u * ks, v0 + 2u * ks, idesc_o, ks == 0 ? first : 1u);
                    tc_mma_ts(to, plo + 8u * ks, v0 + 2u * ks, idesc_o, 1u);
                    if (VPL == 2) tc_mma_ts(to, phi + 8u * ks, v1 + 2u * ks, idesc_o, 1u);
                }
            };
            bool ok = mbar_wait(qfull, 0, p.timeout_ns);
            tc_fence_after();
            if (QB == 2 || t_first < nt) {
                uint64_t bdesc[4];
                ok = ok && k_tile(t_first, bdesc);
                if (ok) {
                    s_product(bdesc);
                    for (int a = 0; a < atoms; ++a) tc_commit(saddr(kempty + ((t_first * atoms + a) % KS)));
                }
            }
            for (int t = t_first; ok && t < nt; t += t_step) {
                // barrier phases count this group's tiles (t = g + 2 i with one row block)
                const uint32_t tp = (uint32_t)(QB == 2 ? t : t >> 1) & 1u;
                for (int h = 0; h < 2; ++h) {  // O_g += P~_g(t) V~(t)
                    const int hh = 2 * t + h, s = hh % NV;
                    if (!mbar_wait(pready + 2 * g + h, tp, p.timeout_ns) ||
                        !mbar_wait(vfull + s, (uint32_t)(hh / NV) & 1u, p.timeout_ns) || *abort_flag) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t vs = saddr(sV + (size_t)s * L.vstage);
                    if (t == t_first && h == 0)
                        pv_half(vs, h, 0u);
                    else
                        pv_half(vs, h, 1u);
                    tc_commit(saddr(vfree + s));
                }
                if (!ok) break;
                tc_commit(saddr(pfree + g));
                const int tn = t + t_step;
                if (tn >= nt) break;
                // this group's next S as soon as its P~ columns are free again
                uint64_t bdesc[4];
                if (!k_tile(tn, bdesc) || !mbar_wait(pfree + g, tp, p.timeout_ns) || *abort_flag) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                s_product(bdesc);
                for (int a = 0; a < atoms; ++a) tc_commit(saddr(kempty + ((tn * atoms + a) % KS)));
            }
            if (!ok) {
                atomicOr(p.err, kDevErrTimeout);
                *abort_flag = 1;
            }
            tc_commit(saddr(ofull));  // completes when every MMA issued here has
            mbar_wait(ofull, 0, p.timeout_ns);
        }
        __syncwarp();
    } else if (warp >= 2 && warp < 10) {
        // ---------------- softmax groups: group g owns row block g ----------------
        const int q = warp & 3;
        const int grp = (warp - 2) >> 2;
        const int rl = q * 32 + lane;
        const int row = rb * QB * kBlockRows + (QB == 2 ? grp : 0) * kBlockRows + rl;
        const bool valid = row < p.rows;
        const size_t prow = (size_t)bz * p.rows_stride + row;
        const float alpha = valid ? (float)(((double)p.pot_row[(size_t)bz * p.rows + row] - (double)p.row_norm[prow]) *
                                            p.scale)
                                  : -INFINITY;
        const float c = (float)(p.scale * (double)p.sscale);
        const uint64_t cc = pack2(c, c), aa = pack2(alpha, alpha);
        const uint32_t lane_base = tmem_base + ((uint32_t)(q * 32) << 16);
        float rs = 0.f;
        bool ok = true;
        for (int t = QB == 2 ? 0 : grp; ok && t < nt; t += (QB == 2 ? 1 : 2)) {
            const int j = t % kQ2Bias;
            if (!mbar_wait(sfull + grp, (uint32_t)(QB == 2 ? t : t >> 1) & 1u, p.timeout_ns) ||
                !mbar_wait(bfull + j, (uint32_t)(t / kQ2Bias) & 1u, p.timeout_ns)) {
                ok = false;
                break;
            }
            tc_fence_after();
#pragma unroll 1
            for (int h = 0; h < 2; ++h) {
                const uint32_t tcol = lane_base + (uint32_t)(grp * kQ2TS + h * kQ2H);
                uint32_t r[kQ2H];
                tmem_ld32(tcol, &r[0]);
                tmem_ld32(tcol + 32u, &r[32]);
                tmem_ld_wait();
                const float4 *bq = reinterpret_cast<const float4 *>(sBias + j * kQ2TS + h * kQ2H);
                uint32_t hi[kQ2H / 2], lo[kQ2H / 2];
                uint64_t acc2 = 0ull;
#pragma unroll
                for (int k = 0; k < kQ2H; k += 4) {
                    const float4 bb = bq[k / 4];
                    float e0, e1, e2, e3;
                    unpack2(add2(fma2(pack2(__uint_as_float(r[k]), __uint_as_float(r[k + 1])), cc, pack2(bb.x, bb.y)),
                                 aa),
                            e0, e1);
                    unpack2(add2(fma2(pack2(__uint_as_float(r[k + 2]), __uint_as_float(r[k + 3])), cc,
                                      pack2(bb.z, bb.w)),
                                 aa),
                            e2, e3);
                    e0 = ex2_approx(e0);
                    e1 = ex2_approx(e1);
                    e2 = ex2_approx(e2);
                    e3 = ex2_approx(e3);
                    acc2 = add2(acc2, add2(pack2(e0, e1), pack2(e2, e3)));
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
                float s0, s1;
                unpack2(acc2, s0, s1);
                rs += s0 + s1;
                // P~ of this half over the S columns just read: hi in the first 32, lo in the next 32
                tmem_st32(tcol, hi);
                tmem_st32(tcol + 32u, lo);
                tmem_st_wait();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(pready + 2 * grp + h);
            }
            if (lane == 0) mbar_arrive(bempty + j);
            if (*abort_flag) break;
        }
        if (!ok) {
            atomicOr(p.err, kDevErrTimeout);
            *abort_flag = 1;
        }
        if constexpr (QB == 1) {  // one row block: group 0 adds group 1's row sums and O
            if (grp == 1) sRs[rl] = rs;
            asm volatile("bar.sync 1, 256;" ::: "memory");
            if (grp == 0) {
                rs += sRs[rl];
                const bool done = mbar_wait(ofull, 0, p.timeout_ns) && !*abort_flag;
                tc_fence_after();
                const float a_i = valid ? (float)exp2((double)p.row_logw2[prow]) : 0.f;
                if constexpr (TAIL) {  // the raw sums of this column part (two tiles or more), for the merge
                    const uint32_t to = lane_base + 256u;
                    const size_t tail_rows = (size_t)(gridDim.x / p.tail_k) * kBlockRows;
                    const size_t slot = (size_t)part * tail_rows + (size_t)(blockIdx.x / p.tail_k) * kBlockRows + rl;
                    for (int c0 = 0; c0 < p.dv_pad; c0 += 32) {
                        uint32_t o[32], o1[32];
                        tmem_ld32(to + (uint32_t)c0, o);
                        tmem_ld32(to + (uint32_t)kQ2TS + (uint32_t)c0, o1);
                        tmem_ld_wait();
                        if (done && valid)
                            for (int k = 0; k < 32 && c0 + k < p.dv; ++k)
                                p.tail_o[slot * p.dv + c0 + k] = __uint_as_float(o[k]) + __uint_as_float(o1[k]);
                    }
                    if (done && valid) p.tail_rs[slot] = rs;
                } else {
                    const float scale_o = p.divide ? 1.f / rs : a_i;
                    const uint32_t to = lane_base + 256u;
                    const bool both = nt > 1;  // group 1's O holds at least one tile
                    for (int c0 = 0; c0 < p.dv_pad; c0 += 32) {
                        uint32_t o[32], o1[32];
                        tmem_ld32(to + (uint32_t)c0, o);
                        if (both) tmem_ld32(to + (uint32_t)kQ2TS + (uint32_t)c0, o1);
                        tmem_ld_wait();
                        if (done && valid)
                            for (int k = 0; k < 32 && c0 + k < p.dv; ++k)
                                p.out[((size_t)bz * p.rows + row) * p.dv + c0 + k] =
                                    (both ? __uint_as_float(o[k]) + __uint_as_float(o1[k]) : __uint_as_float(o[k])) *
                                    scale_o;
                    }
                    if (done && valid && p.rsum) p.rsum[(size_t)bz * p.rows + row] = a_i * rs;
                }
            }
        } else {
            const bool done = mbar_wait(ofull, 0, p.timeout_ns) && !*abort_flag;
            tc_fence_after();
            const float a_i = valid ? (float)exp2((double)p.row_logw2[prow]) : 0.f;
            const float scale_o = p.divide ? 1.f / rs : a_i;
            const uint32_t to = lane_base + 256u + (uint32_t)(grp * kQ2TS);
            for (int c0 = 0; c0 < p.dv_pad; c0 += 32) {
                uint32_t o[32];
                tmem_ld32(to + (uint32_t)c0, o);
                tmem_ld_wait();
                if (done && valid)
                    for (int k = 0; k < 32 && c0 + k < p.dv; ++k)
                        p.out[((size_t)bz * p.rows + row) * p.dv + c0 + k] = __uint_as_float(o[k]) * scale_o;
            }
            if (done && valid && p.rsum) p.rsum[(size_t)bz * p.rows + row] = a_i * rs;
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

// The rows of the split row blocks (batch 1): out_i = (sum over the parts of
// their raw O_i) times 1 / r~_i (barycentric map) or a_i, and rsum_i = a_i r~_i,
// r~_i = the sum over the parts of sum_j p~_ij.  One warp per row.
__global__ void tail_merge_kernel(const ApplyParams p, int tail_rows) {
    if (*p.err & kDevErrTimeout) return;  // a part gave up: its sums were never written
    const int i = (int)((blockIdx.x * blockDim.x + threadIdx.x) >> 5), lane = threadIdx.x & 31;
    if (i >= tail_rows) return;
    const int row = p.main_blocks * kBlockRows + i;
    if (row >= p.rows) return;
    float rs = 0.f;
    for (int part = 0; part < p.tail_k; ++part) rs += p.tail_rs[(size_t)part * tail_rows + i];
    const float a_i = (float)exp2((double)p.row_logw2[row]);
    const float scale_o = p.divide ? 1.f / rs : a_i;
    for (int k = lane; k < p.dv; k += 32) {
        float o = 0.f;
        for (int part = 0; part < p.tail_k; ++part) o += p.tail_o[((size_t)part * tail_rows + i) * p.dv + k];
        p.out[(size_t)row * p.dv + k] = o * scale_o;
    }
    if (lane == 0 && p.rsum) p.rsum[row] = a_i * rs;
}

template <int KIND, int NPASS, int VPL, int PKS, int QB, bool TAIL>
cudaError_t launch_q2_one(const ApplyParams &p, int batch, const void *mq, const void *mk, const void *mv,
                          size_t smem, cudaStream_t s) {
    const int blocks = (p.rows_pad + QB * kBlockRows - 1) / (QB * kBlockRows);
    // one row block per CTA: the whole row blocks, or the split ones' column parts
    dim3 grid(QB == 2 ? blocks : (TAIL ? (blocks - p.main_blocks) * p.tail_k : p.main_blocks), 1, batch);
    auto kern = apply_q2_kernel<KIND, NPASS, VPL, PKS, QB, TAIL>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    kern<<<grid, kQ2Threads, smem, s>>>(*static_cast<const CUtensorMap *>(mq), *static_cast<const CUtensorMap *>(mk),
                                        *static_cast<const CUtensorMap *>(mv), p);
    return cudaGetLastError();
}

template <int KIND, int NPASS, int PKS>
cudaError_t launch_q2_ks(const ApplyParams &p, int batch, int vpl, int qb, const void *mq, const void *mk,
                         const void *mv, size_t smem, cudaStream_t s) {
    if (qb == 1) {
        // the whole row blocks, then the split ones' column parts
        cudaError_t e = cudaSuccess;
        if (p.main_blocks > 0)
            e = vpl == 1 ? launch_q2_one<KIND, NPASS, 1, PKS, 1, false>(p, batch, mq, mk, mv, smem, s)
                         : launch_q2_one<KIND, NPASS, 2, PKS, 1, false>(p, batch, mq, mk, mv, smem, s);
        if (e != cudaSuccess || p.tail_k == 1) return e;
        return vpl == 1 ? launch_q2_one<KIND, NPASS, 1, PKS, 1, true>(p, batch, mq, mk, mv, smem, s)
                        : launch_q2_one<KIND, NPASS, 2, PKS, 1, true>(p, batch, mq, mk, mv, smem, s);
    }
    return vpl == 1 ? launch_q2_one<KIND, NPASS, 1, PKS, 2, false>(p, batch, mq, mk, mv, smem, s)
                    : launch_q2_one<KIND, NPASS, 2, PKS, 2, false>(p, batch, mq, mk, mv, smem, s);
}

template <int NPASS, int KS>
bool q2_fits(const ApplyParams &p) {
    return p.row_bytes == RowGeom<NPASS, KS>::kRowBytes && p.swz == RowGeom<NPASS, KS>::kSwz;
}

// The usual plane widths (d = 16, 32, 64 and, one-plane modes, 128 values)
// take the S products with compile-time offsets; others the table.
template <int KIND, int NPASS>
cudaError_t launch_q2_kind(const ApplyParams &p, int batch, int vpl, int qb, const void *mq, const void *mk,
                           const void *mv,
                           size_t smem, cudaStream_t s) {
    const int ks = p.plane_bytes / 32;
    if (ks * 32 == p.plane_bytes) {
        if (ks == 1 && q2_fits<NPASS, 1>(p)) return launch_q2_ks<KIND, NPASS, 1>(p, batch, vpl, qb, mq, mk, mv, smem, s);
        if (ks == 2 && q2_fits<NPASS, 2>(p)) return launch_q2_ks<KIND, NPASS, 2>(p, batch, vpl, qb, mq, mk, mv, smem, s);
        if (ks == 4 && q2_fits<NPASS, 4>(p)) return launch_q2_ks<KIND, NPASS, 4>(p, batch, vpl, qb, mq, mk, mv, smem, s);
        if constexpr (NPASS == 1)
            if (ks == 8 && q2_fits<NPASS, 8>(p))
                return launch_q2_ks<KIND, NPASS, 8>(p, batch, vpl, qb, mq, mk, mv, smem, s);
    }
    return launch_q2_ks<KIND, NPASS, 0>(p, batch, vpl, qb, mq, mk, mv, smem, s);
}

}  // namespace

// Shared memory of the two-block transport application, its K-ring depth
// (slots of one operand atom of a 128-column tile) and its V~ ring depth (64-
// column halves); 0 if it does not fit or dv_pad exceeds 128 (two O
// accumulators next to the two S / P~ blocks in TMEM).
size_t apply_q2_plan(int row_bytes, int dv_pad, int vpl, int qb, int *kslots, int *stages) {
    const size_t limit = 227 * 1024;
    if (dv_pad < 16 || dv_pad > 128 || dv_pad % 16 != 0 || row_bytes > 256) return 0;
    const int atoms = row_bytes / q2swz(row_bytes);
    // {K slots in atoms, V~ halves}, best first
    const int plans[6][2] = {{2 * atoms, 4}, {2 * atoms, 3}, {atoms, 4}, {atoms, 3}, {2 * atoms, 2}, {atoms, 2}};
    for (const auto &pl : plans) {
        const size_t bytes = (size_t)q2_layout(row_bytes, pl[0], dv_pad, vpl, pl[1], qb).total + 1024;
        if (bytes <= limit) {
            *kslots = pl[0];
            *stages = pl[1];
            return bytes < 120 * 1024 ? 120 * 1024 : bytes;  // one CTA per SM (TMEM)
        }
    }
    return 0;
}

// prec: 1 = bf16, 2 = tf32, 3 = 3xTF32, 4 = 3xF16 (the S product); vpl: planes of V~;
// map_v: V~ with a box of 64 columns x dv_pad rows, 128-byte swizzle.
cudaError_t launch_apply_q2(const ApplyParams &p, int batch, int prec, int vpl, int qb, const void *map_q,
                            const void *map_k, const void *map_v, size_t smem, cudaStream_t s) {
    if (qb != 1 && qb != 2) return cudaErrorInvalidValue;
    const int blocks = p.rows_pad / kBlockRows;
    const bool split = qb == 1 && p.tail_k > 1;
    if (qb == 1 && (p.tail_k < 1 || p.main_blocks < 0 || p.main_blocks > blocks || (split && batch != 1)))
        return cudaErrorInvalidValue;
    cudaError_t e;
    if (prec == 1)
        e = launch_q2_kind<0, 1>(p, batch, vpl, qb, map_q, map_k, map_v, smem, s);
    else if (prec == 2)
        e = launch_q2_kind<1, 1>(p, batch, vpl, qb, map_q, map_k, map_v, smem, s);
    else if (prec == 3)
        e = launch_q2_kind<1, 3>(p, batch, vpl, qb, map_q, map_k, map_v, smem, s);
    else
        e = launch_q2_kind<2, 3>(p, batch, vpl, qb, map_q, map_k, map_v, smem, s);
    if (e != cudaSuccess || !split) return e;
    const int tail_rows = (blocks - p.main_blocks) * kBlockRows;
    tail_merge_kernel<<<(tail_rows * 32 + 255) / 256, 256, 0, s>>>(p, tail_rows);
    return cudaGetLastError();
}

}  // namespace fs
