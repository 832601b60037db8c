// Transport application on the sm_100a tensor cores with two 128-row blocks per
// CTA: out_i = sum_j P_ij V_j at given potentials, without forming P
// ("FlashSinkhorn: IO-aware EOT on GPU", Metodologia section 3: plan-weighted
// averages over the same streamed tiles, an attention-style "P V" product).
//
// The arithmetic is that of the one-block kernel (fs_apply_tc.cu): S = Q K^T
// per 128-column tile, p~_ij = P_ij / a_i = 2^(alpha'_i + beta_j + S_ij c)
// split into bf16 hi + lo planes in shared memory, O += P~ V~ in TMEM, and at
// the end out_i = a_i O_i (or O_i / sum_j p~_ij) and r_i = a_i sum_j p~_ij.
// What changes is the traversal: each CTA keeps 256 rows of Q (two blocks)
// resident, and every K tile and every V~ slice it streams serves both blocks,
// which halves the L2 -> SM stream of K and V~ per cost entry.
//
// TMEM (512 columns): S of block 0 in [0, 128), S of block 1 in [128, 256),
// O of block g in [256 + g dv_pad, 256 + (g + 1) dv_pad), so dv <= 128.
// Shared memory: to hold both blocks' P~ next to Q (64 KB at 256-byte rows),
// a stage is a quarter tile (32 columns): [P~ hi | P~ lo] of block 0 and of
// block 1 (8 KB each, 64-byte rows, 64-byte swizzle) and the 32 columns of
// V~ (dv_pad rows of 64 bytes per plane).  One tcgen05.commit after both
// blocks' P~ V~ products of a quarter frees its stage.
//
// Warps: 0 streams Q, the K tiles and the bias slices; 10 streams the V~
// quarters (its own warp, so a V~ wait never holds back a K tile); 1
// allocates TMEM and issues the MMAs; 2..5 and 6..9 are the softmax groups of
// blocks 0 and 1, one warp per TMEM lane quadrant.
//
// Both groups work on the same tile, so nothing else hides a wait for the
// next S.  The issue order keeps that S ahead of them: the P V products of
// quarters 0 and 1 of tile t - 1 (written first), then both S products of
// tile t (as soon as the groups have read S(t - 1) into registers, half-way
// through that tile), then quarters 2 and 3.  The issuing thread also hands
// tile t's K slots back itself, with a tcgen05.commit after the S products,
// so the ring refills as soon as the tensor core is done with them.
// Every wait is bounded; on expiry the kernel raises kDevErrTimeout, stops,
// drains its own copies and MMAs, frees TMEM and returns.
#include <cuda_bf16.h>

#include "fs_tc_common.cuh"

namespace fs {
namespace {

using namespace tc;

constexpr int kQ2Threads = 352;
constexpr int kQ2TS = 128;   // columns per tile (N of the S product)
constexpr int kQ2Q = 32;     // columns per quarter (K of one P V product)
constexpr int kQ2Bias = 4;   // bias-slice ring (tiles)
constexpr int kQ2MaxKsteps = 64;
constexpr uint32_t kQ2PBytes = kBlockRows * 64;  // one bf16 plane of P~: 128 rows x 32 values

struct Q2Layout {
    uint32_t q, k, st, stage, bias, koff, bars, misc, total;
};

__host__ __device__ inline int q2swz(int row_bytes) { return row_bytes <= 32 ? 32 : (row_bytes <= 64 ? 64 : 128); }

// Stage = [P~ hi, block 0 | P~ lo, block 0 | P~ hi, block 1 | P~ lo, block 1 |
// V~ plane 0 (| V~ plane 1)]; every part is a multiple of 1024 bytes.
__host__ __device__ inline Q2Layout q2_layout(int row_bytes, int kslots, int dv_pad, int vpl, int stages) {
    Q2Layout L;
    const uint32_t swz = (uint32_t)q2swz(row_bytes);
    L.q = 0;
    L.k = L.q + 2u * kBlockRows * (uint32_t)row_bytes;
    L.st = L.k + (uint32_t)kslots * kQ2TS * swz;
    L.stage = 4 * kQ2PBytes + (uint32_t)vpl * dv_pad * 64;
    L.bias = L.st + (uint32_t)stages * L.stage;
    L.koff = L.bias + kQ2Bias * kQ2TS * 4;
    L.bars = L.koff + 3 * kQ2MaxKsteps * 4;
    L.misc = L.bars + (2 * kslots + 2 * kQ2Bias + 3 * stages + 6) * 8;
    L.total = L.misc + 16;
    return L;
}

// PKS > 0: the K-step count of an operand plane, fixed at compile time (the S
// products are issued with immediate descriptor offsets); PKS = 0: any width.
template <int KIND, int NPASS, int VPL, int PKS>
__global__ void __launch_bounds__(kQ2Threads, 1)
    apply_q2_kernel(const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_k,
                    const __grid_constant__ CUtensorMap map_v, const ApplyParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = smem_raw + ((1024u - (saddr(smem_raw) & 1023u)) & 1023u);
    const int KS = p.kslots, NS = p.stages;
    const uint32_t swz = (uint32_t)p.swz;
    const int atoms = p.row_bytes / p.swz;
    const int box_inner = p.swz / (KIND == 1 ? 4 : 2);
    const uint32_t kslot_bytes = (uint32_t)kQ2TS * swz;
    const uint32_t vplane_bytes = (uint32_t)p.dv_pad * 64u;
    const uint32_t qblock_bytes = (uint32_t)kBlockRows * p.row_bytes;
    const Q2Layout L = q2_layout(p.row_bytes, KS, p.dv_pad, VPL, NS);

    uint8_t *sQ = smem + L.q;
    uint8_t *sK = smem + L.k;
    uint8_t *sSt = smem + L.st;
    float *sBias = reinterpret_cast<float *>(smem + L.bias);
    uint32_t *koff = reinterpret_cast<uint32_t *>(smem + L.koff);
    uint64_t *kfull = reinterpret_cast<uint64_t *>(smem + L.bars);
    uint64_t *kempty = kfull + KS;
    uint64_t *bfull = kempty + KS;
    uint64_t *bempty = bfull + kQ2Bias;
    uint64_t *pfull = bempty + kQ2Bias;  // [NS] both blocks' P~ of the stage written
    uint64_t *vfull = pfull + NS;        // [NS] V~ of the stage loaded
    uint64_t *stfree = vfull + NS;       // [NS] the P V products that read the stage are complete
    uint64_t *qfull = stfree + NS;
    uint64_t *sfull = qfull + 1;   // [2] S of block g ready
    uint64_t *sempty = sfull + 2;  // [2] S of block g read out
    uint64_t *ofull = sempty + 2;
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(smem + L.misc);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + L.misc + 8);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int rb = blockIdx.x, bz = blockIdx.z;  // rows [256 rb, 256 rb + 256) of problem bz
    const int ntiles = (p.cols + kQ2TS - 1) / kQ2TS;
    const uint32_t tmem_cols = 512u;

    if (threadIdx.x == 0) {
        for (int s = 0; s < KS; ++s) {
            mbar_init(kfull + s, 1);
            mbar_init(kempty + s, 1);
        }
        for (int j = 0; j < kQ2Bias; ++j) {
            mbar_init(bfull + j, 1);
            mbar_init(bempty + j, 8);  // every softmax warp of both blocks reads each slice
        }
        for (int s = 0; s < NS; ++s) {
            mbar_init(pfull + s, 8);
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

    if (warp == 0) {
        // ---------------- TMA producer: Q (both blocks), K tiles, bias slices ----------------
        if (lane == 0) {
            bool ok = true;
            int k_issued = 0, b_issued = 0;
            mbar_expect_tx(qfull, 2u * qblock_bytes);
            for (int g = 0; g < 2; ++g)
                for (int a = 0; a < atoms; ++a)
                    tma_load_2d(saddr(sQ) + g * qblock_bytes + a * kBlockRows * swz, &map_q, saddr(qfull),
                                a * box_inner, bz * p.rows_pad + rb * 2 * kBlockRows + g * kBlockRows);
            for (int t = 0; ok && t < ntiles; ++t) {
                const int col0 = t * kQ2TS;
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
        // ---------------- TMA producer: V~ quarters ----------------
        if (lane == 0) {
            bool ok = true;
            int v_issued = 0;
            for (int t = 0; ok && t < ntiles; ++t) {
                const int col0 = t * kQ2TS;
                if (*abort_flag) break;
                for (int qq = 0; qq < 4; ++qq) {
                    const int hh = 4 * t + qq, s = hh % NS;
                    if (hh >= NS && !mbar_wait(stfree + s, ((uint32_t)(hh / NS) & 1u) ^ 1u, p.timeout_ns)) {
                        ok = false;
                        break;
                    }
                    uint8_t *sv = sSt + (size_t)s * L.stage + 4 * kQ2PBytes;
                    mbar_expect_tx(vfull + s, (uint32_t)VPL * vplane_bytes);
                    for (int pl = 0; pl < VPL; ++pl)
                        tma_load_2d(saddr(sv + pl * vplane_bytes), &map_v, saddr(vfull + s), col0 + qq * kQ2Q,
                                    (bz * VPL + pl) * p.dv_pad);
                    v_issued = hh + 1;
                }
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
            const uint32_t idesc_s = make_idesc<KIND, kBlockRows, kQ2TS>();
            // P~ V~: bf16 x bf16 -> fp32, M = 128, N = dv_pad
            const uint32_t idesc_o = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(p.dv_pad >> 3) << 17) |
                                     ((uint32_t)(kBlockRows >> 4) << 24);
            const uint32_t plane = (uint32_t)p.plane_bytes;
            const int ksteps = (int)(plane / 32u);
            const int nk = NPASS * ksteps;
            if constexpr (PKS == 0) {
                for (int i = 0; i < nk; ++i) {
                    const int pass = i / ksteps, k = i % ksteps;
                    const uint32_t ao = (pass == 1 ? plane : 0u) + 32u * k;
                    const uint32_t bo = (pass == 2 ? plane : 0u) + 32u * k;
                    koff[i] = ((ao / swz) * (kBlockRows * swz) + ao % swz) >> 4;
                    koff[kQ2MaxKsteps + i] = bo / swz;
                    koff[2 * kQ2MaxKsteps + i] = (bo % swz) >> 4;
                }
            }
            const uint64_t adesc[2] = {make_sdesc(saddr(sQ), swz), make_sdesc(saddr(sQ) + qblock_bytes, swz)};
            bool ok = mbar_wait(qfull, 0, p.timeout_ns);
            tc_fence_after();
            // O_g += P~_g V~ over quarter qq of tile tt (both blocks, one commit)
            auto pv_quarter = [&](const int tt, const int qq) -> bool {
                const int hh = 4 * tt + qq, s = hh % NS;
                const uint32_t ph = (uint32_t)(hh / NS) & 1u;
                if (!mbar_wait(pfull + s, ph, p.timeout_ns) || !mbar_wait(vfull + s, ph, p.timeout_ns)) return false;
                if (*abort_flag) return false;
                tc_fence_after();
                const uint32_t st = saddr(sSt + (size_t)s * L.stage);
                const uint64_t v0 = make_sdesc(st + 4 * kQ2PBytes, 64u);
                const uint64_t v1 = make_sdesc(st + 4 * kQ2PBytes + (VPL - 1) * vplane_bytes, 64u);
                // 16 values = 32 bytes per K step; every offset and accumulate
                // flag an immediate (the kernel's first product starts each O afresh)
                auto pv = [&](const uint32_t first) {
#pragma unroll
                    for (int g = 0; g < 2; ++g) {
                        const uint32_t to = tmem_base + 256u + (uint32_t)(g * p.dv_pad);
                        const uint64_t phi = make_sdesc(st + (2 * g) * kQ2PBytes, 64u);
                        const uint64_t plo = make_sdesc(st + (2 * g + 1) * kQ2PBytes, 64u);
#pragma unroll
                        for (int ks = 0; ks < kQ2Q / 16; ++ks) {
                            tc_mma<0>(to, phi + 2u * ks, v0 + 2u * ks, idesc_o, ks == 0 ? first : 1u);
                            tc_mma<0>(to, plo + 2u * ks, v0 + 2u * ks, idesc_o, 1u);
                            if (VPL == 2) tc_mma<0>(to, phi + 2u * ks, v1 + 2u * ks, idesc_o, 1u);
                        }
                    }
                };
                if (hh == 0)
                    pv(0u);
                else
                    pv(1u);
                tc_commit(saddr(stfree + s));
                return true;
            };
            // S_g(t) = Q_g K(t)^T for both blocks; then tile t's K slots go back to the producer
            auto s_tile = [&](const int t) -> bool {
                uint64_t bdesc[4];
#pragma unroll
                for (int a = 0; a < 4; ++a) {
                    bdesc[a] = 0ull;
                    if (a < atoms) {
                        const int i = t * atoms + a;
                        if (!mbar_wait(kfull + (i % KS), (uint32_t)(i / KS) & 1u, p.timeout_ns)) return false;
                        bdesc[a] = make_sdesc(saddr(sK + (size_t)(i % KS) * kslot_bytes), swz);
                    }
                }
                for (int g = 0; g < 2; ++g) {
                    if (t >= 1 && !mbar_wait(sempty + g, ((uint32_t)t & 1u) ^ 1u, p.timeout_ns)) return false;
                    if (*abort_flag) return false;
                    tc_fence_after();
                    const uint32_t dt = tmem_base + (uint32_t)(g * kQ2TS);
                    if constexpr (PKS > 0) {
                        issue_s_tile<KIND, NPASS, PKS, kBlockRows>(dt, adesc[g], bdesc, idesc_s);
                    } else {
                        for (int i = 0; i < nk; ++i) {
                            const uint32_t ba = koff[kQ2MaxKsteps + i];
                            const uint64_t bd =
                                ba == 0 ? bdesc[0] : (ba == 1 ? bdesc[1] : (ba == 2 ? bdesc[2] : bdesc[3]));
                            tc_mma<KIND>(dt, adesc[g] + koff[i], bd + koff[2 * kQ2MaxKsteps + i], idesc_s,
                                         i > 0 ? 1u : 0u);
                        }
                    }
                    tc_commit(saddr(sfull + g));
                }
                for (int a = 0; a < atoms; ++a) tc_commit(saddr(kempty + ((t * atoms + a) % KS)));
                return true;
            };
            ok = ok && s_tile(0);
            for (int t = 1; ok && t <= ntiles; ++t) {
                ok = pv_quarter(t - 1, 0) && pv_quarter(t - 1, 1);
                if (ok && t < ntiles) ok = s_tile(t);
                ok = ok && pv_quarter(t - 1, 2) && pv_quarter(t - 1, 3);
            }
            if (!ok) {
                atomicOr(p.err, kDevErrTimeout);
                *abort_flag = 1;
            }
            tc_commit(saddr(ofull));  // completes when every MMA issued here has
            mbar_wait(ofull, 0, p.timeout_ns);
        }
        __syncwarp();
    } else {
        // ---------------- softmax groups: group g owns row block g ----------------
        const int q = warp & 3;
        const int grp = (warp - 2) >> 2;
        const int rl = q * 32 + lane;
        const int row = rb * 2 * kBlockRows + grp * kBlockRows + rl;
        const bool valid = row < p.rows;
        const size_t prow = (size_t)bz * p.rows_stride + row;
        const float alpha = valid ? (float)(((double)p.pot_row[(size_t)bz * p.rows + row] - (double)p.row_norm[prow]) *
                                            p.scale)
                                  : -INFINITY;
        const float c = (float)(p.scale * (double)p.sscale);
        const uint64_t cc = pack2(c, c), aa = pack2(alpha, alpha);
        const uint32_t lane_base = tmem_base + ((uint32_t)(q * 32) << 16);
        // this thread's row in a P~ plane: 8-row swizzle atoms of 512 bytes, 64-byte rows
        const uint32_t prow_off = (uint32_t)((rl >> 3) * 512 + (rl & 7) * 64);
        const uint32_t pswz = (uint32_t)((rl >> 1) & 3);
        float rs = 0.f;
        bool ok = true;
        for (int t = 0; ok && t < ntiles; ++t) {
            const int j = t % kQ2Bias;
            if (!mbar_wait(sfull + grp, (uint32_t)t & 1u, p.timeout_ns) ||
                !mbar_wait(bfull + j, (uint32_t)(t / kQ2Bias) & 1u, p.timeout_ns)) {
                ok = false;
                break;
            }
            tc_fence_after();
#pragma unroll 1
            for (int half = 0; ok && half < 2; ++half) {
                uint32_t r[2 * kQ2Q];
                tmem_ld32(lane_base + (uint32_t)(grp * kQ2TS + half * 2 * kQ2Q), &r[0]);
                tmem_ld32(lane_base + (uint32_t)(grp * kQ2TS + half * 2 * kQ2Q + kQ2Q), &r[kQ2Q]);
                tmem_ld_wait();
                if (half == 1) {  // all of S read: the buffer may take the next tile
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(sempty + grp);
                }
#pragma unroll
                for (int qh = 0; qh < 2; ++qh) {
                    const float4 *bq = reinterpret_cast<const float4 *>(sBias + j * kQ2TS + (2 * half + qh) * kQ2Q);
                    uint32_t hi[kQ2Q / 2], lo[kQ2Q / 2];
                    uint64_t acc2 = 0ull;
#pragma unroll
                    for (int k = 0; k < kQ2Q; k += 4) {
                        const float4 bb = bq[k / 4];
                        const int kk = qh * kQ2Q + k;
                        float e0, e1, e2, e3;
                        unpack2(add2(fma2(pack2(__uint_as_float(r[kk]), __uint_as_float(r[kk + 1])), cc,
                                          pack2(bb.x, bb.y)),
                                     aa),
                                e0, e1);
                        unpack2(add2(fma2(pack2(__uint_as_float(r[kk + 2]), __uint_as_float(r[kk + 3])), cc,
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
                    // the stage is free once the P V products that last read it are complete
                    const int hh = 4 * t + 2 * half + qh, s = hh % NS;
                    if (hh >= NS && !mbar_wait(stfree + s, ((uint32_t)(hh / NS) & 1u) ^ 1u, p.timeout_ns)) {
                        ok = false;
                        break;
                    }
                    uint8_t *prow_hi = sSt + (size_t)s * L.stage + (2 * grp) * kQ2PBytes + prow_off;
                    uint8_t *prow_lo = prow_hi + kQ2PBytes;
                    // 64-byte swizzle: 16-byte chunk c of row r sits at chunk c ^ ((r / 2) % 4)
#pragma unroll
                    for (int ch = 0; ch < 4; ++ch) {
                        const uint32_t off = (uint32_t)((ch ^ pswz) << 4);
                        *reinterpret_cast<uint4 *>(prow_hi + off) =
                            make_uint4(hi[4 * ch], hi[4 * ch + 1], hi[4 * ch + 2], hi[4 * ch + 3]);
                        *reinterpret_cast<uint4 *>(prow_lo + off) =
                            make_uint4(lo[4 * ch], lo[4 * ch + 1], lo[4 * ch + 2], lo[4 * ch + 3]);
                    }
                    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // visible to the tensor core
                    __syncwarp();
                    if (lane == 0) mbar_arrive(pfull + s);
                }
            }
            if (!ok) break;
            if (lane == 0) mbar_arrive(bempty + j);
            if (*abort_flag) break;
        }
        if (!ok) {
            atomicOr(p.err, kDevErrTimeout);
            *abort_flag = 1;
        }
        const bool done = mbar_wait(ofull, 0, p.timeout_ns) && !*abort_flag;
        tc_fence_after();
        const float a_i = valid ? (float)exp2((double)p.row_logw2[prow]) : 0.f;
        const float scale_o = p.divide ? 1.f / rs : a_i;
        const uint32_t to = lane_base + 256u + (uint32_t)(grp * p.dv_pad);
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

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(tmem_cols)
                     : "memory");
    }
}

template <int KIND, int NPASS, int VPL, int PKS>
cudaError_t launch_q2_one(const ApplyParams &p, int batch, const void *mq, const void *mk, const void *mv,
                          size_t smem, cudaStream_t s) {
    dim3 grid((p.rows_pad + 2 * kBlockRows - 1) / (2 * kBlockRows), 1, batch);
    auto kern = apply_q2_kernel<KIND, NPASS, VPL, PKS>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    kern<<<grid, kQ2Threads, smem, s>>>(*static_cast<const CUtensorMap *>(mq), *static_cast<const CUtensorMap *>(mk),
                                        *static_cast<const CUtensorMap *>(mv), p);
    return cudaGetLastError();
}

template <int KIND, int NPASS, int PKS>
cudaError_t launch_q2_ks(const ApplyParams &p, int batch, int vpl, const void *mq, const void *mk, const void *mv,
                         size_t smem, cudaStream_t s) {
    return vpl == 1 ? launch_q2_one<KIND, NPASS, 1, PKS>(p, batch, mq, mk, mv, smem, s)
                    : launch_q2_one<KIND, NPASS, 2, PKS>(p, batch, mq, mk, mv, smem, s);
}

template <int NPASS, int KS>
bool q2_fits(const ApplyParams &p) {
    return p.row_bytes == RowGeom<NPASS, KS>::kRowBytes && p.swz == RowGeom<NPASS, KS>::kSwz;
}

// The usual plane widths (d = 16, 32, 64 and, one-plane modes, 128 values)
// take the S products with compile-time offsets; others the table.
template <int KIND, int NPASS>
cudaError_t launch_q2_kind(const ApplyParams &p, int batch, int vpl, const void *mq, const void *mk, const void *mv,
                           size_t smem, cudaStream_t s) {
    const int ks = p.plane_bytes / 32;
    if (ks * 32 == p.plane_bytes) {
        if (ks == 1 && q2_fits<NPASS, 1>(p)) return launch_q2_ks<KIND, NPASS, 1>(p, batch, vpl, mq, mk, mv, smem, s);
        if (ks == 2 && q2_fits<NPASS, 2>(p)) return launch_q2_ks<KIND, NPASS, 2>(p, batch, vpl, mq, mk, mv, smem, s);
        if (ks == 4 && q2_fits<NPASS, 4>(p)) return launch_q2_ks<KIND, NPASS, 4>(p, batch, vpl, mq, mk, mv, smem, s);
        if constexpr (NPASS == 1)
            if (ks == 8 && q2_fits<NPASS, 8>(p))
                return launch_q2_ks<KIND, NPASS, 8>(p, batch, vpl, mq, mk, mv, smem, s);
    }
    return launch_q2_ks<KIND, NPASS, 0>(p, batch, vpl, mq, mk, mv, smem, s);
}

}  // namespace

// Shared memory of the two-block transport application, its K-ring depth
// (slots of one operand atom of a 128-column tile) and its stage count (one
// 32-column quarter of both blocks' P~ and of V~ each); 0 if it does not fit
// or dv_pad exceeds 128 (two O accumulators next to two S buffers in TMEM).
size_t apply_q2_plan(int row_bytes, int dv_pad, int vpl, int *kslots, int *stages) {
    const size_t limit = 227 * 1024;
    if (dv_pad < 16 || dv_pad > 128 || dv_pad % 16 != 0 || row_bytes > 256) return 0;
    const int atoms = row_bytes / q2swz(row_bytes);
    // {K slots in atoms, stages}, best first: three stages before a second K
    // tile (the issuing thread frees a tile's K slots as soon as its S products
    // complete, so one tile of ring already loads a whole tile period ahead;
    // at n = m = 65536, d = 128 this measured 4.20 ms against 4.27 ms for two
    // K tiles and two stages)
    const int plans[6][2] = {{2 * atoms, 3}, {atoms + 1, 3}, {atoms, 3}, {2 * atoms, 2}, {atoms + 1, 2}, {atoms, 2}};
    for (const auto &pl : plans) {
        const size_t bytes = (size_t)q2_layout(row_bytes, pl[0], dv_pad, vpl, pl[1]).total + 1024;
        if (bytes <= limit) {
            *kslots = pl[0];
            *stages = pl[1];
            return bytes < 120 * 1024 ? 120 * 1024 : bytes;  // one CTA per SM (TMEM)
        }
    }
    return 0;
}

// prec: 1 = bf16, 2 = tf32, 3 = 3xTF32, 4 = 3xF16 (the S product); vpl: planes of V~;
// map_v: V~ with a box of 32 columns x dv_pad rows, 64-byte swizzle.
cudaError_t launch_apply_q2(const ApplyParams &p, int batch, int prec, int vpl, const void *map_q, const void *map_k,
                            const void *map_v, size_t smem, cudaStream_t s) {
    if (prec == 1) return launch_q2_kind<0, 1>(p, batch, vpl, map_q, map_k, map_v, smem, s);
    if (prec == 2) return launch_q2_kind<1, 1>(p, batch, vpl, map_q, map_k, map_v, smem, s);
    if (prec == 3) return launch_q2_kind<1, 3>(p, batch, vpl, map_q, map_k, map_v, smem, s);
    return launch_q2_kind<2, 3>(p, batch, vpl, map_q, map_k, map_v, smem, s);
}

}  // namespace fs
