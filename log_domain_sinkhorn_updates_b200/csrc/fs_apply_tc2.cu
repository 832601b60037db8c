// Transport application on CTA pairs: out_i = sum_j P_ij V_j, as in
// fs_apply_tc.cu ("FlashSinkhorn: IO-aware EOT on GPU", Metodologia section 3:
// plan-weighted averages over streamed tiles, without forming P), with every
// MMA spanning the two SMs of a cluster (tcgen05.mma.cta_group::2, M = 256).
//
// Each CTA keeps its own 128 rows of Q.  Of every 128-column tile it loads only
// half of K (64 points) and, of every 64-column half of V~, only half of the
// output columns (dv_pad / 2 rows of V~):
//   S  = Q K^T     M = 256 (128 rows per CTA), N = 128: B rows 0..63 from the
//                  first CTA's shared memory, 64..127 from the second's;
//   O += P~ V~     M = 256, N = dv_pad: A = each CTA's own P~ stage, B = the
//                  two halves of V~.
// So each SM streams half the bytes of K and V~ from L2 that the one-CTA
// kernel does, and a CTA needs half the shared memory per tile, which lets the
// 512-byte operand rows (fp32 clouds at d = 128 in 3xF16 or TF32, 3xTF32 at
// d = 64) run on the tensor cores too.
//
// Roles and data flow are those of the one-CTA kernel (warp 0 the Q / K / bias
// producer, warp 10 the V~ producer, warp 1 TMEM allocator and, in the pair's
// first CTA, MMA issuer, warps 2..9 two softmax groups taking the even and the
// odd tiles).  The V~ producer has a warp of its own: sharing warp 0 with the
// K producer measured 1 % slower at n = m = 65536, d = 128.  Synchronisation
// of the pair:
//  * the TMA copies of both CTAs (Q, K halves, V~ halves) count on the first
//    CTA's barriers, where the MMA issuer waits;
//  * every MMA completion is committed to both CTAs at once (multicast commit):
//    S ready, a stage's P~ V~ product done, the end of the stream;
//  * both CTAs' softmax warps hand an S buffer back, and publish a stage's
//    P~, on the first CTA's barriers (the P~ with a cluster-scope release after
//    the async-proxy fence, since the peer's tensor-core instructions read it);
//  * each CTA frees its own K slots and bias slices.
// Every wait is bounded; both CTAs always reach the final cluster barrier, so
// neither leaves while the pair's MMAs or the peer may still use its memory.
#include <cuda_bf16.h>

#include "fs_tc_common.cuh"

namespace fs {
namespace {

using namespace tc;

constexpr int kP2Threads = 352;
constexpr int kP2TS = 128;          // columns per tile (N of the S product)
constexpr int kP2KRows = 64;        // K rows of a tile held by each CTA
constexpr int kP2TH = 64;           // columns per half (K of one P V product)
constexpr int kP2MaxKsteps = 64;
constexpr int kP2Bias = 4;          // bias-slice ring (tiles)
constexpr uint32_t kP2PBytes = kBlockRows * 128;  // one bf16 plane of P~: 128 rows x 64 values

struct P2Layout {
    uint32_t q, k, st, stage, vhalf, bias, koff, rs, bars, misc, total;
};

__host__ __device__ inline int p2swz(int row_bytes) { return row_bytes <= 32 ? 32 : (row_bytes <= 64 ? 64 : 128); }

// Stage = [P~ hi | P~ lo | V~ plane 0 half (| V~ plane 1 half)]; each part is a
// multiple of 1024 bytes (dv_pad is a multiple of 32).
__host__ __device__ inline P2Layout p2_layout(int row_bytes, int kslots, int dv_pad, int vpl, int stages) {
    P2Layout L;
    const uint32_t swz = (uint32_t)p2swz(row_bytes);
    L.q = 0;
    L.k = L.q + (uint32_t)kBlockRows * row_bytes;
    L.st = L.k + (uint32_t)kslots * kP2KRows * swz;
    L.vhalf = (uint32_t)(dv_pad / 2) * 128;
    L.stage = 2 * kP2PBytes + (uint32_t)vpl * L.vhalf;
    L.bias = L.st + (uint32_t)stages * L.stage;
    L.koff = L.bias + kP2Bias * kP2TS * 4;
    L.rs = L.koff + 3 * kP2MaxKsteps * 4;
    L.bars = L.rs + kBlockRows * 4;
    L.misc = L.bars + (2 * kslots + 2 * kP2Bias + 3 * stages + 6) * 8;
    L.total = L.misc + 16;
    return L;
}

// PKS > 0: the K-step count of an operand plane, fixed at compile time (the S
// product is issued with immediate descriptor offsets); PKS = 0: any width.
template <int KIND, int NPASS, int VPL, int PKS>
__global__ void __launch_bounds__(kP2Threads, 1)
    apply_tc2_kernel(const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_k,
                     const __grid_constant__ CUtensorMap map_v, const ApplyParams p) {
    extern __shared__ uint8_t smem_raw[];
    // the same offset in both CTAs (operands and barriers are addressed by offset in the peer)
    uint8_t *smem = smem_raw + ((1024u - (saddr(smem_raw) & 1023u)) & 1023u);
    const int KSL = p.kslots, NS = p.stages;
    const uint32_t swz = (uint32_t)p.swz;
    const int atoms = p.row_bytes / p.swz;
    const int box_inner = p.swz / (KIND == 1 ? 4 : 2);
    const uint32_t kslot_bytes = (uint32_t)kP2KRows * swz;
    const P2Layout L = p2_layout(p.row_bytes, KSL, p.dv_pad, VPL, NS);

    uint8_t *sQ = smem + L.q;
    uint8_t *sK = smem + L.k;
    uint8_t *sSt = smem + L.st;
    float *sBias = reinterpret_cast<float *>(smem + L.bias);
    uint32_t *koff = reinterpret_cast<uint32_t *>(smem + L.koff);
    float *sRs = reinterpret_cast<float *>(smem + L.rs);
    uint64_t *kfull = reinterpret_cast<uint64_t *>(smem + L.bars);  // [KSL] first CTA
    uint64_t *kempty = kfull + KSL;                                   // [KSL] each CTA
    uint64_t *bfull = kempty + KSL;                                   // [kP2Bias] local
    uint64_t *bempty = bfull + kP2Bias;                               // [kP2Bias] local
    uint64_t *pfull = bempty + kP2Bias;  // [NS] first CTA: both CTAs' P~ of the stage written (8 arrivals)
    uint64_t *vfull = pfull + NS;        // [NS] first CTA: both halves of V~ loaded
    uint64_t *stfree = vfull + NS;       // [NS] each CTA: the P V product that read the stage is complete
    uint64_t *qfull = stfree + NS;       // first CTA
    uint64_t *sfull = qfull + 1;         // [2] each CTA
    uint64_t *sempty = sfull + 2;        // [2] first CTA (8 arrivals)
    uint64_t *ofull = sempty + 2;        // each CTA
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(smem + L.misc);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + L.misc + 8);

    const uint32_t rank = cluster_rank();  // 0: the CTA that issues the pair's MMAs
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int rb = blockIdx.x, bz = blockIdx.z;
    const int ntiles = (p.cols + kP2TS - 1) / kP2TS;
    const uint32_t tmem_cols = 512u;  // S buffers in [0, 256), O from column 256

    if (threadIdx.x == 0) {
        for (int s = 0; s < KSL; ++s) {
            mbar_init(kfull + s, 1);
            mbar_init(kempty + s, 1);
        }
        for (int j = 0; j < kP2Bias; ++j) {
            mbar_init(bfull + j, 1);
            mbar_init(bempty + j, 4);
        }
        for (int s = 0; s < NS; ++s) {
            mbar_init(pfull + s, 8);
            mbar_init(vfull + s, 1);
            mbar_init(stfree + s, 1);
        }
        mbar_init(qfull, 1);
        for (int b = 0; b < 2; ++b) {
            mbar_init(sfull + b, 1);
            mbar_init(sempty + b, 8);
        }
        mbar_init(ofull, 1);
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(saddr(tmem_holder)),
                     "r"(tmem_cols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    cluster_sync();  // both CTAs' barriers initialised before any cross-CTA signal
    tc_fence_after();
    const uint32_t tmem_base = *tmem_holder;
    const uint32_t tmem_o = tmem_base + 256u;

    if (warp == 0) {
        // ---------------- TMA producers (both CTAs) ----------------
        // Warp 0 streams Q, this CTA's K halves and the bias slices; warp 10
        // this CTA's V~ halves.  Each waits only on its own rings, so a V~ stage
        // that is still being read never holds back the next K tile.
        if (lane == 0) {
            bool ok = true;
            int k_issued = 0, b_issued = 0;
            const uint32_t q_bytes = (uint32_t)kBlockRows * p.row_bytes;
            if (rank == 0) mbar_expect_tx(qfull, 2u * q_bytes);
            for (int a = 0; a < atoms; ++a)
                tma_load_2d_pair(saddr(sQ) + a * kBlockRows * swz, &map_q, cluster_addr(saddr(qfull), 0),
                                 a * box_inner, bz * p.rows_pad + rb * kBlockRows);
            for (int t = 0; ok && t < ntiles; ++t) {
                const int col0 = t * kP2TS;
                if (*abort_flag) break;
                for (int a = 0; a < atoms && ok; ++a) {
                    const int i = t * atoms + a, s = i % KSL;
                    if (i >= KSL && !mbar_wait(kempty + s, ((uint32_t)(i / KSL) & 1u) ^ 1u, p.timeout_ns)) {
                        ok = false;
                        break;
                    }
                    if (rank == 0) mbar_expect_tx(kfull + s, 2u * kslot_bytes);
                    tma_load_2d_pair(saddr(sK + (size_t)s * kslot_bytes), &map_k, cluster_addr(saddr(kfull + s), 0),
                                     a * box_inner, bz * p.cols_rows + col0 + (int)rank * kP2KRows);
                    k_issued = i + 1;
                }
                if (!ok) break;
                const int j = t % kP2Bias;
                if (t >= kP2Bias && !mbar_wait(bempty + j, ((uint32_t)(t / kP2Bias) & 1u) ^ 1u, p.timeout_ns)) {
                    ok = false;
                    break;
                }
                mbar_expect_tx(bfull + j, kP2TS * 4);
                bulk_load(saddr(sBias + j * kP2TS), p.col_bias + (size_t)bz * p.cols_stride + col0, kP2TS * 4,
                          saddr(bfull + j));
                b_issued = t + 1;
            }
            if (!ok) {
                atomicOr(p.err, kDevErrTimeout);
                *abort_flag = 1;
            }
            // Never leave with copies in flight: both CTAs' Q and K copies count on
            // the first CTA's barriers, so that CTA waits for them; each CTA waits
            // for its own bias copies.
            if (rank == 0) {
                mbar_wait(qfull, 0, p.timeout_ns);
                for (int i = max(0, k_issued - KSL); i < k_issued; ++i)
                    mbar_wait(kfull + (i % KSL), (uint32_t)(i / KSL) & 1u, p.timeout_ns);
            }
            for (int t = max(0, b_issued - kP2Bias); t < b_issued; ++t)
                mbar_wait(bfull + (t % kP2Bias), (uint32_t)(t / kP2Bias) & 1u, p.timeout_ns);
        }
        __syncwarp();
    } else if (warp == 10) {
        if (lane == 0) {
            bool ok = true;
            int v_issued = 0;
            for (int t = 0; ok && t < ntiles; ++t) {
                const int col0 = t * kP2TS;
                if (*abort_flag) break;
                for (int half = 0; half < 2; ++half) {
                    const int hh = 2 * t + half, s = hh % NS;
                    if (hh >= NS && !mbar_wait(stfree + s, ((uint32_t)(hh / NS) & 1u) ^ 1u, p.timeout_ns)) {
                        ok = false;
                        break;
                    }
                    uint8_t *sv = sSt + (size_t)s * L.stage + 2 * kP2PBytes;
                    if (rank == 0) mbar_expect_tx(vfull + s, 2u * (uint32_t)VPL * L.vhalf);
                    for (int pl = 0; pl < VPL; ++pl)
                        tma_load_2d_pair(saddr(sv + pl * L.vhalf), &map_v, cluster_addr(saddr(vfull + s), 0),
                                         col0 + half * kP2TH, (bz * VPL + pl) * p.dv_pad + (int)rank * (p.dv_pad / 2));
                    v_issued = hh + 1;
                }
            }
            if (!ok) {
                atomicOr(p.err, kDevErrTimeout);
                *abort_flag = 1;
            }
            // both CTAs' V~ copies count on the first CTA's barriers
            if (rank == 0)
                for (int i = max(0, v_issued - NS); i < v_issued; ++i)
                    mbar_wait(vfull + (i % NS), (uint32_t)(i / NS) & 1u, p.timeout_ns);
        }
        __syncwarp();
    } else if (warp == 1) {
        // ---------------- MMA issuer (the pair's first CTA) ----------------
        if (lane == 0 && rank == 0) {
            const uint32_t idesc_s = make_idesc<KIND, 2 * kBlockRows, kP2TS>();
            // P~ V~: bf16 x bf16 -> fp32, M = 256 over the pair, N = dv_pad
            const uint32_t idesc_o = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(p.dv_pad >> 3) << 17) |
                                     ((uint32_t)((2 * kBlockRows) >> 4) << 24);
            const uint32_t plane = (uint32_t)p.plane_bytes;
            const int ksteps = (int)(plane / 32u);
            const int nk = NPASS * ksteps;
            for (int i = 0; i < nk; ++i) {
                const int pass = i / ksteps, k = i % ksteps;
                const uint32_t ao = (pass == 1 ? plane : 0u) + 32u * k;
                const uint32_t bo = (pass == 2 ? plane : 0u) + 32u * k;
                koff[i] = ((ao / swz) * (kBlockRows * swz) + ao % swz) >> 4;
                koff[kP2MaxKsteps + i] = bo / swz;
                koff[2 * kP2MaxKsteps + i] = (bo % swz) >> 4;
            }
            const uint64_t adesc0 = make_sdesc(saddr(sQ), swz);
            bool ok = mbar_wait(qfull, 0, p.timeout_ns);
            tc_fence_after();
            for (int t = 0; ok && t <= ntiles; ++t) {
                if (t < ntiles) {  // S(t) = Q K(t)^T over the pair
                    const int b = t & 1;
                    if (t >= 2 && !mbar_wait_cluster(sempty + b, ((uint32_t)(t >> 1) & 1u) ^ 1u, p.timeout_ns)) {
                        ok = false;
                        break;
                    }
                    uint64_t bdesc[4];
#pragma unroll
                    for (int a = 0; a < 4; ++a) {
                        bdesc[a] = 0ull;
                        if (a < atoms) {
                            const int i = t * atoms + a;
                            if (!mbar_wait(kfull + (i % KSL), (uint32_t)(i / KSL) & 1u, p.timeout_ns)) ok = false;
                            bdesc[a] = make_sdesc(saddr(sK + (size_t)(i % KSL) * kslot_bytes), swz);
                        }
                    }
                    if (!ok || *abort_flag) break;
                    tc_fence_after();
                    const uint32_t dt = tmem_base + (uint32_t)(b * kP2TS);
                    if constexpr (PKS > 0) {
                        issue_s_tile<KIND, NPASS, PKS, kBlockRows, true>(dt, adesc0, bdesc, idesc_s);
                    } else {
                        for (int i = 0; i < nk; ++i) {
                            const uint32_t ba = koff[kP2MaxKsteps + i];
                            const uint64_t bd =
                                ba == 0 ? bdesc[0] : (ba == 1 ? bdesc[1] : (ba == 2 ? bdesc[2] : bdesc[3]));
                            tc_mma_pair<KIND>(dt, adesc0 + koff[i], bd + koff[2 * kP2MaxKsteps + i], idesc_s,
                                              i > 0 ? 1u : 0u);
                        }
                    }
                    tc_commit_pair(saddr(sfull + b), (uint16_t)3);
                }
                if (t >= 1) {  // O += P~ V~ over the two halves of tile t - 1
                    for (int half = 0; ok && half < 2; ++half) {
                        const int hh = 2 * (t - 1) + half, s = hh % NS;
                        const uint32_t ph = (uint32_t)(hh / NS) & 1u;
                        if (!mbar_wait_cluster(pfull + s, ph, p.timeout_ns) || !mbar_wait(vfull + s, ph, p.timeout_ns)) {
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
                        const uint64_t plo = make_sdesc(st + kP2PBytes, 128u);
                        const uint64_t v0 = make_sdesc(st + 2 * kP2PBytes, 128u);
                        const uint64_t v1 = make_sdesc(st + 2 * kP2PBytes + (VPL - 1) * L.vhalf, 128u);
                        auto pv = [&](const uint32_t first) {
#pragma unroll
                            for (int ks = 0; ks < kP2TH / 16; ++ks) {
                                tc_mma_pair<0>(tmem_o, phi + 2u * ks, v0 + 2u * ks, idesc_o, ks == 0 ? first : 1u);
                                tc_mma_pair<0>(tmem_o, plo + 2u * ks, v0 + 2u * ks, idesc_o, 1u);
                                if (VPL == 2) tc_mma_pair<0>(tmem_o, phi + 2u * ks, v1 + 2u * ks, idesc_o, 1u);
                            }
                        };
                        if (hh == 0)
                            pv(0u);
                        else
                            pv(1u);
                        tc_commit_pair(saddr(stfree + s), (uint16_t)3);
                    }
                }
            }
            if (!ok) {
                atomicOr(p.err, kDevErrTimeout);
                *abort_flag = 1;
            }
            tc_commit_pair(saddr(ofull), (uint16_t)3);  // completes when every MMA issued here has
            mbar_wait(ofull, 0, p.timeout_ns);
        }
        __syncwarp();
    } else if (warp >= 2 && warp < 10) {
        // ---------------- softmax groups (both CTAs) ----------------
        const int q = warp & 3;
        const int grp = (warp - 2) >> 2;
        const int rl = q * 32 + lane;
        const int row = rb * kBlockRows + rl;
        const bool valid = row < p.rows;
        const size_t prow = (size_t)bz * p.rows_stride + row;
        const float alpha = valid ? (float)(((double)p.pot_row[(size_t)bz * p.rows + row] - (double)p.row_norm[prow]) *
                                            p.scale)
                                  : -INFINITY;
        const float c = (float)(p.scale * (double)p.sscale);
        const uint64_t cc = pack2(c, c), aa = pack2(alpha, alpha);
        const uint32_t lane_base = tmem_base + ((uint32_t)(q * 32) << 16);
        const uint32_t prow_off = (uint32_t)((rl >> 3) * 1024 + (rl & 7) * 128);
        const uint32_t sempty0 = cluster_addr(saddr(sempty + grp), 0);
        float rs = 0.f;
        bool ok = true;
        for (int t = grp; ok && t < ntiles; t += 2) {
            const int j = t % kP2Bias;
            if (!mbar_wait(sfull + grp, (uint32_t)(t >> 1) & 1u, p.timeout_ns) ||
                !mbar_wait(bfull + j, (uint32_t)(t / kP2Bias) & 1u, p.timeout_ns)) {
                ok = false;
                break;
            }
            tc_fence_after();
            if (q == 2 && lane == 0)  // S(t) is complete: this CTA's K slots of tile t are free
                for (int a = 0; a < atoms; ++a) mbar_arrive(kempty + ((t * atoms + a) % KSL));
#pragma unroll 1
            for (int half = 0; half < 2; ++half) {
                uint32_t r[kP2TH];
                tmem_ld32(lane_base + (uint32_t)(grp * kP2TS + half * kP2TH), &r[0]);
                tmem_ld32(lane_base + (uint32_t)(grp * kP2TS + half * kP2TH + 32), &r[32]);
                tmem_ld_wait();
                if (half == 1) {  // both halves read: the S buffer is free
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive_cluster(sempty0);
                }
                const float4 *bq = reinterpret_cast<const float4 *>(sBias + j * kP2TS + half * kP2TH);
                uint32_t hi[kP2TH / 2], lo[kP2TH / 2];
                uint64_t acc2 = 0ull;
#pragma unroll
                for (int k = 0; k < kP2TH; k += 4) {
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
                // the stage is free once the pair's P V product that last read it is complete
                const int hh = 2 * t + half, s = hh % NS;
                if (hh >= NS && !mbar_wait(stfree + s, ((uint32_t)(hh / NS) & 1u) ^ 1u, p.timeout_ns)) {
                    ok = false;
                    break;
                }
                uint8_t *prow_hi = sSt + (size_t)s * L.stage + prow_off;
                uint8_t *prow_lo = prow_hi + kP2PBytes;
                // 128-byte swizzle: 16-byte chunk c of row r sits at chunk c ^ (r % 8)
#pragma unroll
                for (int ch = 0; ch < 8; ++ch) {
                    const uint32_t off = (uint32_t)((ch ^ (rl & 7)) << 4);
                    *reinterpret_cast<uint4 *>(prow_hi + off) =
                        make_uint4(hi[4 * ch], hi[4 * ch + 1], hi[4 * ch + 2], hi[4 * ch + 3]);
                    *reinterpret_cast<uint4 *>(prow_lo + off) =
                        make_uint4(lo[4 * ch], lo[4 * ch + 1], lo[4 * ch + 2], lo[4 * ch + 3]);
                }
                asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // visible to the tensor cores
                __syncwarp();
                if (lane == 0) mbar_arrive_cluster_release(cluster_addr(saddr(pfull + s), 0));
            }
            if (!ok) break;
            if (lane == 0) mbar_arrive(bempty + j);
            if (*abort_flag) break;
        }
        if (!ok) {
            atomicOr(p.err, kDevErrTimeout);
            *abort_flag = 1;
        }
        if (grp == 1) sRs[rl] = rs;
        named_barrier(1, 256);
        if (grp == 0) {
            rs += sRs[rl];
            const bool done = mbar_wait(ofull, 0, p.timeout_ns) && !*abort_flag;
            tc_fence_after();
            const float a_i = valid ? (float)exp2((double)p.row_logw2[prow]) : 0.f;
            const float scale_o = p.divide ? 1.f / rs : a_i;
            for (int c0 = 0; c0 < p.dv_pad; c0 += 32) {
                uint32_t o[32];
                tmem_ld32(lane_base + 256u + (uint32_t)c0, o);
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
    cluster_sync();  // neither CTA leaves while the pair's MMAs or the peer may touch its memory
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(tmem_cols)
                     : "memory");
    }
}

template <int KIND, int NPASS, int VPL, int PKS>
cudaError_t launch_one2(const ApplyParams &p, int batch, const void *mq, const void *mk, const void *mv,
                        size_t smem, cudaStream_t s) {
    auto kern = apply_tc2_kernel<KIND, NPASS, VPL, PKS>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(p.rows_pad / kBlockRows, 1, batch);
    cfg.blockDim = dim3(kP2Threads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, kern, *static_cast<const CUtensorMap *>(mq), *static_cast<const CUtensorMap *>(mk),
                           *static_cast<const CUtensorMap *>(mv), p);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

template <int KIND, int NPASS, int PKS>
cudaError_t launch_ks2(const ApplyParams &p, int batch, int vpl, const void *mq, const void *mk, const void *mv,
                       size_t smem, cudaStream_t s) {
    return vpl == 1 ? launch_one2<KIND, NPASS, 1, PKS>(p, batch, mq, mk, mv, smem, s)
                    : launch_one2<KIND, NPASS, 2, PKS>(p, batch, mq, mk, mv, smem, s);
}

// The compile-time row geometry matches the pass's packed rows.
template <int NPASS, int KS>
bool fits2(const ApplyParams &p) {
    return p.plane_bytes == 32 * KS && p.row_bytes == RowGeom<NPASS, KS>::kRowBytes &&
           p.swz == RowGeom<NPASS, KS>::kSwz;
}

// Compile-time S-product offsets for the usual widths: d = 32, 64 and 128
// values per plane for one-plane modes (and 256 for bf16, 512-byte rows), hi/lo
// planes of 32, 64 and 128 values (the last two fill 256- and 512-byte rows).
template <int KIND, int NPASS>
cudaError_t launch_kind2(const ApplyParams &p, int batch, int vpl, const void *mq, const void *mk, const void *mv,
                         size_t smem, cudaStream_t s) {
    if (fits2<NPASS, 2>(p)) return launch_ks2<KIND, NPASS, 2>(p, batch, vpl, mq, mk, mv, smem, s);
    if (fits2<NPASS, 4>(p)) return launch_ks2<KIND, NPASS, 4>(p, batch, vpl, mq, mk, mv, smem, s);
    if (fits2<NPASS, 8>(p)) return launch_ks2<KIND, NPASS, 8>(p, batch, vpl, mq, mk, mv, smem, s);
    if constexpr (NPASS == 1)
        if (fits2<NPASS, 16>(p)) return launch_ks2<KIND, NPASS, 16>(p, batch, vpl, mq, mk, mv, smem, s);
    return launch_ks2<KIND, NPASS, 0>(p, batch, vpl, mq, mk, mv, smem, s);
}

}  // namespace

// Shared memory, K-ring depth (slots of one operand atom of a tile's 64-row
// half) and P~/V~ stage count of the CTA-pair transport application for
// operand rows of row_bytes, dv_pad output columns (a multiple of 32, at most
// 256) and vpl planes of V~; 0 if it does not fit.
size_t apply_tc2_plan(int row_bytes, int dv_pad, int vpl, int *kslots, int *stages) {
    const size_t limit = 227 * 1024;
    if (dv_pad % 32 != 0 || dv_pad < 32 || dv_pad > 256) return 0;
    const int atoms = row_bytes / p2swz(row_bytes);
    const int plans[4][2] = {{2, 3}, {1, 3}, {2, 2}, {1, 2}};  // {K tiles, stages}, best first
    for (const auto &pl : plans) {
        const size_t bytes = (size_t)p2_layout(row_bytes, pl[0] * atoms, dv_pad, vpl, pl[1]).total + 1024;
        if (bytes <= limit) {
            *kslots = pl[0] * atoms;
            *stages = pl[1];
            return bytes < 120 * 1024 ? 120 * 1024 : bytes;  // one CTA per SM (TMEM)
        }
    }
    return 0;
}

// prec: 1 = bf16, 2 = tf32, 3 = 3xTF32, 4 = 3xF16 (the S product); vpl: planes of V~.
// rows_pad / 128 must be even (the pairs tile the rows).
cudaError_t launch_apply_tc2(const ApplyParams &p, int batch, int prec, int vpl, const void *map_q, const void *map_k,
                             const void *map_v, size_t smem, cudaStream_t s) {
    if ((p.rows_pad / kBlockRows) % 2 != 0) return cudaErrorInvalidValue;
    if (prec == 1) return launch_kind2<0, 1>(p, batch, vpl, map_q, map_k, map_v, smem, s);
    if (prec == 2) return launch_kind2<1, 1>(p, batch, vpl, map_q, map_k, map_v, smem, s);
    if (prec == 3) return launch_kind2<1, 3>(p, batch, vpl, map_q, map_k, map_v, smem, s);
    return launch_kind2<2, 3>(p, batch, vpl, map_q, map_k, map_v, smem, s);
}

}  // namespace fs
