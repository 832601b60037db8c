// Transport application on the sm_100a tensor cores: out_i = sum_j P_ij V_j
// for the plan P_ij = a_i b_j exp((f_i + g_j - C_ij)/eps) at given potentials,
// without forming P ("FlashSinkhorn: IO-aware EOT on GPU", Metodologia
// section 3: plan-weighted averages over the same streamed tiles, an
// attention-style "P V" product).
//
// One CTA owns 128 rows.  Column tiles of 128 points stream through:
//   1. S = Q K^T (M = 128, N = 128, the handle's operand precision) into one
//      of two TMEM buffers;
//   2. the tile's softmax group reads S in two halves of 64 columns.  For each
//      half it forms p~_ij = P_ij / a_i = 2^(alpha'_i + beta_j + S_ij c) with
//      alpha'_i = (f_i - |x_i|^2) log2(e)/eps and the pass's column bias
//      beta_j, adds it to the row sum, splits it into bf16 hi + lo and writes
//      both planes into a shared-memory stage in the 128-byte-swizzled K-major
//      layout of an MMA operand;
//   3. O += P~ V~ (M = 128, N = dv rounded up to 16, K = 64) accumulates in
//      TMEM, one product per half; V~ is V transposed and packed in bf16 (one
//      plane for bf16 inputs, hi + lo planes otherwise), so the product is
//      hi.hi + lo.hi (+ hi.lo).
// A stage holds one half's P~ planes and its V~ planes; it is refilled once
// the P~ V~ product that read it has completed (one tcgen05.commit frees both).
// The reference a_i makes every p~ at most about 1 near a solution, so no
// running maximum or rescaling is needed; bf16 keeps fp32's range, so small
// entries do not underflow.  At the end out_i = a_i O_i (or O_i / sum_j p~_ij
// for the barycentric map) and r_i = a_i sum_j p~_ij.
//
// Warp roles as in the streamed LSE pass: warp 0 TMA producer, warp 1 TMEM
// allocator and MMA issuer (the S product of tile t, then the two P V
// products of tile t - 1), warps 2..9 two softmax groups taking the even and
// the odd tiles.  Every wait is bounded; on expiry the kernel raises
// kDevErrTimeout, stops, drains its own copies and MMAs, frees TMEM and
// returns.
#include <cuda_bf16.h>

#include "fs_tc_common.cuh"

namespace fs {
namespace {

using namespace tc;

constexpr int kAThreads = 320;
constexpr int kTS = 128;          // columns per tile (N of the S product)
constexpr int kTH = 64;           // columns per half (K of one P V product)
constexpr int kAMaxKsteps = 64;
constexpr int kABias = 4;         // bias-slice ring (tiles)
constexpr uint32_t kPBytes = kBlockRows * 128;  // one bf16 plane of P~: 128 rows x 64 values

struct ALayout {
    uint32_t q, k, st, stage, bias, koff, rs, bars, misc, total;
};

__host__ __device__ inline int aswz(int row_bytes) { return row_bytes <= 32 ? 32 : (row_bytes <= 64 ? 64 : 128); }

// Stage = [P~ hi | P~ lo | V~ plane 0 (| V~ plane 1)]; every part is a
// multiple of 1024 bytes, so each starts on a swizzle-atom boundary.
__host__ __device__ inline ALayout a_layout(int row_bytes, int kslots, int dv_pad, int vpl, int stages) {
    ALayout L;
    const uint32_t swz = (uint32_t)aswz(row_bytes);
    L.q = 0;
    L.k = L.q + (uint32_t)kBlockRows * row_bytes;
    L.st = L.k + (uint32_t)kslots * kTS * swz;
    L.stage = 2 * kPBytes + (uint32_t)vpl * dv_pad * 128;
    L.bias = L.st + (uint32_t)stages * L.stage;
    L.koff = L.bias + kABias * kTS * 4;
    L.rs = L.koff + 3 * kAMaxKsteps * 4;
    L.bars = L.rs + kBlockRows * 4;
    L.misc = L.bars + (2 * kslots + 2 * kABias + 3 * stages + 6) * 8;
    L.total = L.misc + 16;
    return L;
}

// PKS > 0: the K-step count of an operand plane, fixed at compile time (the S
// product is issued with immediate descriptor offsets); PKS = 0: any width.
template <int KIND, int NPASS, int VPL, int PKS>
__global__ void __launch_bounds__(kAThreads, 1)
    apply_tc_kernel(const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_k,
                    const __grid_constant__ CUtensorMap map_v, const ApplyParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = smem_raw + ((1024u - (saddr(smem_raw) & 1023u)) & 1023u);
    const int KS = p.kslots, NS = p.stages;
    const uint32_t swz = (uint32_t)p.swz;
    const int atoms = p.row_bytes / p.swz;
    const int box_inner = p.swz / (KIND == 1 ? 4 : 2);
    const uint32_t kslot_bytes = (uint32_t)kTS * swz;
    const uint32_t vplane_bytes = (uint32_t)p.dv_pad * 128u;
    const ALayout L = a_layout(p.row_bytes, KS, p.dv_pad, VPL, NS);

    uint8_t *sQ = smem + L.q;
    uint8_t *sK = smem + L.k;
    uint8_t *sSt = smem + L.st;
    float *sBias = reinterpret_cast<float *>(smem + L.bias);
    uint32_t *koff = reinterpret_cast<uint32_t *>(smem + L.koff);
    float *sRs = reinterpret_cast<float *>(smem + L.rs);
    uint64_t *kfull = reinterpret_cast<uint64_t *>(smem + L.bars);
    uint64_t *kempty = kfull + KS;
    uint64_t *bfull = kempty + KS;
    uint64_t *bempty = bfull + kABias;
    uint64_t *pfull = bempty + kABias;  // [NS] P~ of the stage written
    uint64_t *vfull = pfull + NS;       // [NS] V~ of the stage loaded
    uint64_t *stfree = vfull + NS;      // [NS] the P V product that read the stage is complete
    uint64_t *qfull = stfree + NS;
    uint64_t *sfull = qfull + 1;   // [2]
    uint64_t *sempty = sfull + 2;  // [2]
    uint64_t *ofull = sempty + 2;
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(smem + L.misc);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + L.misc + 8);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int rb = blockIdx.x, bz = blockIdx.z;
    const int ntiles = (p.cols + kTS - 1) / kTS;
    // S buffers in columns [0, 256), the O accumulator from column 256 (it
    // never straddles the middle of the allocation).
    const uint32_t tmem_cols = 512u;

    if (threadIdx.x == 0) {
        for (int s = 0; s < KS; ++s) {
            mbar_init(kfull + s, 1);
            mbar_init(kempty + s, 1);
        }
        for (int j = 0; j < kABias; ++j) {
            mbar_init(bfull + j, 1);
            mbar_init(bempty + j, 4);
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
        // Lane 0 streams Q, the K tiles and the bias slices; lane 1 streams the
        // V~ halves.  Each waits only on its own rings, so a V~ stage that is
        // still being read never holds back the next K tile.
        if (lane == 0) {
            bool ok = true;
            int k_issued = 0, b_issued = 0;
            mbar_expect_tx(qfull, (uint32_t)kBlockRows * p.row_bytes);
            for (int a = 0; a < atoms; ++a)
                tma_load_2d(saddr(sQ) + a * kBlockRows * swz, &map_q, saddr(qfull), a * box_inner,
                            bz * p.rows_pad + rb * kBlockRows);
            for (int t = 0; ok && t < ntiles; ++t) {
                const int col0 = t * kTS;
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
                const int j = t % kABias;
                if (t >= kABias && !mbar_wait(bempty + j, ((uint32_t)(t / kABias) & 1u) ^ 1u, p.timeout_ns)) {
                    ok = false;
                    break;
                }
                mbar_expect_tx(bfull + j, kTS * 4);
                bulk_load(saddr(sBias + j * kTS), p.col_bias + (size_t)bz * p.cols_stride + col0, kTS * 4,
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
            for (int t = max(0, b_issued - kABias); t < b_issued; ++t)
                mbar_wait(bfull + (t % kABias), (uint32_t)(t / kABias) & 1u, p.timeout_ns);
        } else if (lane == 1) {
            bool ok = true;
            int v_issued = 0;
            for (int t = 0; ok && t < ntiles; ++t) {
                const int col0 = t * kTS;
                if (*abort_flag) break;
                for (int half = 0; half < 2; ++half) {
                    const int hh = 2 * t + half, s = hh % NS;
                    if (hh >= NS && !mbar_wait(stfree + s, ((uint32_t)(hh / NS) & 1u) ^ 1u, p.timeout_ns)) {
                        ok = false;
                        break;
                    }
                    uint8_t *sv = sSt + (size_t)s * L.stage + 2 * kPBytes;
                    mbar_expect_tx(vfull + s, (uint32_t)VPL * vplane_bytes);
                    for (int pl = 0; pl < VPL; ++pl)
                        tma_load_2d(saddr(sv + pl * vplane_bytes), &map_v, saddr(vfull + s), col0 + half * kTH,
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
            const uint32_t idesc_s = make_idesc<KIND, kBlockRows, kTS>();
            // P~ V~: bf16 x bf16 -> fp32, M = 128, N = dv_pad
            const uint32_t idesc_o = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(p.dv_pad >> 3) << 17) |
                                     ((uint32_t)(kBlockRows >> 4) << 24);
            const uint32_t plane = (uint32_t)p.plane_bytes;
            const int ksteps = (int)(plane / 32u);
            const int nk = NPASS * ksteps;
            for (int i = 0; i < nk; ++i) {
                const int pass = i / ksteps, k = i % ksteps;
                const uint32_t ao = (pass == 1 ? plane : 0u) + 32u * k;
                const uint32_t bo = (pass == 2 ? plane : 0u) + 32u * k;
                koff[i] = ((ao / swz) * (kBlockRows * swz) + ao % swz) >> 4;
                koff[kAMaxKsteps + i] = bo / swz;
                koff[2 * kAMaxKsteps + i] = (bo % swz) >> 4;
            }
            const uint64_t adesc0 = make_sdesc(saddr(sQ), swz);
            bool ok = mbar_wait(qfull, 0, p.timeout_ns);
            tc_fence_after();
            for (int t = 0; ok && t <= ntiles; ++t) {
                if (t < ntiles) {  // S(t) = Q K(t)^T
                    const int b = t & 1;
                    if (t >= 2 && !mbar_wait(sempty + b, ((uint32_t)(t >> 1) & 1u) ^ 1u, p.timeout_ns)) {
                        ok = false;
                        break;
                    }
                    uint64_t bdesc[4];
#pragma unroll
                    for (int a = 0; a < 4; ++a) {
                        bdesc[a] = 0ull;
                        if (a < atoms) {
                            const int i = t * atoms + a;
                            if (!mbar_wait(kfull + (i % KS), (uint32_t)(i / KS) & 1u, p.timeout_ns)) ok = false;
                            bdesc[a] = make_sdesc(saddr(sK + (size_t)(i % KS) * kslot_bytes), swz);
                        }
                    }
                    if (!ok || *abort_flag) break;
                    tc_fence_after();
                    const uint32_t dt = tmem_base + (uint32_t)(b * kTS);
                    if constexpr (PKS > 0) {
                        issue_s_tile<KIND, NPASS, PKS, kBlockRows>(dt, adesc0, bdesc, idesc_s);
                    } else {
                        for (int i = 0; i < nk; ++i) {
                            const uint32_t ba = koff[kAMaxKsteps + i];
                            const uint64_t bd =
                                ba == 0 ? bdesc[0] : (ba == 1 ? bdesc[1] : (ba == 2 ? bdesc[2] : bdesc[3]));
                            tc_mma<KIND>(dt, adesc0 + koff[i], bd + koff[2 * kAMaxKsteps + i], idesc_s,
                                         i > 0 ? 1u : 0u);
                        }
                    }
                    tc_commit(saddr(sfull + b));
                }
                if (t >= 1) {  // O += P~ V~ over the two halves of tile t - 1
                    for (int half = 0; ok && half < 2; ++half) {
                        const int hh = 2 * (t - 1) + half, s = hh % NS;
                        const uint32_t ph = (uint32_t)(hh / NS) & 1u;
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
                        const uint64_t plo = make_sdesc(st + kPBytes, 128u);
                        const uint64_t v0 = make_sdesc(st + 2 * kPBytes, 128u);
                        const uint64_t v1 = make_sdesc(st + 2 * kPBytes + (VPL - 1) * vplane_bytes, 128u);
                        // 16 values = 32 bytes per K step; every offset and accumulate
                        // flag an immediate (the kernel's first product starts O afresh)
                        auto pv = [&](const uint32_t first) {
#pragma unroll
                            for (int ks = 0; ks < kTH / 16; ++ks) {
                                tc_mma<0>(tmem_o, phi + 2u * ks, v0 + 2u * ks, idesc_o, ks == 0 ? first : 1u);
                                tc_mma<0>(tmem_o, plo + 2u * ks, v0 + 2u * ks, idesc_o, 1u);
                                if (VPL == 2) tc_mma<0>(tmem_o, phi + 2u * ks, v1 + 2u * ks, idesc_o, 1u);
                            }
                        };
                        if (hh == 0)
                            pv(0u);
                        else
                            pv(1u);
                        tc_commit(saddr(stfree + s));
                    }
                }
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
        // ---------------- softmax groups ----------------
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
        // this thread's row in a P~ plane (8-row swizzle atoms of 1024 bytes)
        const uint32_t prow_off = (uint32_t)((rl >> 3) * 1024 + (rl & 7) * 128);
        float rs = 0.f;
        bool ok = true;
        for (int t = grp; ok && t < ntiles; t += 2) {
            const int j = t % kABias;
            if (!mbar_wait(sfull + grp, (uint32_t)(t >> 1) & 1u, p.timeout_ns) ||
                !mbar_wait(bfull + j, (uint32_t)(t / kABias) & 1u, p.timeout_ns)) {
                ok = false;
                break;
            }
            tc_fence_after();
            if (q == 2 && lane == 0)  // S(t) is complete: tile t's K slots are free
                for (int a = 0; a < atoms; ++a) mbar_arrive(kempty + ((t * atoms + a) % KS));
#pragma unroll 1
            for (int half = 0; half < 2; ++half) {
                uint32_t r[kTH];
                tmem_ld32(lane_base + (uint32_t)(grp * kTS + half * kTH), &r[0]);
                tmem_ld32(lane_base + (uint32_t)(grp * kTS + half * kTH + 32), &r[32]);
                tmem_ld_wait();
                if (half == 1) {  // both halves read: the S buffer is free
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(sempty + grp);
                }
                const float4 *bq = reinterpret_cast<const float4 *>(sBias + j * kTS + half * kTH);
                uint32_t hi[kTH / 2], lo[kTH / 2];
                uint64_t acc2 = 0ull;
#pragma unroll
                for (int k = 0; k < kTH; k += 4) {
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
                // the stage is free once the P V product that last read it is complete
                const int hh = 2 * t + half, s = hh % NS;
                if (hh >= NS && !mbar_wait(stfree + s, ((uint32_t)(hh / NS) & 1u) ^ 1u, p.timeout_ns)) {
                    ok = false;
                    break;
                }
                uint8_t *prow_hi = sSt + (size_t)s * L.stage + prow_off;
                uint8_t *prow_lo = prow_hi + kPBytes;
                // 128-byte swizzle: 16-byte chunk c of row r sits at chunk c ^ (r % 8)
#pragma unroll
                for (int ch = 0; ch < 8; ++ch) {
                    const uint32_t off = (uint32_t)((ch ^ (rl & 7)) << 4);
                    *reinterpret_cast<uint4 *>(prow_hi + off) =
                        make_uint4(hi[4 * ch], hi[4 * ch + 1], hi[4 * ch + 2], hi[4 * ch + 3]);
                    *reinterpret_cast<uint4 *>(prow_lo + off) =
                        make_uint4(lo[4 * ch], lo[4 * ch + 1], lo[4 * ch + 2], lo[4 * ch + 3]);
                }
                asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // visible to the tensor core
                __syncwarp();
                if (lane == 0) mbar_arrive(pfull + s);
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
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(tmem_cols)
                     : "memory");
    }
}

// V~[bz][plane][c][j] = split_plane(V[bz][j][c]) in bf16, zero beyond dv and m.
template <typename T>
__global__ void vt_pack_kernel(const T *V, int m, int dv, int m_pad, int dv_pad, int vpl, __nv_bfloat16 *out) {
    __shared__ float tile[32][33];
    const int j0 = blockIdx.x * 32, c0 = blockIdx.y * 32, bz = blockIdx.z;
    const int tx = threadIdx.x, ty = threadIdx.y;  // 32 x 8
    for (int y = ty; y < 32; y += 8) {
        const int j = j0 + y, c = c0 + tx;
        float v = 0.f;
        if (j < m && c < dv) {
            const size_t i = ((size_t)bz * m + j) * dv + c;
            if constexpr (sizeof(T) == 2)
                v = __bfloat162float(reinterpret_cast<const __nv_bfloat16 *>(V)[i]);
            else
                v = reinterpret_cast<const float *>(V)[i];
        }
        tile[y][tx] = v;
    }
    __syncthreads();
    for (int y = ty; y < 32; y += 8) {
        const int c = c0 + y, j = j0 + tx;
        if (c >= dv_pad || j >= m_pad) continue;
        const float v = tile[tx][y];
        const __nv_bfloat16 h = __float2bfloat16_rn(v);
        out[(((size_t)bz * vpl + 0) * dv_pad + c) * m_pad + j] = h;
        if (vpl == 2) out[(((size_t)bz * vpl + 1) * dv_pad + c) * m_pad + j] = __float2bfloat16_rn(v - __bfloat162float(h));
    }
}

template <int KIND, int NPASS, int VPL, int KS>
cudaError_t launch_one(const ApplyParams &p, int batch, const void *mq, const void *mk, const void *mv, size_t smem,
                       cudaStream_t s) {
    dim3 grid(p.rows_pad / kBlockRows, 1, batch);
    auto kern = apply_tc_kernel<KIND, NPASS, VPL, KS>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    kern<<<grid, kAThreads, smem, s>>>(*static_cast<const CUtensorMap *>(mq), *static_cast<const CUtensorMap *>(mk),
                                       *static_cast<const CUtensorMap *>(mv), p);
    return cudaGetLastError();
}

template <int KIND, int NPASS, int KS>
cudaError_t launch_ks(const ApplyParams &p, int batch, int vpl, const void *mq, const void *mk, const void *mv,
                      size_t smem, cudaStream_t s) {
    return vpl == 1 ? launch_one<KIND, NPASS, 1, KS>(p, batch, mq, mk, mv, smem, s)
                    : launch_one<KIND, NPASS, 2, KS>(p, batch, mq, mk, mv, smem, s);
}

// The usual plane widths (d = 16, 32, 64 and, one-plane modes, 128 values)
// take the S product with compile-time offsets; others the table.
// The compile-time row geometry matches the pass's packed rows.
template <int NPASS, int KS, typename Params>
bool fits(const Params &p) {
    return p.row_bytes == RowGeom<NPASS, KS>::kRowBytes && p.swz == RowGeom<NPASS, KS>::kSwz;
}

template <int KIND, int NPASS>
cudaError_t launch_kind(const ApplyParams &p, int batch, int vpl, const void *mq, const void *mk, const void *mv,
                        size_t smem, cudaStream_t s) {
    const int ks = p.plane_bytes / 32;
    if (ks * 32 == p.plane_bytes) {
        if (ks == 1 && fits<NPASS, 1>(p)) return launch_ks<KIND, NPASS, 1>(p, batch, vpl, mq, mk, mv, smem, s);
        if (ks == 2 && fits<NPASS, 2>(p)) return launch_ks<KIND, NPASS, 2>(p, batch, vpl, mq, mk, mv, smem, s);
        if (ks == 4 && fits<NPASS, 4>(p)) return launch_ks<KIND, NPASS, 4>(p, batch, vpl, mq, mk, mv, smem, s);
        if constexpr (NPASS == 1)
            if (ks == 8 && fits<NPASS, 8>(p)) return launch_ks<KIND, NPASS, 8>(p, batch, vpl, mq, mk, mv, smem, s);
    }
    return launch_ks<KIND, NPASS, 0>(p, batch, vpl, mq, mk, mv, smem, s);
}

}  // namespace

// Shared memory of the tensor-core transport application, its K-ring depth
// (slots of one operand atom of a 128-column tile) and its stage count (one
// 64-column half of P~ and V~ each); 0 if it does not fit.  A third stage
// pays more than a second K tile: with two stages, writing P~ of a half waits
// for the P V product of the half two back, which is issued only after the
// S product this group has just read.
size_t apply_tc_plan(int row_bytes, int dv_pad, int vpl, int *kslots, int *stages) {
    const size_t limit = 227 * 1024;
    const int atoms = row_bytes / aswz(row_bytes);
    const int plans[4][2] = {{2, 3}, {1, 3}, {2, 2}, {1, 2}};  // {K tiles, stages}, best first
    for (const auto &pl : plans) {
        const size_t bytes = (size_t)a_layout(row_bytes, pl[0] * atoms, dv_pad, vpl, pl[1]).total + 1024;
        if (bytes <= limit) {
            *kslots = pl[0] * atoms;
            *stages = pl[1];
            return bytes < 120 * 1024 ? 120 * 1024 : bytes;  // one CTA per SM (TMEM)
        }
    }
    return 0;
}

cudaError_t launch_vt_pack(const void *V, bool bf16, int batch, int m, int dv, int m_pad, int dv_pad, int vpl,
                           void *out, cudaStream_t s) {
    dim3 grid((m_pad + 31) / 32, (dv_pad + 31) / 32, batch), block(32, 8);
    if (bf16)
        vt_pack_kernel<<<grid, block, 0, s>>>(static_cast<const __nv_bfloat16 *>(V), m, dv, m_pad, dv_pad, vpl,
                                              static_cast<__nv_bfloat16 *>(out));
    else
        vt_pack_kernel<<<grid, block, 0, s>>>(static_cast<const float *>(V), m, dv, m_pad, dv_pad, vpl,
                                              static_cast<__nv_bfloat16 *>(out));
    return cudaGetLastError();
}

// prec: 1 = bf16, 2 = tf32, 3 = 3xTF32, 4 = 3xF16 (the S product); vpl: planes of V~.
cudaError_t launch_apply_tc(const ApplyParams &p, int batch, int prec, int vpl, const void *map_q, const void *map_k,
                            const void *map_v, size_t smem, cudaStream_t s) {
    if (prec == 1) return launch_kind<0, 1>(p, batch, vpl, map_q, map_k, map_v, smem, s);
    if (prec == 2) return launch_kind<1, 1>(p, batch, vpl, map_q, map_k, map_v, smem, s);
    if (prec == 3) return launch_kind<1, 3>(p, batch, vpl, map_q, map_k, map_v, smem, s);
    return launch_kind<2, 3>(p, batch, vpl, map_q, map_k, map_v, smem, s);
}

}  // namespace fs
