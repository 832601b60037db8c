// Streamed LSE pass on the sm_100a tensor cores (tcgen05 + TMEM + TMA).
//
// One CTA owns a block of 128 rows of the row side ("row-stationary
// traversal", FlashSinkhorn Metodologia section 2): its packed operand tile
// Q (128 x row_bytes) is loaded once by TMA and stays in shared memory, while
// tiles K (128 columns x row_bytes) of the column side stream through a
// `stages`-deep TMA ring.  For every column tile one thread issues the
// tcgen05.mma chain S = Q K^T into one of two TMEM accumulators (128 lanes x
// 128 fp32 columns each), so the MMA of tile t+1 overlaps the exponentials of
// tile t.  Eight "softmax" warps (two per TMEM lane quadrant; one group of
// four takes the even tiles, the other the odd ones) read S with tcgen05.ld, form
//   z_ij = S_ij * log2(e)/eps + beta_j        (beta_j staged next to the K tile)
// and update a per-row online maximum and sum of 2^(z - max) in registers
// (online LSE, section 2).  Nothing of size n*m ever leaves the SM: the pass
// writes one potential per row (fused epilogue, section 2).
//
// Warp roles (320 threads): warp 0 = TMA producer, warp 1 = TMEM allocator and
// MMA issuer, warps 2..9 = softmax.  Every mbarrier wait is bounded by
// p.timeout_ns; on expiry the kernel raises kDevErrTimeout, stops issuing,
// drains its own copies and MMAs, frees TMEM and returns.
//
// Operand precision: KIND 0 = kind::f16 with bf16 operands (one pass);
// KIND 1 = kind::tf32.  NPASS 3 forms hi*hi + lo*hi + hi*lo from operand
// rows packed as [hi plane | lo plane] (the "3xTF32" split); NPASS 1 uses
// plane 0 only.
#include <cuda.h>

#include "fs_finish.cuh"

namespace fs {
namespace {

constexpr int kThreads = 320;
// Largest growth (base 2) of a row's maximum that is absorbed without a
// rescale: terms up to 2^kLazy stay in the running sum as they are.
constexpr float kLazy = 12.f;
constexpr int kTmemCols = 256;  // two 128-column fp32 accumulators

__device__ __forceinline__ uint32_t saddr(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ---- mbarrier -------------------------------------------------------------
__device__ __forceinline__ void mbar_init(uint64_t *b, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(saddr(b)), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint64_t *b, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(saddr(b)), "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t *b) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(saddr(b)) : "memory");
}
__device__ __forceinline__ bool mbar_test(uint64_t *b, uint32_t parity) {
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred P;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 P, [%1], %2;\n\t"
        "selp.b32 %0, 1, 0, P;\n\t}"
        : "=r"(done)
        : "r"(saddr(b)), "r"(parity)
        : "memory");
    return done != 0;
}
// Wait for the phase of parity `parity` to complete; false after limit_ns.
__device__ __forceinline__ bool mbar_wait(uint64_t *b, uint32_t parity, unsigned long long limit_ns) {
    if (mbar_test(b, parity)) return true;
    const unsigned long long t0 = globaltimer_ns();
    while (!mbar_test(b, parity)) {
        if (globaltimer_ns() - t0 > limit_ns) return false;
    }
    return true;
}

// ---- TMA ----------------------------------------------------------------------
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const void *map, uint32_t bar, int x, int y) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
        "l"(map), "r"(x), "r"(y), "r"(bar)
        : "memory");
}
__device__ __forceinline__ void bulk_load(uint32_t dst, const void *src, uint32_t bytes, uint32_t bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
        "l"(src), "r"(bytes), "r"(bar)
        : "memory");
}

// ---- tcgen05 ------------------------------------------------------------------
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_commit(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
                 : "memory");
}
template <int KIND>
__device__ __forceinline__ void tc_mma(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                       uint32_t accum) {
    if constexpr (KIND == 0) {
        asm volatile(
            "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
            "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
            "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accum)
            : "memory");
    } else {
        asm volatile(
            "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
            "tcgen05.mma.cta_group::1.kind::tf32 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
            "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accum)
            : "memory");
    }
}
// 32 TMEM lanes (this warp's quadrant) x 32 consecutive 32-bit columns.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
        "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]),
          "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]),
          "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]),
          "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
}
__device__ __forceinline__ void tmem_ld_wait() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// Shared-memory matrix descriptor of a K-major operand tile stored as
// swizzle atoms: 8-row groups are `8 * swz` bytes apart (stride byte offset),
// the leading byte offset is unused for swizzled K-major layouts, bits 46-47
// hold the sm_100 descriptor version (1), bits 61-63 the swizzle mode.
__device__ __forceinline__ uint64_t make_sdesc(uint32_t addr, uint32_t swz) {
    const uint64_t layout = swz == 128 ? 2ull : (swz == 64 ? 4ull : 6ull);
    uint64_t desc = (uint64_t)((addr >> 4) & 0x3FFFu);
    desc |= (uint64_t)1u << 16;
    desc |= (uint64_t)(((8u * swz) >> 4) & 0x3FFFu) << 32;
    desc |= (uint64_t)1u << 46;
    desc |= layout << 61;
    return desc;
}

// Descriptor of the 32-byte K slice at byte offset `off` of every row of a
// 128-row tile whose swizzle atoms (128 rows x swz bytes) are stored one
// after another.
__device__ __forceinline__ uint64_t slice_desc(uint32_t tile_addr, uint32_t off, uint32_t swz) {
    const uint32_t atom = off / swz, inner = off % swz;
    return make_sdesc(tile_addr + atom * (kBlockRows * swz) + inner, swz);
}

// Instruction descriptor: fp32 accumulator, A/B format (1 = bf16 for
// kind::f16, 2 = tf32 for kind::tf32), both K-major, N = M = 128.
template <int KIND>
__device__ __forceinline__ uint32_t make_idesc() {
    const uint32_t fmt = KIND == 0 ? 1u : 2u;
    return (1u << 4) | (fmt << 7) | (fmt << 10) | ((uint32_t)(kBlockCols >> 3) << 17) |
           ((uint32_t)(kBlockRows >> 4) << 24);
}

// sum_k 2^(z_k - ref) over a 128-column tile, fp32 pairs.
__device__ __forceinline__ float sum_exp2_tile(const float (&z)[128], float ref) {
    const uint64_t rn = pack2(-ref, -ref);
    uint64_t acc[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
    for (int k = 0; k < 128; k += 2) {
        float d0, d1;
        unpack2(add2(pack2(z[k], z[k + 1]), rn), d0, d1);
        acc[(k / 2) & 3] = add2(acc[(k / 2) & 3], pack2(ex2_approx(d0), ex2_approx(d1)));
    }
    float a0, a1, a2, a3, a4, a5, a6, a7;
    unpack2(acc[0], a0, a1);
    unpack2(acc[1], a2, a3);
    unpack2(acc[2], a4, a5);
    unpack2(acc[3], a6, a7);
    return ((a0 + a1) + (a2 + a3)) + ((a4 + a5) + (a6 + a7));
}

struct SmemLayout {
    uint32_t q, k, bias, cnorm, merge, red, bars, misc, total;
};

__host__ __device__ inline SmemLayout smem_layout(int row_bytes, int stages, bool measure) {
    SmemLayout L;
    const uint32_t tile = (uint32_t)kBlockRows * row_bytes;
    L.q = 0;
    L.k = tile;
    L.bias = L.k + tile * stages;
    L.cnorm = L.bias + stages * kBlockCols * 4;
    L.merge = L.cnorm + (measure ? stages * kBlockCols * 4 : 0);
    L.red = L.merge + kBlockRows * 16;
    L.bars = L.red + 4 * kBlockRows * 8;
    L.misc = L.bars + (2 * stages + 6) * 8;
    L.total = L.misc + 16;
    return L;
}

template <int KIND, int NPASS, bool MEASURE>
__global__ void __launch_bounds__(kThreads, 1)
    lse_tc_kernel(const __grid_constant__ CUtensorMap map_rows, const __grid_constant__ CUtensorMap map_cols,
                  const PassParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = smem_raw + ((1024u - (saddr(smem_raw) & 1023u)) & 1023u);

    const int NST = p.stages;
    const uint32_t swz = (uint32_t)p.swz;
    const uint32_t tile_bytes = (uint32_t)kBlockRows * p.row_bytes;
    const int atoms = p.row_bytes / p.swz;
    const int box_inner = p.swz / (KIND == 0 ? 2 : 4);
    const SmemLayout L = smem_layout(p.row_bytes, NST, MEASURE);

    uint8_t *sQ = smem + L.q;
    uint8_t *sK = smem + L.k;
    float *sBias = reinterpret_cast<float *>(smem + L.bias);
    float *sCN = reinterpret_cast<float *>(smem + L.cnorm);
    float4 *sMerge = reinterpret_cast<float4 *>(smem + L.merge);
    double *sRed = reinterpret_cast<double *>(smem + L.red);
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + L.bars);
    uint64_t *empty = full + NST;
    uint64_t *qfull = empty + NST;
    uint64_t *sfull = qfull + 1;   // [2]
    uint64_t *sempty = sfull + 2;  // [2]
    uint64_t *drain = sempty + 2;
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(smem + L.misc);
    int *flag = reinterpret_cast<int *>(smem + L.misc + 4);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + L.misc + 8);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int rb = blockIdx.x, split = blockIdx.y, bz = blockIdx.z;
    const int tile_begin = split * p.tiles_per_split;
    const int ntiles = min(p.tiles_per_split, p.col_tiles - tile_begin);

    if (threadIdx.x == 0) {
        for (int s = 0; s < NST; ++s) {
            mbar_init(full + s, 1);
            mbar_init(empty + s, 1 + 4);  // MMA commit + the four warps of the tile's group
        }
        mbar_init(qfull, 1);
        for (int b = 0; b < 2; ++b) {
            mbar_init(sfull + b, 1);
            mbar_init(sempty + b, 4);
        }
        mbar_init(drain, 1);
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(saddr(tmem_holder)),
                     "r"(kTmemCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_holder;

    if (warp == 0) {
        // ---------------- TMA producer ----------------
        if (lane == 0) {
            bool ok = true;
            int issued = 0;
            const int qrow = bz * p.rows_pad + rb * kBlockRows;
            mbar_expect_tx(qfull, tile_bytes);
            for (int a = 0; a < atoms; ++a)
                tma_load_2d(saddr(sQ) + a * kBlockRows * swz, &map_rows, saddr(qfull), a * box_inner, qrow);
            const uint32_t extra = kBlockCols * 4 * (MEASURE ? 2 : 1);
            for (int t = 0; t < ntiles; ++t) {
                const int s = t % NST;
                const uint32_t ph = (uint32_t)(t / NST) & 1u;
                if (t >= NST && !mbar_wait(empty + s, ph ^ 1u, p.timeout_ns)) {
                    ok = false;
                    break;
                }
                if (*abort_flag) break;
                const int col0 = (tile_begin + t) * kBlockCols;
                const uint32_t fb = saddr(full + s);
                mbar_expect_tx(full + s, tile_bytes + extra);
                for (int a = 0; a < atoms; ++a)
                    tma_load_2d(saddr(sK + (size_t)s * tile_bytes) + a * kBlockRows * swz, &map_cols, fb,
                                a * box_inner, bz * p.cols_pad + col0);
                bulk_load(saddr(sBias + s * kBlockCols), p.col_bias + (size_t)bz * p.cols_pad + col0,
                          kBlockCols * 4, fb);
                if (MEASURE)
                    bulk_load(saddr(sCN + s * kBlockCols), p.col_norm + (size_t)bz * p.cols_pad + col0,
                              kBlockCols * 4, fb);
                issued = t + 1;
            }
            if (!ok) {
                atomicOr(p.err, kDevErrTimeout);
                *abort_flag = 1;
            }
            // Never leave with copies in flight: wait for the last ring's worth.
            mbar_wait(qfull, 0, p.timeout_ns);
            for (int t = max(0, issued - NST); t < issued; ++t)
                mbar_wait(full + (t % NST), (uint32_t)(t / NST) & 1u, p.timeout_ns);
        }
        __syncwarp();
    } else if (warp == 1) {
        // ---------------- MMA issuer ----------------
        if (lane == 0) {
            const uint32_t idesc = make_idesc<KIND>();
            const uint32_t plane = (uint32_t)p.plane_bytes;
            const uint32_t ksteps = plane / 32u;
            bool ok = mbar_wait(qfull, 0, p.timeout_ns);
            for (int t = 0; ok && t < ntiles; ++t) {
                const int s = t % NST;
                const uint32_t ph = (uint32_t)(t / NST) & 1u;
                const int b = t & 1;
                const uint32_t bph = (uint32_t)(t >> 1) & 1u;
                if (t >= 2 && !mbar_wait(sempty + b, bph ^ 1u, p.timeout_ns)) {
                    ok = false;
                    break;
                }
                if (!mbar_wait(full + s, ph, p.timeout_ns)) {
                    ok = false;
                    break;
                }
                if (*abort_flag) break;
                tc_fence_after();
                const uint32_t dt = tmem_base + (uint32_t)(b * kBlockCols);
                const uint32_t qa = saddr(sQ), ka = saddr(sK + (size_t)s * tile_bytes);
                uint32_t acc = 0;
#pragma unroll
                for (int pass = 0; pass < NPASS; ++pass) {
                    // (A plane, B plane) = (hi,hi), (lo,hi), (hi,lo)
                    const uint32_t ap = (pass == 1) ? plane : 0u;
                    const uint32_t bp = (pass == 2) ? plane : 0u;
                    for (uint32_t k = 0; k < ksteps; ++k) {
                        tc_mma<KIND>(dt, slice_desc(qa, ap + 32u * k, swz), slice_desc(ka, bp + 32u * k, swz), idesc,
                                     acc);
                        acc = 1;
                    }
                }
                tc_commit(saddr(empty + s));
                tc_commit(saddr(sfull + b));
            }
            if (!ok) {
                atomicOr(p.err, kDevErrTimeout);
                *abort_flag = 1;
            }
            // Drain every MMA this thread issued before TMEM is released.
            tc_commit(saddr(drain));
            mbar_wait(drain, 0, p.timeout_ns);
        }
        __syncwarp();
    } else {
        // ---------------- softmax warps ----------------
        // Group 0 (warps 2..5) takes the even tiles, which the MMA writes to TMEM
        // buffer 0; group 1 (warps 6..9) the odd tiles in buffer 1.  The two
        // warps sharing an SM sub-partition therefore work on different tiles
        // and their max / exp phases interleave on the MUFU.
        const int q = warp & 3;          // TMEM lane quadrant this warp may access
        const int grp = (warp - 2) >> 2; // tile parity handled by this warp
        const int rl = q * 32 + lane;    // row within the block
        const float c = p.scale2;
        const float xn = MEASURE ? p.row_norm[(size_t)bz * p.rows_pad + rb * kBlockRows + rl] : 0.f;
        float m = -INFINITY, l = 0.f, w = 0.f;
        const uint32_t taddr = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(grp * kBlockCols);
        bool ok = true;
        for (int t = grp; t < ntiles; t += 2) {
            const int s = t % NST;
            const uint32_t ph = (uint32_t)(t / NST) & 1u;
            const uint32_t bph = (uint32_t)(t >> 1) & 1u;
            if (!mbar_wait(sfull + grp, bph, p.timeout_ns)) {
                ok = false;
                break;
            }
            tc_fence_after();
            if (!MEASURE) {
                uint32_t r[128];
                tmem_ld32(taddr + 0u, *reinterpret_cast<uint32_t(*)[32]>(&r[0]));
                tmem_ld32(taddr + 32u, *reinterpret_cast<uint32_t(*)[32]>(&r[32]));
                tmem_ld32(taddr + 64u, *reinterpret_cast<uint32_t(*)[32]>(&r[64]));
                tmem_ld32(taddr + 96u, *reinterpret_cast<uint32_t(*)[32]>(&r[96]));
                tmem_ld_wait();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(sempty + grp);
                // the bias slice arrived with the K tile; make its bytes visible here too
                if (!mbar_wait(full + s, ph, p.timeout_ns)) {
                    ok = false;
                    break;
                }
                const float4 *bq = reinterpret_cast<const float4 *>(sBias + s * kBlockCols);
                const uint64_t cc = pack2(c, c);
                float z[128];
#pragma unroll
                for (int k = 0; k < 128; k += 4) {
                    const float4 bb = bq[k / 4];
                    unpack2(fma2(pack2(__uint_as_float(r[k]), __uint_as_float(r[k + 1])), cc, pack2(bb.x, bb.y)),
                            z[k], z[k + 1]);
                    unpack2(fma2(pack2(__uint_as_float(r[k + 2]), __uint_as_float(r[k + 3])), cc, pack2(bb.z, bb.w)),
                            z[k + 2], z[k + 3]);
                }
                if (m == -INFINITY) {
                    // first tile of this warp: two passes (max, then exponentials)
                    float mx[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
                    for (int k = 0; k < 128; k += 8) {
                        mx[(k / 8) & 3] = max3(mx[(k / 8) & 3], z[k], z[k + 1]);
                        mx[(k / 8) & 3] = max3(mx[(k / 8) & 3], z[k + 2], z[k + 3]);
                        mx[(k / 8) & 3] = max3(mx[(k / 8) & 3], z[k + 4], z[k + 5]);
                        mx[(k / 8) & 3] = max3(mx[(k / 8) & 3], z[k + 6], z[k + 7]);
                    }
                    const float tmax = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3]));
                    if (tmax != -INFINITY) {
                        l = sum_exp2_tile(z, tmax);
                        m = tmax;
                    }
                } else {
                    // Later tiles: exponentials relative to the running max as it
                    // stood, the tile max alongside (no dependency between the two).
                    // Terms up to 2^kLazy are kept as they are; a larger jump of the
                    // maximum redoes the tile against the new maximum.
                    float mx[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
                    const uint64_t mneg = pack2(-m, -m);
                    uint64_t acc[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
                    for (int k = 0; k < 128; k += 2) {
                        float d0, d1;
                        unpack2(add2(pack2(z[k], z[k + 1]), mneg), d0, d1);
                        acc[(k / 2) & 3] = add2(acc[(k / 2) & 3], pack2(ex2_approx(d0), ex2_approx(d1)));
                        mx[(k / 2) & 3] = max3(mx[(k / 2) & 3], z[k], z[k + 1]);
                    }
                    const float tmax = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3]));
                    if (tmax > m + kLazy) {
                        l = l * ex2_approx(m - tmax) + sum_exp2_tile(z, tmax);
                        m = tmax;
                    } else {
                        float a0, a1, a2, a3, a4, a5, a6, a7;
                        unpack2(acc[0], a0, a1);
                        unpack2(acc[1], a2, a3);
                        unpack2(acc[2], a4, a5);
                        unpack2(acc[3], a6, a7);
                        l += ((a0 + a1) + (a2 + a3)) + ((a4 + a5) + (a6 + a7));
                    }
                }
            } else {
                // measure passes also need the raw score (C_ij = |row|^2 + |col|^2 - S_ij);
                // they run once per solve, so take the tile in two 64-column halves.
                if (!mbar_wait(full + s, ph, p.timeout_ns)) {
                    ok = false;
                    break;
                }
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    uint32_t ra[32], rb2[32];
                    tmem_ld32(taddr + 64u * half, ra);
                    tmem_ld32(taddr + 64u * half + 32u, rb2);
                    tmem_ld_wait();
                    if (half == 1) {
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive(sempty + grp);
                    }
                    const float4 *bq = reinterpret_cast<const float4 *>(sBias + s * kBlockCols + half * 64);
                    const float4 *cq = reinterpret_cast<const float4 *>(sCN + s * kBlockCols + half * 64);
                    float sv[64], z[64];
#pragma unroll
                    for (int k = 0; k < 32; ++k) {
                        sv[k] = __uint_as_float(ra[k]);
                        sv[32 + k] = __uint_as_float(rb2[k]);
                    }
                    float t0 = -INFINITY, t1 = -INFINITY, t2 = -INFINITY, t3 = -INFINITY;
#pragma unroll
                    for (int k = 0; k < 64; k += 4) {
                        const float4 bb = bq[k / 4];
                        z[k + 0] = fmaf(sv[k + 0], c, bb.x);
                        z[k + 1] = fmaf(sv[k + 1], c, bb.y);
                        z[k + 2] = fmaf(sv[k + 2], c, bb.z);
                        z[k + 3] = fmaf(sv[k + 3], c, bb.w);
                        t0 = fmaxf(t0, z[k + 0]);
                        t1 = fmaxf(t1, z[k + 1]);
                        t2 = fmaxf(t2, z[k + 2]);
                        t3 = fmaxf(t3, z[k + 3]);
                    }
                    const float mnew = fmaxf(m, fmaxf(fmaxf(t0, t1), fmaxf(t2, t3)));
                    if (mnew != -INFINITY) {
                        const float scale = ex2_approx(m - mnew);
                        float a0 = 0.f, a1 = 0.f, w0 = 0.f, w1 = 0.f;
#pragma unroll
                        for (int k = 0; k < 64; k += 4) {
                            const float4 cn = cq[k / 4];
                            const float e0 = ex2_approx(z[k + 0] - mnew);
                            const float e1 = ex2_approx(z[k + 1] - mnew);
                            const float e2 = ex2_approx(z[k + 2] - mnew);
                            const float e3 = ex2_approx(z[k + 3] - mnew);
                            a0 += e0 + e2;
                            a1 += e1 + e3;
                            w0 = fmaf(e0, xn + cn.x - sv[k + 0], w0);
                            w1 = fmaf(e1, xn + cn.y - sv[k + 1], w1);
                            w0 = fmaf(e2, xn + cn.z - sv[k + 2], w0);
                            w1 = fmaf(e3, xn + cn.w - sv[k + 3], w1);
                        }
                        l = l * scale + (a0 + a1);
                        w = w * scale + (w0 + w1);
                        m = mnew;
                    }
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(empty + s);
            if (*abort_flag) break;
        }
        if (!ok) {
            atomicOr(p.err, kDevErrTimeout);
            *abort_flag = 1;
        }
        // Merge the two tile-parity groups' states of each row, then finish the row block.
        if (grp == 1) sMerge[rl] = make_float4(m, l, w, 0.f);
        named_barrier(1, 256);
        if (grp == 0) {
            const float4 o = sMerge[rl];
            lse_merge(m, l, w, o.x, o.y, o.z);
            finish_rows<MEASURE>(p, rl, m, l, w, 2, sRed, flag);
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(kTmemCols)
                     : "memory");
    }
}

template <int KIND, int NPASS, bool MEASURE>
cudaError_t launch_variant(const PassParams &p, int batch, const void *map_rows, const void *map_cols,
                           size_t smem, cudaStream_t s) {
    auto kern = lse_tc_kernel<KIND, NPASS, MEASURE>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    dim3 grid(p.rows_pad / kBlockRows, p.splits, batch);
    kern<<<grid, kThreads, smem, s>>>(*static_cast<const CUtensorMap *>(map_rows),
                                      *static_cast<const CUtensorMap *>(map_cols), p);
    return cudaGetLastError();
}

}  // namespace

size_t tc_smem_bytes(int row_bytes, int stages, bool measure) {
    return (size_t)smem_layout(row_bytes, stages, measure).total + 1024;  // + alignment slack
}

int tc_max_stages(int row_bytes, bool measure) {
    const size_t limit = 227 * 1024;
    int best = 0;
    for (int s = 2; s <= 8; ++s)
        if (tc_smem_bytes(row_bytes, s, measure) <= limit) best = s;
    return best;
}

// prec: 1 = bf16, 2 = tf32 (one pass), 3 = 3xTF32.
cudaError_t launch_lse_tc(const PassParams &p, int batch, bool measure, int prec, const void *map_rows,
                          const void *map_cols, size_t smem, cudaStream_t s) {
    if (prec == 1)
        return measure ? launch_variant<0, 1, true>(p, batch, map_rows, map_cols, smem, s)
                       : launch_variant<0, 1, false>(p, batch, map_rows, map_cols, smem, s);
    if (prec == 2)
        return measure ? launch_variant<1, 1, true>(p, batch, map_rows, map_cols, smem, s)
                       : launch_variant<1, 1, false>(p, batch, map_rows, map_cols, smem, s);
    return measure ? launch_variant<1, 3, true>(p, batch, map_rows, map_cols, smem, s)
                   : launch_variant<1, 3, false>(p, batch, map_rows, map_cols, smem, s);
}

}  // namespace fs
