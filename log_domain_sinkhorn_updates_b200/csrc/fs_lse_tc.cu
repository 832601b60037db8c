// Streamed LSE pass on the sm_100a tensor cores (tcgen05 + TMEM + TMA).
//
// One CTA owns QT blocks of 128 rows of the row side ("row-stationary
// traversal", FlashSinkhorn Metodologia section 2): their packed operand
// tiles Q_0..Q_{QT-1} (128 x row_bytes each) are loaded once by TMA and stay in
// shared memory, while 256-column tiles K of the column side stream through a
// ring of TMA slots (one slot = 256 rows x one swizzle atom of the row).  Every
// K tile is multiplied by each resident Q tile, so with QT = 2 a tile crosses
// L2 -> SM, and is written into shared memory, once per 256 rows instead of
// once per 128.
//
// The MMA issuer runs a sequence of jobs; job j computes S = Q K^T (M = 128,
// N = 256, both operands in shared memory) into TMEM buffer j & 1 (two buffers
// of 256 fp32 columns), so the MMA of one job overlaps the exponentials of the
// previous ones.  With QT = 1, job j is tile j; with QT = 2, job j is tile j/2
// times Q tile j % 2.  Eight "softmax" warps in two groups of four (one warp per
// TMEM lane quadrant) take the jobs of their buffer: group g handles jobs
// j = g mod 2, i.e. the even or odd tiles (QT = 1) or every tile of Q tile g
// (QT = 2).  They read S with tcgen05.ld, form
//   z_ij = S_ij * log2(e)/eps + beta_j
// and update a per-row online maximum and sum of 2^(z - max) in registers
// (online LSE, section 2).  In the update passes (and the vector passes, which
// weight column j by v_j) the column bias enters the S product itself: each
// job ends with one more K step, a constant tile of rows (1, 1, 1, 0, ...)
// times the tile's bias rows (beta_j / c in three parts, store_bias_mm), so
// TMEM holds S_ij + beta_j / c and the softmax forms z - max with one packed
// FMA per two entries, with no bias load.  (Measured without the bias work at
// all: 6 % less time per pass.)  The bias rows stream through a ring of two
// tiles beside the K slots and go back to the producer through the issuers'
// commits.  Measure passes with statistics need S itself (C_ij from it): they
// read fp32 bias and |y|^2 slices in the softmax, from a ring of their own,
// from which vector passes read v.
// Nothing of size n*m ever leaves the SM: the pass writes one potential per
// row (fused epilogue, section 2).
//
// Warp roles (352 threads): warp 0 = TMA producer, warp 1 = TMEM allocator and
// MMA issuer, warps 2..9 = softmax, warp 10 = the second MMA issuer when
// p.issuers = 2: warp 1 then issues the even jobs and warp 10 the odd ones, so
// one softmax group's wait for its buffer never holds back the other group's
// next S.  Measured per pass: bf16 at d = 128 (8 MMAs per job) 2 % faster at
// equal clock, 3xF16 at d = 3 (3 MMAs) 2 % faster, 3xF16 at d = 32 (6 MMAs)
// 1 % slower, 3xF16 at d = 64 (12 MMAs) 5 % slower: the two groups' MMAs
// interleave in the pipe and both S arrive late.  So two threads issue for
// one-pass operands and for split jobs of at most 4 MMAs.  The K slots of a
// tile go back to the producer through a commit after each of its jobs.
// Every mbarrier wait is bounded by
// p.timeout_ns; on expiry the kernel raises kDevErrTimeout, stops issuing,
// drains its own copies and MMAs, frees TMEM and returns.
//
// Operand precision: KIND 0 = kind::f16 with bf16 operands, KIND 1 =
// kind::tf32, KIND 2 = kind::f16 with fp16 operands.  NPASS 3 forms
// hi*hi + lo*hi + hi*lo from operand rows packed as [hi plane | lo plane]
// (the 3xTF32 / 3xF16 splits); NPASS 1 uses plane 0 only.
#include "fs_tc_common.cuh"

namespace fs {
namespace {

using namespace tc;

constexpr int kThreads = 352;
constexpr int kTmemCols = 512;   // two 256-column fp32 accumulators
constexpr int kMaxKsteps = 64;   // MMA instructions per tile: NPASS x (plane bytes / 32) <= 3 x 16
constexpr int kMaxAtoms = 4;     // swizzle atoms per packed row (row_bytes <= 512)
constexpr int kBiasSlots = 4;    // measure passes: tiles whose fp32 column slices may be in flight
constexpr int kBiasTiles = 2;    // update and vector passes: tiles whose bias rows (32 bytes a column) may be in flight
constexpr int kBiasRowBytes = 32;

// Pass modes: an update; a measure pass with statistics; a measure pass that
// weights each column by v_j (col_vec).  The update and vector passes add the
// bias inside the S product; the statistics pass needs S itself (C_ij from it)
// and reads fp32 bias slices.
constexpr int kUpdate = 0, kStats = 1, kVector = 2;

struct SmemLayout {
    uint32_t q, k, bias, ones, cnorm, merge, red, koff, bars, misc, total;
};

__host__ __device__ inline int swizzle_of(int row_bytes) { return row_bytes <= 32 ? 32 : (row_bytes <= 64 ? 64 : 128); }

// slots: K ring slots of kBlockCols rows x one swizzle atom each; qt: resident Q tiles.
__host__ __device__ inline SmemLayout smem_layout(int row_bytes, int slots, int mode, int qt) {
    SmemLayout L;
    const uint32_t swz = (uint32_t)swizzle_of(row_bytes);
    const bool fold = mode != kStats;
    L.q = 0;
    L.k = (uint32_t)(qt * kBlockRows) * row_bytes;
    // the bias-row ring and the tile of ones (128 rows of 32 bytes) of the bias step
    L.bias = L.k + (uint32_t)slots * kBlockCols * swz;
    L.ones = L.bias + (fold ? kBiasTiles * kBlockCols * kBiasRowBytes : 0);
    // the fp32 column slices of measure passes: bias (statistics) and |y|^2 or v
    L.cnorm = L.ones + (fold ? kBlockRows * kBiasRowBytes : 0) + (mode == kStats ? kBiasSlots * kBlockCols * 4 : 0);
    L.merge = L.cnorm + (mode != kUpdate ? kBiasSlots * kBlockCols * 4 : 0);
    L.red = L.merge + kBlockRows * 16;
    L.koff = L.red + (mode == kVector ? 0u : (uint32_t)qt * 4 * kBlockRows * 8);  // a vector pass keeps no statistics
    L.bars = L.koff + 3 * kMaxKsteps * 4;
    L.misc = L.bars + (2 * slots + 2 * kBiasTiles + 2 * kBiasSlots + 6) * 8;
    L.total = L.misc + 32;
    return L;
}

// KS > 0: the plane's K-step count, fixed at compile time (the MMAs of a job
// are issued with immediate descriptor offsets); KS = 0: any width, offsets
// from a table in shared memory.
template <int KIND, int NPASS, int MODE, int QT, int KS>
__global__ void __launch_bounds__(kThreads, 1)
    lse_tc_kernel(const __grid_constant__ CUtensorMap map_rows, const __grid_constant__ CUtensorMap map_cols,
                  const __grid_constant__ CUtensorMap map_bias, const PassParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = smem_raw + ((1024u - (saddr(smem_raw) & 1023u)) & 1023u);

    const int NS = p.stages;  // K ring slots
    const uint32_t swz = (uint32_t)p.swz;
    const int atoms = p.row_bytes / p.swz;
    const uint32_t slot_bytes = (uint32_t)kBlockCols * swz;
    const int box_inner = p.swz / (KIND == 1 ? 4 : 2);
    constexpr bool MEASURE = MODE != kUpdate;
    constexpr bool FOLD = MODE != kStats;  // the bias enters the S product
    const SmemLayout L = smem_layout(p.row_bytes, NS, MODE, QT);

    uint8_t *sQ = smem + L.q;
    uint8_t *sK = smem + L.k;
    float *sBias = reinterpret_cast<float *>(smem + L.ones);  // statistics passes: fp32 bias slices
    float *sCN = reinterpret_cast<float *>(smem + L.cnorm);   // measure passes: |y|^2 or v slices
    float4 *sMerge = reinterpret_cast<float4 *>(smem + L.merge);
    double *sRed = reinterpret_cast<double *>(smem + L.red);
    uint32_t *koff = reinterpret_cast<uint32_t *>(smem + L.koff);
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + L.bars);  // [NS]
    uint64_t *empty = full + NS;                                   // [NS]
    uint64_t *rfull = empty + NS;                                  // [kBiasTiles] bias rows landed
    uint64_t *rempty = rfull + kBiasTiles;                         // [kBiasTiles] read by every job of the tile
    uint64_t *cfull = rempty + kBiasTiles;                         // [kBiasSlots] column slices landed
    uint64_t *cempty = cfull + kBiasSlots;                         // [kBiasSlots] read by the softmax warps
    uint64_t *qfull = cempty + kBiasSlots;
    uint64_t *sfull = qfull + 1;   // [2]
    uint64_t *sempty = sfull + 2;  // [2]
    uint64_t *drain = sempty + 2;
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(smem + L.misc);
    int *flag = reinterpret_cast<int *>(smem + L.misc + 4);  // [QT]
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + L.misc + 16);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int rb = blockIdx.x, split = blockIdx.y, bz = blockIdx.z;
    const int tile_begin = split * p.tiles_per_split;
    const int ntiles = min(p.tiles_per_split, p.col_tiles - tile_begin);
    const int njobs = ntiles * QT;

    if (threadIdx.x == 0) {
        for (int s = 0; s < NS; ++s) {
            mbar_init(full + s, 1);
            mbar_init(empty + s, QT);  // a commit after each of the tile's jobs
        }
        for (int j = 0; j < kBiasTiles; ++j) {
            mbar_init(rfull + j, 1);
            mbar_init(rempty + j, QT);  // a commit after each of the tile's jobs
        }
        for (int j = 0; j < kBiasSlots; ++j) {
            mbar_init(cfull + j, 1);
            mbar_init(cempty + j, 4 * QT);  // the warps of the softmax groups that read the tile
        }
        mbar_init(qfull, 1);
        for (int b = 0; b < 2; ++b) {
            mbar_init(sfull + b, 1);
            mbar_init(sempty + b, 4);
        }
        mbar_init(drain, p.issuers == 2 ? 2 : 1);
        {  // descriptor offsets of a tile's MMAs (A slice in the Q tile; B atom and offset)
            const uint32_t plane = (uint32_t)p.plane_bytes;
            const int ksteps = (int)(plane / 32u);
            for (int i = 0; i < NPASS * ksteps; ++i) {
                const int pass = i / ksteps, k = i % ksteps;
                // (A plane, B plane) = (hi,hi), (lo,hi), (hi,lo)
                const uint32_t ao = (pass == 1 ? plane : 0u) + 32u * k;
                const uint32_t bo = (pass == 2 ? plane : 0u) + 32u * k;
                koff[i] = ((ao / swz) * (kBlockRows * swz) + ao % swz) >> 4;
                koff[kMaxKsteps + i] = bo / swz;
                koff[2 * kMaxKsteps + i] = (bo % swz) >> 4;
            }
        }
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(saddr(tmem_holder)),
                     "r"(kTmemCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    if constexpr (FOLD) {
        // The A operand of the bias step: every row (1, 1, 1, 0, ...) in both 16-byte
        // halves, so the 32-byte swizzle (which may exchange the halves) leaves it as is.
        const uint32_t one2 = KIND == 1 ? 0x3F800000u : 0x3F803F80u;  // two bf16 ones, or one fp32 one
        const uint32_t w0 = one2, w1 = KIND == 1 ? 0x3F800000u : 0x3F80u, w2 = KIND == 1 ? 0x3F800000u : 0u;
        uint32_t *ones = reinterpret_cast<uint32_t *>(smem + L.ones);
        for (int i = threadIdx.x; i < kBlockRows * kBiasRowBytes / 4; i += blockDim.x) {
            const int w = i & 3;  // word within a 16-byte half
            ones[i] = w == 0 ? w0 : (w == 1 ? w1 : (w == 2 ? w2 : 0u));
        }
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_holder;

    if (warp == 0) {
        // ---------------- TMA producer ----------------
        if (lane == 0) {
            bool ok = true;
            int slots_issued = 0, rows_issued = 0, slices_issued = 0;
            const int qrow = bz * p.rows_pad + rb * (QT * kBlockRows);
            mbar_expect_tx(qfull, (uint32_t)(QT * kBlockRows) * p.row_bytes);
            for (int g = 0; g < QT; ++g)
                for (int a = 0; a < atoms; ++a)
                    tma_load_2d(saddr(sQ) + (g * atoms + a) * kBlockRows * swz, &map_rows, saddr(qfull),
                                a * box_inner, qrow + g * kBlockRows);
            const uint32_t bias_bytes = kBlockCols * 4;
            const uint32_t brow_tile = kBlockCols * kBiasRowBytes;
            for (int t = 0; ok && t < ntiles; ++t) {
                const int col0 = (tile_begin + t) * kBlockCols;
                if (*abort_flag) break;
                for (int a = 0; a < atoms; ++a) {
                    const int i = t * atoms + a;
                    const int s = i % NS;
                    if (i >= NS && !mbar_wait(empty + s, ((uint32_t)(i / NS) & 1u) ^ 1u, p.timeout_ns)) {
                        ok = false;
                        break;
                    }
                    mbar_expect_tx(full + s, slot_bytes);
                    tma_load_2d(saddr(sK + (size_t)s * slot_bytes), &map_cols, saddr(full + s), a * box_inner,
                                bz * p.cols_rows + col0);
                    slots_issued = i + 1;
                }
                if (!ok) break;
                // the tile's bias rows and column slices, after its K slots so they never delay them
                if constexpr (FOLD) {  // bias rows: 256 x 32 bytes, 32-byte swizzle
                    const int j = t % kBiasTiles;
                    if (t >= kBiasTiles &&
                        !mbar_wait(rempty + j, ((uint32_t)(t / kBiasTiles) & 1u) ^ 1u, p.timeout_ns)) {
                        ok = false;
                        break;
                    }
                    mbar_expect_tx(rfull + j, brow_tile);
                    tma_load_2d(saddr(smem + L.bias + j * brow_tile), &map_bias, saddr(rfull + j), 0,
                                bz * p.cols_stride + col0);
                    rows_issued = t + 1;
                }
                if constexpr (MEASURE) {  // fp32 slices: bias and |y|^2 (statistics), or v (vector)
                    const int j = t % kBiasSlots;
                    if (t >= kBiasSlots &&
                        !mbar_wait(cempty + j, ((uint32_t)(t / kBiasSlots) & 1u) ^ 1u, p.timeout_ns)) {
                        ok = false;
                        break;
                    }
                    mbar_expect_tx(cfull + j, bias_bytes * (MODE == kStats ? 2 : 1));
                    if constexpr (MODE == kStats) {
                        bulk_load(saddr(sBias + j * kBlockCols), p.col_bias + (size_t)bz * p.cols_stride + col0,
                                  bias_bytes, saddr(cfull + j));
                        bulk_load(saddr(sCN + j * kBlockCols), p.col_norm + (size_t)bz * p.cols_stride + col0,
                                  bias_bytes, saddr(cfull + j));
                    } else {
                        bulk_load(saddr(sCN + j * kBlockCols), p.col_vec + (size_t)bz * p.cols_stride + col0,
                                  bias_bytes, saddr(cfull + j));
                    }
                    slices_issued = t + 1;
                }
            }
            if (!ok) {
                atomicOr(p.err, kDevErrTimeout);
                *abort_flag = 1;
            }
            // Never leave with copies in flight: wait for every copy not yet consumed.
            mbar_wait(qfull, 0, p.timeout_ns);
            for (int i = max(0, slots_issued - NS); i < slots_issued; ++i)
                mbar_wait(full + (i % NS), (uint32_t)(i / NS) & 1u, p.timeout_ns);
            for (int t = max(0, rows_issued - kBiasTiles); t < rows_issued; ++t)
                mbar_wait(rfull + (t % kBiasTiles), (uint32_t)(t / kBiasTiles) & 1u, p.timeout_ns);
            for (int t = max(0, slices_issued - kBiasSlots); t < slices_issued; ++t)
                mbar_wait(cfull + (t % kBiasSlots), (uint32_t)(t / kBiasSlots) & 1u, p.timeout_ns);
        }
        __syncwarp();
    } else if (warp == 1 || (warp == 10 && p.issuers == 2)) {  // (the launcher admits 1 or 2)
        // ---------------- MMA issuer(s) ----------------
        // One thread issues every job, or (issuers = 2) warp 1 the even jobs
        // (TMEM buffer 0) and warp 10 the odd ones (buffer 1).
        if (lane == 0) {
            const uint32_t idesc = make_idesc<KIND>();
            const int nk = NPASS * (p.plane_bytes / 32);
            const int jstep = p.issuers == 2 ? 2 : 1, jb0 = warp == 1 ? 0 : 1;
            const uint64_t adesc0 = make_sdesc(saddr(sQ), swz);
            const uint32_t qstride = (uint32_t)(atoms * kBlockRows * swz) >> 4;  // one Q tile, in descriptor units
            // the bias step: bf16 (or tf32) ones against the tile's bias rows
            constexpr int BK = KIND == 1 ? 1 : 0;
            const uint32_t idesc_b = make_idesc<BK>();
            const uint64_t ones_desc = make_sdesc(saddr(smem + L.ones), (uint32_t)kBiasRowBytes);
            bool ok = mbar_wait(qfull, 0, p.timeout_ns);
            uint64_t bdesc[kMaxAtoms], brow_desc = 0ull;
            for (int jb = jb0; ok && jb < njobs; jb += jstep) {
                const int b = jb & 1;
                const int t = QT == 2 ? (jb >> 1) : jb;
                const int qt = QT == 2 ? b : 0;
                if (jb >= 2 && !mbar_wait(sempty + b, ((uint32_t)(jb >> 1) & 1u) ^ 1u, p.timeout_ns)) {
                    ok = false;
                    break;
                }
                if (qt == 0 || jstep == 2) {  // tile t's K slots (the first job of the tile, or each job)
#pragma unroll
                    for (int a = 0; a < kMaxAtoms; ++a) {
                        if (a < atoms) {
                            const int i = t * atoms + a;
                            if (!mbar_wait(full + (i % NS), (uint32_t)(i / NS) & 1u, p.timeout_ns)) ok = false;
                            bdesc[a] = make_sdesc(saddr(sK + (size_t)(i % NS) * slot_bytes), swz);
                        } else {
                            bdesc[a] = 0ull;
                        }
                    }
                    if constexpr (FOLD) {
                        const int j = t % kBiasTiles;
                        if (!mbar_wait(rfull + j, (uint32_t)(t / kBiasTiles) & 1u, p.timeout_ns)) ok = false;
                        brow_desc = make_sdesc(saddr(smem + L.bias + j * kBlockCols * kBiasRowBytes),
                                               (uint32_t)kBiasRowBytes);
                    }
                }
                if (!ok || *abort_flag) break;
                tc_fence_after();
                const uint32_t dt = tmem_base + (uint32_t)(b * kBlockCols);
                const uint64_t adesc = adesc0 + (uint64_t)(qt * qstride);
                if constexpr (KS > 0) {
                    issue_s_tile<KIND, NPASS, KS, kBlockRows>(dt, adesc, bdesc, idesc);
                } else {
                    for (int i = 0; i < nk; ++i) {
                        const uint32_t ba = koff[kMaxKsteps + i];
                        const uint64_t bd = ba == 0 ? bdesc[0] : (ba == 1 ? bdesc[1] : (ba == 2 ? bdesc[2] : bdesc[3]));
                        tc_mma<KIND>(dt, adesc + koff[i], bd + koff[2 * kMaxKsteps + i], idesc, i > 0 ? 1u : 0u);
                    }
                }
                if constexpr (FOLD) tc_mma<BK>(dt, ones_desc, brow_desc, idesc_b, 1u);  // + beta_j / c
                // A commit per job for its softmax group, and one per K slot (and
                // bias tile): free once every job of its tile has read it (QT arrivals).
                tc_commit(saddr(sfull + b));
                for (int a = 0; a < atoms; ++a) tc_commit(saddr(empty + ((t * atoms + a) % NS)));
                if constexpr (FOLD) tc_commit(saddr(rempty + (t % kBiasTiles)));
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
    } else if (warp >= 2 && warp < 10) {
        // ---------------- softmax warps ----------------
        // Group 0 (warps 2..5) takes the even tiles, which the MMA writes to TMEM
        // buffer 0; group 1 (warps 6..9) the odd tiles in buffer 1.  The two
        // warps sharing an SM sub-partition therefore work on different tiles
        // and their exponentials interleave on the MUFU.
        const int q = warp & 3;          // TMEM lane quadrant this warp may access
        const int grp = (warp - 2) >> 2; // tile parity handled by this warp
        const int rl = q * 32 + lane;    // row within the block
        const int rblk = rb * QT + (QT == 2 ? grp : 0);  // this warp's 128-row block
        const float c = p.scale2;
        const float xn = MODE == kStats ? p.row_norm[(size_t)bz * p.rows_stride + rblk * kBlockRows + rl] : 0.f;
        float m = -INFINITY, l = 0.f, w = 0.f;
        const uint32_t taddr = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(grp * kBlockCols);
        bool ok = true;
        for (int jb = grp; jb < njobs; jb += 2) {
            const int t = QT == 2 ? (jb >> 1) : jb;
            const int j = t % kBiasSlots;
            if (!mbar_wait(sfull + grp, (uint32_t)(jb >> 1) & 1u, p.timeout_ns) ||
                (MEASURE && !mbar_wait(cfull + j, (uint32_t)(t / kBiasSlots) & 1u, p.timeout_ns))) {
                ok = false;
                break;
            }
            tc_fence_after();
            if constexpr (FOLD) {
#pragma unroll 1
                for (int half = 0; half < 2; ++half) {
                    uint32_t r[128];
                    const uint32_t ta = taddr + 128u * half;
                    tmem_ld32(ta + 0u, &r[0]);
                    tmem_ld32(ta + 32u, &r[32]);
                    tmem_ld32(ta + 64u, &r[64]);
                    tmem_ld32(ta + 96u, &r[96]);
                    tmem_ld_wait();
                    if (half == 1) {  // the accumulator may now take the next tile
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive(sempty + grp);
                    }
                    if constexpr (MODE == kUpdate)
                        consume128_folded(r, c, m, l);
                    else  // w = sum_j 2^(z_j - m) v_j beside (m, l)
                        consume128_vec_folded(r, sCN + j * kBlockCols + 128 * half, c, m, l, w);
                }
                if constexpr (MODE == kVector) {
                    __syncwarp();
                    if (lane == 0) mbar_arrive(cempty + j);
                }
            } else {
                const float *bias = sBias + j * kBlockCols;
                const float *cnorm = sCN + j * kBlockCols;
#pragma unroll 1
                for (int qt = 0; qt < 4; ++qt) {
                    uint32_t ra[32], rb2[32];
                    tmem_ld32(taddr + 64u * qt, ra);
                    tmem_ld32(taddr + 64u * qt + 32u, rb2);
                    tmem_ld_wait();
                    if (qt == 3) {
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive(sempty + grp);
                    }
                    consume64_measure(ra, rb2, bias + 64 * qt, cnorm + 64 * qt, c, p.sscale, xn, m, l, w);
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(cempty + j);
            }
            if (*abort_flag) break;
        }
        if (!ok) {
            atomicOr(p.err, kDevErrTimeout);
            *abort_flag = 1;
        }
        if (QT == 1) {
            // Merge the two tile-parity groups' states of each row, then finish the row block.
            if (grp == 1) sMerge[rl] = make_float4(m, l, w, 0.f);
            named_barrier(1, 256);
            if (grp == 0) {
                const float4 o = sMerge[rl];
                lse_merge(m, l, w, o.x, o.y, o.z);
                finish_rows<MEASURE>(p, rblk, rl, m, l, w, 2, sRed, flag);
            }
        } else {
            // Each group holds whole rows of its own row block.
            finish_rows<MEASURE>(p, rblk, rl, m, l, w, 2 + grp, sRed + grp * 4 * kBlockRows, flag + grp);
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

template <int KIND, int NPASS, int MODE, int QT, int KS>
cudaError_t launch_variant(const PassParams &p, int batch, const void *map_rows, const void *map_cols,
                           const void *map_bias, size_t smem, cudaStream_t s) {
    auto kern = lse_tc_kernel<KIND, NPASS, MODE, QT, KS>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    dim3 grid(p.rows_pad / (QT * kBlockRows), p.splits, batch);
    kern<<<grid, kThreads, smem, s>>>(*static_cast<const CUtensorMap *>(map_rows),
                                      *static_cast<const CUtensorMap *>(map_cols),
                                      *static_cast<const CUtensorMap *>(map_bias), p);
    return cudaGetLastError();
}

// The compile-time row geometry matches the pass's packed rows.
template <int NPASS, int KS, typename Params>
bool fits(const Params &p) {
    return p.row_bytes == RowGeom<NPASS, KS>::kRowBytes && p.swz == RowGeom<NPASS, KS>::kSwz;
}

template <int KIND, int NPASS, int MODE, int KS>
cudaError_t launch_qt(const PassParams &p, int batch, int qt, const void *map_rows, const void *map_cols,
                      const void *map_bias, size_t smem, cudaStream_t s) {
    return qt == 2 ? launch_variant<KIND, NPASS, MODE, 2, KS>(p, batch, map_rows, map_cols, map_bias, smem, s)
                   : launch_variant<KIND, NPASS, MODE, 1, KS>(p, batch, map_rows, map_cols, map_bias, smem, s);
}

// The update and vector passes of the usual widths issue their MMAs from
// compile-time offsets (d = 16, 32, 64 and, for one-plane modes, 128 values per plane).
template <int KIND, int NPASS, int MODE>
cudaError_t launch_ks(const PassParams &p, int batch, int qt, const void *map_rows, const void *map_cols,
                      const void *map_bias, size_t smem, cudaStream_t s) {
    const int ks = p.plane_bytes / 32;
    if (ks * 32 == p.plane_bytes) {
        if (ks == 1 && fits<NPASS, 1>(p)) return launch_qt<KIND, NPASS, MODE, 1>(p, batch, qt, map_rows, map_cols, map_bias, smem, s);
        if (ks == 2 && fits<NPASS, 2>(p)) return launch_qt<KIND, NPASS, MODE, 2>(p, batch, qt, map_rows, map_cols, map_bias, smem, s);
        if (ks == 4 && fits<NPASS, 4>(p)) return launch_qt<KIND, NPASS, MODE, 4>(p, batch, qt, map_rows, map_cols, map_bias, smem, s);
        if constexpr (NPASS == 1)
            if (ks == 8 && fits<NPASS, 8>(p)) return launch_qt<KIND, NPASS, MODE, 8>(p, batch, qt, map_rows, map_cols, map_bias, smem, s);
    }
    return launch_qt<KIND, NPASS, MODE, 0>(p, batch, qt, map_rows, map_cols, map_bias, smem, s);
}

template <int KIND, int NPASS>
cudaError_t launch_kind(const PassParams &p, int batch, bool measure, int qt, const void *map_rows,
                        const void *map_cols, const void *map_bias, size_t smem, cudaStream_t s) {
    if (!measure) return launch_ks<KIND, NPASS, kUpdate>(p, batch, qt, map_rows, map_cols, map_bias, smem, s);
    if (p.col_vec) return launch_ks<KIND, NPASS, kVector>(p, batch, qt, map_rows, map_cols, map_bias, smem, s);
    return launch_qt<KIND, NPASS, kStats, 0>(p, batch, qt, map_rows, map_cols, map_bias, smem, s);
}

}  // namespace

// measure: the larger of the statistics and the vector layouts (one size serves both).
size_t tc_smem_bytes(int row_bytes, int qt, int slots, bool measure) {
    uint32_t total = smem_layout(row_bytes, slots, kUpdate, qt).total;
    if (measure) {
        const uint32_t a = smem_layout(row_bytes, slots, kStats, qt).total;
        const uint32_t b = smem_layout(row_bytes, slots, kVector, qt).total;
        total = a > b ? a : b;
    }
    return (size_t)total + 1024;  // + alignment slack
}

// The deepest K ring that fits (at most 8 slots) with qt resident Q tiles; 0
// if not even one tile plus one slot of look-ahead fits.
int tc_max_stages(int row_bytes, int qt, bool measure) {
    const size_t limit = 227 * 1024;
    const int atoms = row_bytes / swizzle_of(row_bytes);
    int best = 0;
    for (int s = atoms + 1; s <= 8; ++s)
        if (tc_smem_bytes(row_bytes, qt, s, measure) <= limit) best = s;
    return best;
}

// prec: 1 = bf16, 2 = tf32 (one pass), 3 = 3xTF32, 4 = 3xF16; qt: 128-row blocks per CTA (1 or 2);
// map_bias: the column side's bias rows (update and vector passes; store_bias_mm
// in the operand type of prec, 32-byte swizzle, boxes of 256 rows).
cudaError_t launch_lse_tc(const PassParams &p, int batch, bool measure, int prec, int qt, const void *map_rows,
                          const void *map_cols, const void *map_bias, size_t smem, cudaStream_t s) {
    if (p.issuers != 1 && p.issuers != 2) return cudaErrorInvalidValue;
    if (qt != 1 && qt != 2) return cudaErrorInvalidValue;
    if (prec == 1) return launch_kind<0, 1>(p, batch, measure, qt, map_rows, map_cols, map_bias, smem, s);
    if (prec == 2) return launch_kind<1, 1>(p, batch, measure, qt, map_rows, map_cols, map_bias, smem, s);
    if (prec == 3) return launch_kind<1, 3>(p, batch, measure, qt, map_rows, map_cols, map_bias, smem, s);
    return launch_kind<2, 3>(p, batch, measure, qt, map_rows, map_cols, map_bias, smem, s);
}

}  // namespace fs
