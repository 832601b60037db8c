// Streamed LSE pass on a CTA pair: one tcgen05 MMA spans two SMs.
//
// The same pass as fs_lse_tc.cu -- row-stationary traversal, online LSE in
// registers, one potential per row written (FlashSinkhorn Metodologia section
// 2) -- but the two CTAs of a cluster share every MMA (tcgen05.mma.cta_group::2,
// M = 256, N = 256).  Each CTA keeps its own 128 rows of Q and loads only half
// (128 rows) of every 256-column K tile; the pair's first CTA issues the MMA,
// which reads A and B from both CTAs' shared memory and writes each CTA's
// 128 x 256 block of S into that CTA's TMEM.  Each CTA spends only half the
// shared memory per K tile, which is what lets the rows of 512 bytes (3xTF32 at
// d = 64, TF32 and 3xF16 at d = 128) that no single-CTA ring can hold run on
// the tensor cores; FS_CTA_PAIR=1 selects it for every width.
//
// Synchronisation of the pair: both CTAs' TMA loads of a slot count on the
// first CTA's `full` barrier; the MMA's completion is committed to the `sfull`
// barriers of both CTAs at once (multicast commit), and each CTA's softmax
// groups then hand that CTA's K slots back; both CTAs' softmax groups release
// a TMEM buffer on the first CTA's `sempty` barrier.
// All waits are bounded as in the single-CTA kernel; both CTAs always reach
// the final cluster barrier, so neither leaves while the other may still read
// its shared memory or TMEM.
#include "fs_tc_common.cuh"

namespace fs {
namespace {

using namespace tc;

constexpr int kThreads = 320;
constexpr int kTmemCols = 512;   // two 256-column fp32 accumulators
constexpr int kMaxKsteps = 64;
constexpr int kMaxAtoms = 4;
constexpr int kBiasSlots = 8;  // more tiles than the K ring holds, so bias never gates the K loads
constexpr int kHalfCols = kBlockCols / 2;  // K rows of a tile held by each CTA

struct SmemLayout2 {
    uint32_t q, k, bias, cnorm, merge, red, koff, bars, misc, total;
};

__host__ __device__ inline int swizzle_of2(int row_bytes) { return row_bytes <= 32 ? 32 : (row_bytes <= 64 ? 64 : 128); }

// slots: K ring slots of kHalfCols rows x one swizzle atom each.
__host__ __device__ inline SmemLayout2 smem_layout2(int row_bytes, int slots, bool measure) {
    SmemLayout2 L;
    const uint32_t swz = (uint32_t)swizzle_of2(row_bytes);
    L.q = 0;
    L.k = (uint32_t)kBlockRows * row_bytes;
    L.bias = L.k + (uint32_t)slots * kHalfCols * swz;
    L.cnorm = L.bias + kBiasSlots * kBlockCols * 4;
    L.merge = L.cnorm + (measure ? kBiasSlots * kBlockCols * 4 : 0);
    L.red = L.merge + kBlockRows * 16;
    L.koff = L.red + 4 * kBlockRows * 8;
    L.bars = L.koff + 3 * kMaxKsteps * 4;
    L.misc = L.bars + (2 * slots + 2 * kBiasSlots + 6) * 8;
    L.total = L.misc + 16;
    return L;
}

// KS > 0: the K-step count of an operand plane, fixed at compile time
// (immediate descriptor offsets); KS = 0: any width, offsets from a table.
template <int KIND, int NPASS, bool MEASURE, int KS>
__global__ void __launch_bounds__(kThreads, 1)
    lse_tc2_kernel(const __grid_constant__ CUtensorMap map_rows, const __grid_constant__ CUtensorMap map_cols,
                   const PassParams p) {
    extern __shared__ uint8_t smem_raw[];
    // The offset must be the same in both CTAs (MMA operands and barriers are
    // addressed by offset in the peer): the dynamic shared window starts at the
    // same address in every CTA of a kernel, so the alignment pad is equal.
    uint8_t *smem = smem_raw + ((1024u - (saddr(smem_raw) & 1023u)) & 1023u);

    const int NS = p.stages;
    const uint32_t swz = (uint32_t)p.swz;
    const int atoms = p.row_bytes / p.swz;
    const uint32_t slot_bytes = (uint32_t)kHalfCols * swz;
    const uint32_t q_bytes = (uint32_t)kBlockRows * p.row_bytes;
    const int box_inner = p.swz / (KIND == 1 ? 4 : 2);
    const SmemLayout2 L = smem_layout2(p.row_bytes, NS, MEASURE);

    uint8_t *sQ = smem + L.q;
    uint8_t *sK = smem + L.k;
    float *sBias = reinterpret_cast<float *>(smem + L.bias);
    float *sCN = reinterpret_cast<float *>(smem + L.cnorm);
    float4 *sMerge = reinterpret_cast<float4 *>(smem + L.merge);
    double *sRed = reinterpret_cast<double *>(smem + L.red);
    uint32_t *koff = reinterpret_cast<uint32_t *>(smem + L.koff);
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + L.bars);  // [NS]   used in the first CTA
    uint64_t *empty = full + NS;                                   // [NS]   both CTAs
    uint64_t *bfull = empty + NS;                                  // [kBiasSlots] local
    uint64_t *bempty = bfull + kBiasSlots;                         // [kBiasSlots] local
    uint64_t *qfull = bempty + kBiasSlots;                         // first CTA
    uint64_t *sfull = qfull + 1;                                   // [2] both CTAs
    uint64_t *sempty = sfull + 2;                                  // [2] first CTA (8 arrivals)
    uint64_t *drain = sempty + 2;
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(smem + L.misc);
    int *flag = reinterpret_cast<int *>(smem + L.misc + 4);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + L.misc + 8);

    const uint32_t rank = cluster_rank();  // 0: the CTA that issues the pair's MMAs
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int rb = blockIdx.x, split = blockIdx.y, bz = blockIdx.z;
    const int tile_begin = split * p.tiles_per_split;
    const int ntiles = min(p.tiles_per_split, p.col_tiles - tile_begin);

    if (threadIdx.x == 0) {
        for (int s = 0; s < NS; ++s) {
            mbar_init(full + s, 1);
            mbar_init(empty + s, 1);
        }
        for (int j = 0; j < kBiasSlots; ++j) {
            mbar_init(bfull + j, 1);
            mbar_init(bempty + j, 4);
        }
        mbar_init(qfull, 1);
        for (int b = 0; b < 2; ++b) {
            mbar_init(sfull + b, 1);
            mbar_init(sempty + b, 8);  // four softmax warps in each CTA of the pair
        }
        mbar_init(drain, 1);
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(saddr(tmem_holder)),
                     "r"(kTmemCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    cluster_sync();  // barriers of both CTAs initialised before any cross-CTA signal
    tc_fence_after();
    const uint32_t tmem_base = *tmem_holder;

    if (warp == 0) {
        // ---------------- TMA producer (both CTAs) ----------------
        if (lane == 0) {
            bool ok = true;
            int slots_issued = 0, bias_issued = 0;
            const uint32_t qbar0 = cluster_addr(saddr(qfull), 0);
            if (rank == 0) mbar_expect_tx(qfull, 2u * q_bytes);
            for (int a = 0; a < atoms; ++a)
                tma_load_2d_pair(saddr(sQ) + a * kBlockRows * swz, &map_rows, qbar0, a * box_inner,
                                 bz * p.rows_pad + rb * kBlockRows);
            const uint32_t bias_bytes = kBlockCols * 4;
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
                    if (rank == 0) mbar_expect_tx(full + s, 2u * slot_bytes);
                    tma_load_2d_pair(saddr(sK + (size_t)s * slot_bytes), &map_cols, cluster_addr(saddr(full + s), 0),
                                     a * box_inner, bz * p.cols_rows + col0 + (int)rank * kHalfCols);
                    slots_issued = i + 1;
                }
                if (!ok) break;
                const int j = t % kBiasSlots;
                if (t >= kBiasSlots && !mbar_wait(bempty + j, ((uint32_t)(t / kBiasSlots) & 1u) ^ 1u, p.timeout_ns)) {
                    ok = false;
                    break;
                }
                mbar_expect_tx(bfull + j, bias_bytes * (MEASURE ? 2 : 1));
                bulk_load(saddr(sBias + j * kBlockCols), p.col_bias + (size_t)bz * p.cols_stride + col0, bias_bytes,
                          saddr(bfull + j));
                if (MEASURE)
                    bulk_load(saddr(sCN + j * kBlockCols),
                              (p.col_vec ? p.col_vec : p.col_norm) + (size_t)bz * p.cols_stride + col0, bias_bytes,
                              saddr(bfull + j));
                bias_issued = t + 1;
            }
            if (!ok) {
                atomicOr(p.err, kDevErrTimeout);
                *abort_flag = 1;
            }
            // Never leave with copies in flight.  Both CTAs' slot and Q copies
            // count on the first CTA's barriers, so that CTA waits for them; each
            // CTA waits for its own bias copies.
            if (rank == 0) {
                mbar_wait(qfull, 0, p.timeout_ns);
                for (int i = max(0, slots_issued - NS); i < slots_issued; ++i)
                    mbar_wait(full + (i % NS), (uint32_t)(i / NS) & 1u, p.timeout_ns);
            }
            for (int t = max(0, bias_issued - kBiasSlots); t < bias_issued; ++t)
                mbar_wait(bfull + (t % kBiasSlots), (uint32_t)(t / kBiasSlots) & 1u, p.timeout_ns);
        }
        __syncwarp();
    } else if (warp == 1) {
        // ---------------- MMA issuer (first CTA of the pair) ----------------
        if (lane == 0 && rank == 0) {
            const uint32_t idesc = make_idesc<KIND, 2 * kBlockRows>();
            const uint32_t plane = (uint32_t)p.plane_bytes;
            const int ksteps = (int)(plane / 32u);
            const int nk = NPASS * ksteps;
            for (int i = 0; i < nk; ++i) {
                const int pass = i / ksteps, k = i % ksteps;
                // (A plane, B plane) = (hi,hi), (lo,hi), (hi,lo)
                const uint32_t ao = (pass == 1 ? plane : 0u) + 32u * k;
                const uint32_t bo = (pass == 2 ? plane : 0u) + 32u * k;
                koff[i] = ((ao / swz) * (kBlockRows * swz) + ao % swz) >> 4;
                koff[kMaxKsteps + i] = bo / swz;
                koff[2 * kMaxKsteps + i] = (bo % swz) >> 4;
            }
            const uint64_t adesc0 = make_sdesc(saddr(sQ), swz);
            bool ok = mbar_wait(qfull, 0, p.timeout_ns);
            for (int t = 0; ok && t < ntiles; ++t) {
                const int b = t & 1;
                if (t >= 2 && !mbar_wait_cluster(sempty + b, ((uint32_t)(t >> 1) & 1u) ^ 1u, p.timeout_ns)) {
                    ok = false;
                    break;
                }
                uint64_t bdesc[kMaxAtoms];
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
                if (!ok || *abort_flag) break;
                tc_fence_after();
                const uint32_t dt = tmem_base + (uint32_t)(b * kBlockCols);
                if constexpr (KS > 0) {
                    issue_s_tile<KIND, NPASS, KS, kBlockRows, true>(dt, adesc0, bdesc, idesc);
                } else {
                    for (int i = 0; i < nk; ++i) {
                        const uint32_t ba = koff[kMaxKsteps + i];
                        const uint64_t bd = ba == 0 ? bdesc[0] : (ba == 1 ? bdesc[1] : (ba == 2 ? bdesc[2] : bdesc[3]));
                        tc_mma_pair<KIND>(dt, adesc0 + koff[i], bd + koff[2 * kMaxKsteps + i], idesc,
                                          i > 0 ? 1u : 0u);
                    }
                }
                // One commit per tile (a commit stalls the MMA pipe): the softmax
                // groups of both CTAs hand the tile's K slots back when it lands.
                tc_commit_pair(saddr(sfull + b), (uint16_t)3);
            }
            if (!ok) {
                atomicOr(p.err, kDevErrTimeout);
                *abort_flag = 1;
            }
            // Drain every MMA of the pair before either CTA releases TMEM.
            tc_commit_pair(saddr(drain), (uint16_t)1);
            mbar_wait(drain, 0, p.timeout_ns);
        }
        __syncwarp();
    } else {
        // ---------------- softmax warps (both CTAs) ----------------
        const int q = warp & 3;
        const int grp = (warp - 2) >> 2;
        const int rl = q * 32 + lane;
        const float c = p.scale2;
        // a vector pass weights each column by v_j alone: no row norm, no score term
        const float xn = MEASURE && !p.col_vec ? p.row_norm[(size_t)bz * p.rows_stride + rb * kBlockRows + rl] : 0.f;
        const float wsscale = p.col_vec ? 0.f : p.sscale;
        float m = -INFINITY, l = 0.f, w = 0.f;
        const uint32_t taddr = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(grp * kBlockCols);
        const uint32_t sempty0 = cluster_addr(saddr(sempty + grp), 0);
        bool ok = true;
        for (int t = grp; t < ntiles; t += 2) {
            const int j = t % kBiasSlots;
            if (!mbar_wait(sfull + grp, (uint32_t)(t >> 1) & 1u, p.timeout_ns) ||
                !mbar_wait(bfull + j, (uint32_t)(t / kBiasSlots) & 1u, p.timeout_ns)) {
                ok = false;
                break;
            }
            tc_fence_after();
            if (q == 2 && lane == 0)  // the pair's MMAs of tile t are complete: this CTA's K slots are free
                for (int a = 0; a < atoms; ++a) mbar_arrive(empty + ((t * atoms + a) % NS));
            const float *bias = sBias + j * kBlockCols;
            if (!MEASURE) {
#pragma unroll 1
                for (int half = 0; half < 2; ++half) {
                    uint32_t r[128];
                    const uint32_t ta = taddr + 128u * half;
                    tmem_ld32(ta + 0u, &r[0]);
                    tmem_ld32(ta + 32u, &r[32]);
                    tmem_ld32(ta + 64u, &r[64]);
                    tmem_ld32(ta + 96u, &r[96]);
                    tmem_ld_wait();
                    if (half == 1) {
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive_cluster(sempty0);
                    }
                    consume128(r, bias + 128 * half, c, m, l);
                }
            } else {
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
                        if (lane == 0) mbar_arrive_cluster(sempty0);
                    }
                    consume64_measure(ra, rb2, bias + 64 * qt, cnorm + 64 * qt, c, wsscale, xn, m, l, w);
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(bempty + j);
            if (*abort_flag) break;
        }
        if (!ok) {
            atomicOr(p.err, kDevErrTimeout);
            *abort_flag = 1;
        }
        if (grp == 1) sMerge[rl] = make_float4(m, l, w, 0.f);
        named_barrier(1, 256);
        if (grp == 0) {
            const float4 o = sMerge[rl];
            lse_merge(m, l, w, o.x, o.y, o.z);
            finish_rows<MEASURE>(p, blockIdx.x, rl, m, l, w, 2, sRed, flag);
        }
    }

    tc_fence_before();
    __syncthreads();
    cluster_sync();  // neither CTA leaves while the pair's MMAs or the peer may touch its memory
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(kTmemCols)
                     : "memory");
    }
}

template <int KIND, int NPASS, bool MEASURE, int KS>
cudaError_t launch_variant2(const PassParams &p, int batch, const void *map_rows, const void *map_cols,
                            size_t smem, cudaStream_t s) {
    auto kern = lse_tc2_kernel<KIND, NPASS, MEASURE, KS>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(p.rows_pad / kBlockRows, p.splits, batch);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, kern, *static_cast<const CUtensorMap *>(map_rows),
                           *static_cast<const CUtensorMap *>(map_cols), p);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

// The 512-byte rows this kernel exists for (one plane of 256 values, or hi/lo
// planes of 128) take the update passes with compile-time offsets.
template <int KIND, int NPASS>
cudaError_t launch_kind2(const PassParams &p, int batch, bool measure, const void *map_rows, const void *map_cols,
                         size_t smem, cudaStream_t s) {
    if (measure) return launch_variant2<KIND, NPASS, true, 0>(p, batch, map_rows, map_cols, smem, s);
    constexpr int kWideKs = NPASS == 1 ? 16 : 8;
    if (p.plane_bytes == 32 * kWideKs && p.row_bytes == RowGeom<NPASS, kWideKs>::kRowBytes &&
        p.swz == RowGeom<NPASS, kWideKs>::kSwz)
        return launch_variant2<KIND, NPASS, false, kWideKs>(p, batch, map_rows, map_cols, smem, s);
    return launch_variant2<KIND, NPASS, false, 0>(p, batch, map_rows, map_cols, smem, s);
}

}  // namespace

size_t tc2_smem_bytes(int row_bytes, int slots, bool measure) {
    return (size_t)smem_layout2(row_bytes, slots, measure).total + 1024;
}

// Deepest K ring (at most 12 slots of 128 rows) that fits; 0 if not even one
// tile plus one slot of look-ahead fits.
int tc2_max_stages(int row_bytes, bool measure) {
    const size_t limit = 227 * 1024;
    const int atoms = row_bytes / swizzle_of2(row_bytes);
    int best = 0;
    for (int s = atoms + 1; s <= 12; ++s)
        if (tc2_smem_bytes(row_bytes, s, measure) <= limit) best = s;
    return best;
}

// prec: 1 = bf16, 2 = tf32 (one pass), 3 = 3xTF32, 4 = 3xF16.  rows_pad / 128 must be even.
cudaError_t launch_lse_tc2(const PassParams &p, int batch, bool measure, int prec, const void *map_rows,
                           const void *map_cols, size_t smem, cudaStream_t s) {
    if (prec == 1) return launch_kind2<0, 1>(p, batch, measure, map_rows, map_cols, smem, s);
    if (prec == 2) return launch_kind2<1, 1>(p, batch, measure, map_rows, map_cols, smem, s);
    if (prec == 3) return launch_kind2<1, 3>(p, batch, measure, map_rows, map_cols, smem, s);
    return launch_kind2<2, 3>(p, batch, measure, map_rows, map_cols, smem, s);
}

}  // namespace fs
