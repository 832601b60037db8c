// Device helpers shared by the tensor-core LSE passes: mbarrier, TMA and
// tcgen05 wrappers, shared-memory matrix descriptors, and the per-row online
// LSE update of the softmax warps.
#pragma once

#include <cuda.h>

#include "fs_finish.cuh"

namespace fs {
namespace tc {

// Lazy rescaling of a row's running maximum: a block whose exponentials, taken
// against the running max, sum to more than 2^12 forces the rescale; smaller
// sums (every entry at most 12 above the running max) join the running sum as
// they are.
constexpr float kLazySum = 4096.f;

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
// D (TMEM) (+)= A (shared memory) x B^T (shared memory), both K-major.
template <int KIND>
__device__ __forceinline__ void tc_mma(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                       uint32_t accum) {
    if constexpr (KIND != 1) {
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
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t *r) {
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
// Store 32 consecutive 32-bit columns of this warp's 32 TMEM lanes (the mirror of tmem_ld32).
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t *r) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
        "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, "
        "%17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]),
        "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]),
        "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]),
        "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
        : "memory");
}
__device__ __forceinline__ void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }
// D (+)= A B^T, kind::f16, with A read from TMEM (M = 128 lanes; 16-bit elements
// in pairs, two per 32-bit column, so one K step of 16 spans 8 columns) and B
// from shared memory through its descriptor.
__device__ __forceinline__ void tc_mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc, uint32_t idesc,
                                          uint32_t accum) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
        "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accum)
        : "memory");
}

// Shared-memory matrix descriptor of a K-major operand stored as swizzle
// atoms: 8-row groups are `8 * swz` bytes apart (stride byte offset), the
// leading byte offset is unused for swizzled K-major layouts, bits 46-47 hold
// the sm_100 descriptor version (1), bits 61-63 the swizzle mode.  Adding n to
// the descriptor moves its start address by 16 n bytes.
__device__ __forceinline__ uint64_t make_sdesc(uint32_t addr, uint32_t swz) {
    const uint64_t layout = swz == 128 ? 2ull : (swz == 64 ? 4ull : 6ull);
    uint64_t desc = (uint64_t)((addr >> 4) & 0x3FFFu);
    desc |= (uint64_t)1u << 16;
    desc |= (uint64_t)(((8u * swz) >> 4) & 0x3FFFu) << 32;
    desc |= (uint64_t)1u << 46;
    desc |= layout << 61;
    return desc;
}

// Instruction descriptor: fp32 accumulator, A/B format (kind::f16: 0 = fp16,
// 1 = bf16; kind::tf32: 2), both K-major, M rows (128, or 256 for a CTA pair),
// N = 256.
template <int KIND, int M = kBlockRows, int N = kBlockCols>
__device__ __forceinline__ uint32_t make_idesc() {
    const uint32_t fmt = KIND == 0 ? 1u : (KIND == 1 ? 2u : 0u);
    return (1u << 4) | (fmt << 7) | (fmt << 10) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

// ---- CTA pairs (cluster of two CTAs on two SMs sharing one MMA) -------------
__device__ __forceinline__ uint32_t cluster_rank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
__device__ __forceinline__ void cluster_sync() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// Shared::cluster address of the same shared-memory offset in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t cluster_addr(uint32_t local_saddr, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(local_saddr), "r"(rank));
    return r;
}
// Bounded wait with cluster-scope acquire, for barriers that other CTAs arrive on.
__device__ __forceinline__ bool mbar_wait_cluster(uint64_t *b, uint32_t parity, unsigned long long limit_ns) {
    const unsigned long long t0 = globaltimer_ns();
    while (true) {
        uint32_t done;
        asm volatile(
            "{\n\t.reg .pred P;\n\t"
            "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 P, [%1], %2;\n\t"
            "selp.b32 %0, 1, 0, P;\n\t}"
            : "=r"(done)
            : "r"(saddr(b)), "r"(parity)
            : "memory");
        if (done) return true;
        if (globaltimer_ns() - t0 > limit_ns) return false;
    }
}
// Arrive on an mbarrier of another CTA of the cluster.  Used after
// tcgen05.wait::ld to hand a TMEM buffer back: the TMEM reads are complete,
// no memory written by this thread needs to become visible, so the default
// CTA-scope release suffices.
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_bar) {
    asm volatile("mbarrier.arrive.shared::cluster.b64 _, [%0];" ::"r"(cluster_bar) : "memory");
}
// Arrive on an mbarrier of another CTA of the cluster, releasing at cluster
// scope what this thread wrote before (shared-memory operands that the peer's
// tensor-core instructions will read, after fence.proxy.async).
__device__ __forceinline__ void mbar_arrive_cluster_release(uint32_t cluster_bar) {
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_bar) : "memory");
}
// TMA box load into this CTA's shared memory whose completion is counted on
// an mbarrier of either CTA of the pair (here: the pair's first CTA).
__device__ __forceinline__ void tma_load_2d_pair(uint32_t dst, const void *map, uint32_t cluster_bar, int x, int y) {
    asm volatile(
        "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
        "l"(map), "r"(x), "r"(y), "r"(cluster_bar)
        : "memory");
}
// D (+)= A x B^T over the CTA pair: A rows 0..127 and B rows 0..127 from the
// first CTA's shared memory, A rows 128..255 and B rows 128..255 from the
// second CTA's (same offsets); each CTA's TMEM receives its 128 rows x N.
template <int KIND>
__device__ __forceinline__ void tc_mma_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                            uint32_t accum) {
    if constexpr (KIND != 1) {
        asm volatile(
            "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
            "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
            "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accum)
            : "memory");
    } else {
        asm volatile(
            "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
            "tcgen05.mma.cta_group::2.kind::tf32 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
            "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accum)
            : "memory");
    }
}
// Arrive on the mbarrier at this offset in every CTA of `cta_mask` once all
// MMAs issued so far by this thread have completed.
__device__ __forceinline__ void tc_commit_pair(uint32_t local_bar, uint16_t cta_mask) {
    asm volatile(
        "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
            local_bar),
        "h"(cta_mask)
        : "memory");
}

// Geometry of a packed operand row whose plane holds KS K-steps of 32 bytes
// and which carries one plane (NPASS = 1) or hi and lo planes (NPASS = 3),
// known at compile time; the host packs rows by the same rule.
template <int NPASS, int KS>
struct RowGeom {
    static constexpr int kPlane = 32 * KS;
    static constexpr int kUsed = (NPASS == 3 ? 2 : 1) * kPlane;
    static constexpr int kRowBytes = kUsed <= 32 ? 32 : (kUsed <= 64 ? 64 : (kUsed + 127) / 128 * 128);
    static constexpr int kSwz = kRowBytes <= 32 ? 32 : (kRowBytes <= 64 ? 64 : 128);
    static constexpr int kAtoms = kRowBytes / kSwz;
};

// The MMAs of one S tile, D (+)= A x B^T over the row's K-steps (and, for
// NPASS = 3, the products (hi, hi), (lo, hi), (hi, lo) of the split planes).
// A: AROWS-row tile of K-major swizzle atoms at adesc; B: one ring slot per
// atom, bdesc[atom].  Every descriptor is a per-tile base plus an immediate:
// an issue loop whose offsets are run-time values (a table in shared memory, or
// arithmetic on a loop counter) spends far longer per instruction than the
// tensor pipe needs for the MMA itself.
// PAIR: one tcgen05.mma.cta_group::2 per K-step over a CTA pair (same
// shared-memory offsets in both CTAs).  The wrapper is defined below.
template <int KIND>
__device__ __forceinline__ void tc_mma_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                            uint32_t accum);
// ONTO: accumulate onto what D holds already (else the first MMA starts D afresh).
template <int KIND, int NPASS, int KS, int AROWS, bool PAIR = false, bool ONTO = false>
__device__ __forceinline__ void issue_s_tile(uint32_t d_tmem, uint64_t adesc, const uint64_t (&bdesc)[4],
                                             uint32_t idesc) {
    using G = RowGeom<NPASS, KS>;
#pragma unroll
    for (int i = 0; i < NPASS * KS; ++i) {
        const int pass = i / KS, k = i % KS;
        const int ao = (pass == 1 ? G::kPlane : 0) + 32 * k;
        const int bo = (pass == 2 ? G::kPlane : 0) + 32 * k;
        const uint64_t ad = adesc + (uint64_t)(((ao / G::kSwz) * (AROWS * G::kSwz) + ao % G::kSwz) >> 4);
        const uint64_t bd = bdesc[bo / G::kSwz] + (uint64_t)((bo % G::kSwz) >> 4);
        const uint32_t acc = (ONTO || i > 0) ? 1u : 0u;
        if constexpr (PAIR)
            tc_mma_pair<KIND>(d_tmem, ad, bd, idesc, acc);
        else
            tc_mma<KIND>(d_tmem, ad, bd, idesc, acc);
    }
}

// sum_k 2^(z_k - ref) over CNT columns, fp32 pairs.
template <int CNT>
__device__ __forceinline__ float sum_exp2(const float (&z)[CNT], float ref) {
    const uint64_t rn = pack2(-ref, -ref);
    uint64_t acc[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
    for (int k = 0; k < CNT; k += 2) {
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

// The block's max taken, (m, l) moved to max(m, block max) and the block's
// exponentials added against it (the rare path of the folds below).
template <int CNT>
__device__ __forceinline__ void rescale_block(const float (&z)[CNT], float &m, float &l) {
    float mx[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
    for (int k = 0; k < CNT; k += 8) {
        mx[(k / 8) & 3] = max3(mx[(k / 8) & 3], z[k], z[k + 1]);
        mx[(k / 8) & 3] = max3(mx[(k / 8) & 3], z[k + 2], z[k + 3]);
        mx[(k / 8) & 3] = max3(mx[(k / 8) & 3], z[k + 4], z[k + 5]);
        mx[(k / 8) & 3] = max3(mx[(k / 8) & 3], z[k + 6], z[k + 7]);
    }
    const float tmax = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3]));
    if (tmax == -INFINITY) return;  // nothing but padding so far
    const float mnew = fmaxf(m, tmax);
    l = (m == -INFINITY ? 0.f : l * ex2_approx(m - mnew)) + sum_exp2<CNT>(z, mnew);
    m = mnew;
}

// Fold CNT scores (raw fp32 bits from TMEM) into a row's online state (m, l):
// z = S * c + beta.  The first block of a row takes two passes (max, then
// exponentials).  Later blocks take their exponentials against the running max
// as it stood and add them up; only when that block sum exceeds 2^12 (which
// every entry more than 12 above the running max forces, and which an
// overflow to inf or a NaN also fails) is the block's max taken and the block
// redone against it.  The common case thus spends no instruction on the max.
template <int CNT>
__device__ __forceinline__ void consume(const uint32_t (&r)[CNT], const float *bias, float c, float &m, float &l) {
    const float4 *bq = reinterpret_cast<const float4 *>(bias);
    const uint64_t cc = pack2(c, c);
    float z[CNT];
#pragma unroll
    for (int k = 0; k < CNT; k += 4) {
        const float4 bb = bq[k / 4];
        unpack2(fma2(pack2(__uint_as_float(r[k]), __uint_as_float(r[k + 1])), cc, pack2(bb.x, bb.y)), z[k],
                z[k + 1]);
        unpack2(fma2(pack2(__uint_as_float(r[k + 2]), __uint_as_float(r[k + 3])), cc, pack2(bb.z, bb.w)), z[k + 2],
                z[k + 3]);
    }
    float s;
    if (m != -INFINITY) {
        const uint64_t mneg = pack2(-m, -m);
        uint64_t acc[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
        for (int k = 0; k < CNT; k += 2) {
            float d0, d1;
            unpack2(add2(pack2(z[k], z[k + 1]), mneg), d0, d1);
            acc[(k / 2) & 3] = add2(acc[(k / 2) & 3], pack2(ex2_approx(d0), ex2_approx(d1)));
        }
        float a0, a1, a2, a3, a4, a5, a6, a7;
        unpack2(acc[0], a0, a1);
        unpack2(acc[1], a2, a3);
        unpack2(acc[2], a4, a5);
        unpack2(acc[3], a6, a7);
        s = ((a0 + a1) + (a2 + a3)) + ((a4 + a5) + (a6 + a7));
        if (s <= kLazySum) {
            l += s;
            return;
        }
    }
    rescale_block<CNT>(z, m, l);
}
__device__ __forceinline__ void consume128(const uint32_t (&r)[128], const float *bias, float c, float &m,
                                           float &l) {
    consume<128>(r, bias, c, m, l);
}

// The same fold for scores that already hold the column bias (the update
// pass's S product adds beta_j / c, store_bias_mm): z = S' c, and the common
// case is one packed FMA (S' c - max) per two entries, then the exponentials.
template <int CNT>
__device__ __forceinline__ void consume_folded(const uint32_t (&r)[CNT], float c, float &m, float &l) {
    const uint64_t cc = pack2(c, c);
    if (m != -INFINITY) {
        const uint64_t mneg = pack2(-m, -m);
        uint64_t acc[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
        for (int k = 0; k < CNT; k += 2) {
            float d0, d1;
            unpack2(fma2(pack2(__uint_as_float(r[k]), __uint_as_float(r[k + 1])), cc, mneg), d0, d1);
            acc[(k / 2) & 3] = add2(acc[(k / 2) & 3], pack2(ex2_approx(d0), ex2_approx(d1)));
        }
        float a0, a1, a2, a3, a4, a5, a6, a7;
        unpack2(acc[0], a0, a1);
        unpack2(acc[1], a2, a3);
        unpack2(acc[2], a4, a5);
        unpack2(acc[3], a6, a7);
        const float s = ((a0 + a1) + (a2 + a3)) + ((a4 + a5) + (a6 + a7));
        if (s <= kLazySum) {
            l += s;
            return;
        }
    }
    float z[CNT];
#pragma unroll
    for (int k = 0; k < CNT; k += 2)
        unpack2(fma2(pack2(__uint_as_float(r[k]), __uint_as_float(r[k + 1])), cc, 0ull), z[k], z[k + 1]);
    rescale_block<CNT>(z, m, l);
}
__device__ __forceinline__ void consume128_folded(const uint32_t (&r)[128], float c, float &m, float &l) {
    consume_folded<128>(r, c, m, l);
}

// The vector pass's fold (scores holding the column bias, as above): beside
// (m, l) it accumulates w = sum_j 2^(z_j - m) v_j, with v_j from shared memory.
// The same lazy max; the rare path moves l and w to the new max together.
template <int CNT>
__device__ __forceinline__ void consume_vec_folded(const uint32_t (&r)[CNT], const float *vec, float c, float &m,
                                                   float &l, float &w) {
    const float4 *vq = reinterpret_cast<const float4 *>(vec);
    const uint64_t cc = pack2(c, c);
    if (m != -INFINITY) {
        const uint64_t mneg = pack2(-m, -m);
        uint64_t al[2] = {0ull, 0ull}, aw[2] = {0ull, 0ull};
#pragma unroll
        for (int k = 0; k < CNT; k += 4) {
            const float4 v = vq[k / 4];
            float d0, d1, d2, d3;
            unpack2(fma2(pack2(__uint_as_float(r[k]), __uint_as_float(r[k + 1])), cc, mneg), d0, d1);
            unpack2(fma2(pack2(__uint_as_float(r[k + 2]), __uint_as_float(r[k + 3])), cc, mneg), d2, d3);
            const uint64_t e01 = pack2(ex2_approx(d0), ex2_approx(d1));
            const uint64_t e23 = pack2(ex2_approx(d2), ex2_approx(d3));
            al[0] = add2(al[0], e01);
            al[1] = add2(al[1], e23);
            aw[0] = fma2(e01, pack2(v.x, v.y), aw[0]);
            aw[1] = fma2(e23, pack2(v.z, v.w), aw[1]);
        }
        float a0, a1, a2, a3;
        unpack2(al[0], a0, a1);
        unpack2(al[1], a2, a3);
        const float s = (a0 + a1) + (a2 + a3);
        if (s <= kLazySum) {
            float w0, w1, w2, w3;
            unpack2(aw[0], w0, w1);
            unpack2(aw[1], w2, w3);
            l += s;
            w += (w0 + w1) + (w2 + w3);
            return;
        }
    }
    float z[CNT];
#pragma unroll
    for (int k = 0; k < CNT; k += 2)
        unpack2(fma2(pack2(__uint_as_float(r[k]), __uint_as_float(r[k + 1])), cc, 0ull), z[k], z[k + 1]);
    float mx[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
    for (int k = 0; k < CNT; k += 4) {
        mx[(k / 4) & 3] = max3(mx[(k / 4) & 3], z[k], z[k + 1]);
        mx[(k / 4) & 3] = max3(mx[(k / 4) & 3], z[k + 2], z[k + 3]);
    }
    const float tmax = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3]));
    if (tmax == -INFINITY) return;  // nothing but padding so far
    const float mnew = fmaxf(m, tmax);
    const float sc = m == -INFINITY ? 0.f : ex2_approx(m - mnew);
    float sl = 0.f, sw = 0.f;
#pragma unroll
    for (int k = 0; k < CNT; ++k) {
        const float e = ex2_approx(z[k] - mnew);
        sl += e;
        sw = fmaf(e, vec[k], sw);
    }
    l = l * sc + sl;
    w = w * sc + sw;
    m = mnew;
}
__device__ __forceinline__ void consume128_vec_folded(const uint32_t (&r)[128], const float *vec, float c, float &m,
                                                      float &l, float &w) {
    consume_vec_folded<128>(r, vec, c, m, l, w);
}

// Measure-mode fold over 64 columns (two 32-column TMEM loads): besides (m, l)
// it accumulates w = sum_j 2^(z_j - m) C_ij with C_ij = |row|^2 + |col|^2 - S_ij
// (S_ij = raw score * sscale), the plan-weighted cost of the row.
__device__ __forceinline__ void consume64_measure(const uint32_t *ra, const uint32_t *rb, const float *bias,
                                                  const float *cnorm, float c, float sscale, float xn, float &m,
                                                  float &l, float &w) {
    const float4 *bq = reinterpret_cast<const float4 *>(bias);
    const float4 *cq = reinterpret_cast<const float4 *>(cnorm);
    float sv[64], z[64];
#pragma unroll
    for (int k = 0; k < 32; ++k) {
        sv[k] = __uint_as_float(ra[k]);
        sv[32 + k] = __uint_as_float(rb[k]);
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
    if (mnew == -INFINITY) return;
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
        w0 = fmaf(e0, fmaf(-sv[k + 0], sscale, xn + cn.x), w0);
        w1 = fmaf(e1, fmaf(-sv[k + 1], sscale, xn + cn.y), w1);
        w0 = fmaf(e2, fmaf(-sv[k + 2], sscale, xn + cn.z), w0);
        w1 = fmaf(e3, fmaf(-sv[k + 3], sscale, xn + cn.w), w1);
    }
    l = l * scale + (a0 + a1);
    w = w * scale + (w0 + w1);
    m = mnew;
}

}  // namespace tc
}  // namespace fs
