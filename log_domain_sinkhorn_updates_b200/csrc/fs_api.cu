// C ABI of the library: handle lifetime, layout planning, pass scheduling.
//
// Everything the functions below compute runs in the kernels of this
// directory; the host code only validates arguments, allocates the handle's
// O(batch (n+m) d) buffers, builds TMA descriptors and enqueues launches on
// the handle's stream.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <algorithm>
#include <atomic>
#include <mutex>
#include <string>
#include <vector>

#include "flashsinkhorn.h"
#include "fs_internal.cuh"
#include "fs_prep.cuh"

using fs::kBlockCols;
using fs::kBlockRows;

struct fs_handle {
    fs_desc desc{};
    int prec = 0;  // resolved fs_precision
    cudaStream_t stream = nullptr;
    int device = 0, sms = 148;
    // packed operand layout
    int d_p = 0, planes = 1, elem = 4, row_bytes = 0, swz = 0, plane_bytes = 0, pack_mode = 0, row_elems = 0;
    // Packed operand rows per problem (a multiple of 256: 128-row blocks, in
    // pairs for the 256-row and CTA-pair passes), and the per-problem stride of
    // the per-point arrays (norms, log-weights, biases): 256 more, so that a
    // column tile starting below the valid count stays inside them.
    int n_pad = 0, m_pad = 0, n_stride = 0, m_stride = 0;
    int qt = 1;  // 128-row blocks per CTA of the single-CTA tensor-core pass
    // device memory (one allocation, carved)
    void *block = nullptr;
    size_t bytes = 0;
    void *packX = nullptr, *packY = nullptr;
    float *xn = nullptr, *yn = nullptr, *la2 = nullptr, *lb2 = nullptr;
    float *bias_row = nullptr, *bias_col = nullptr, *center = nullptr;
    float *rsum = nullptr;  // row sums of a transport application [batch][max(n_pad, m_pad)]
    float4 *part = nullptr;
    unsigned *counters = nullptr;
    double *stats = nullptr, *red = nullptr, *wstat = nullptr;
    int *err = nullptr;
    // The solve's tail: the last alternating fs_solve leaves the column-marginal
    // statistics of its final g-pass in tail_stats and copies of its output
    // potentials in snap_f / snap_g.  fs_marginal_err and fs_ot_cost reuse them
    // (and one f-direction measure pass between them) while f and g still equal
    // the copies bit for bit.
    double *tail_stats = nullptr;
    float *snap_f = nullptr, *snap_g = nullptr;
    int *cmp = nullptr;
    bool tail_ok = false;
    const float *tail_f = nullptr, *tail_g = nullptr;
    bool meas_ok = false;            // meas_cache holds the f-direction measure at the snapshot
    std::vector<double> meas_cache;  // [batch][8] as in h->red
    int last_measure_fused = 0;
    int last_hvp_fused = 0;  // 1: the last fs_hvp_x formed sum_j P_ij (v_i.y_j) y_j in one fused pass
    int last_apply_parts = 1;  // column parts of the split row blocks of the last application (1: none)
    std::vector<double> host_red;  // staging of scalar results (ordinary host memory)
    int host_err[4] = {0, 0, 0, 0};
    CUtensorMap mapX_r{}, mapX_c{}, mapY_r{}, mapY_c{};  // row-side (128-row box) / column-side (256-row box)
    // The biases again as score-product rows (32 bytes a point, store_bias_mm), which the
    // single-CTA update pass adds to S in one more K step, and their maps (256-row boxes).
    void *bmm_row = nullptr, *bmm_col = nullptr;
    CUtensorMap mapBmm_row{}, mapBmm_col{};
    int splits_f = 1, tps_f = 1, splits_g = 1, tps_g = 1;
    int stages = 2, stages_meas = 2;
    bool pair = false;  // run the passes on CTA pairs (one MMA over two SMs); FS_CTA_PAIR=1
    int last_apply = 0;  // kernel of the last transport application: 1 tensor cores, 2 CUDA cores
    // fs_solve's CUDA graph: captured on a private stream for one (f, g, iters,
    // schedule), replayed there between two events on the caller's stream
    cudaStream_t gstream = nullptr;
    cudaEvent_t gev_in = nullptr, gev_out = nullptr;
    cudaGraphExec_t gexec = nullptr;
    const float *gkey_f = nullptr, *gkey_g = nullptr;
    int gkey_iters = 0, gkey_sched = -1, gkernels = 0;
    int last_solve_graph = 0;  // 1: the last fs_solve replayed its graph; 2: it launched directly
    size_t smem = 0, smem_meas = 0;
    unsigned long long timeout_ns = 2000000000ull;
    float sscale = 1.f;             // raw MMA score -> S_ij (3xF16 operand scaling)
    float qscale = 1.f, kscale = 1.f;  // power-of-two operand scales (3xF16)
    std::string last_error;
};

namespace {

thread_local std::string g_last_error;
std::atomic<unsigned long long> g_launches{0};  // kernels this library has launched
// While this thread captures a graph, launches are counted here instead (they
// run when the graph is replayed, and are counted then).
thread_local bool t_capturing = false;
thread_local int t_captured = 0;

fs_status fail(fs_handle *h, fs_status st, const char *fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof(buf), fmt, ap);
    va_end(ap);
    if (h)
        h->last_error = buf;
    else
        g_last_error = buf;
    return st;
}

#define FS_CUDA(h, call)                                                                                    \
    do {                                                                                                    \
        cudaError_t e_ = (call);                                                                            \
        if (e_ != cudaSuccess)                                                                              \
            return fail((h), e_ == cudaErrorMemoryAllocation ? FS_ERR_OOM : FS_ERR_CUDA, "%s: %s (%s:%d)", \
                        #call, cudaGetErrorString(e_), __FILE__, __LINE__);                                 \
    } while (0)

// FS_CUDA for a call that launches one kernel: also counts the launch.
#define FS_LAUNCH(h, call)                                        \
    do {                                                          \
        FS_CUDA(h, call);                                         \
        if (t_capturing)                                          \
            ++t_captured;                                         \
        else                                                      \
            g_launches.fetch_add(1, std::memory_order_relaxed);   \
    } while (0)

size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }
int round_up(int x, int k) { return (x + k - 1) / k * k; }

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

// Library-owned stream-ordered memory pool of a device.  Handles allocate
// and free their buffers on their stream from this pool, so creating and
// destroying handles neither synchronises the device nor returns memory to
// the driver each time; up to 1 GiB of freed memory stays cached.
cudaError_t device_pool(int device, cudaMemPool_t *out) {
    static std::mutex mu;
    static std::vector<cudaMemPool_t> pools;
    std::lock_guard<std::mutex> lock(mu);
    if ((int)pools.size() <= device) pools.resize(device + 1, nullptr);
    if (!pools[device]) {
        cudaMemPoolProps props{};
        props.allocType = cudaMemAllocationTypePinned;
        props.location.type = cudaMemLocationTypeDevice;
        props.location.id = device;
        cudaMemPool_t pool;
        cudaError_t e = cudaMemPoolCreate(&pool, &props);
        if (e != cudaSuccess) return e;
        unsigned long long keep = 1ull << 30;
        e = cudaMemPoolSetAttribute(pool, cudaMemPoolAttrReleaseThreshold, &keep);
        if (e != cudaSuccess) return e;
        pools[device] = pool;
    }
    *out = pools[device];
    return cudaSuccess;
}

// Column split plan for a pass with `row_blocks` CTAs-worth of rows (all
// problems) and `col_tiles` column tiles: pick the split count S that
// minimises (waves) x (tiles per CTA + per-CTA overhead), one CTA per SM.
void plan_splits(int row_blocks, int col_tiles, int sms, int *splits, int *tps) {
    const double overhead = 6.0;  // per-CTA set-up + epilogue, in tile-equivalents
    double best = 1e300;
    *splits = 1;
    *tps = col_tiles;
    for (int s = 1; s <= col_tiles && s <= 64; ++s) {
        const int t = (col_tiles + s - 1) / s;
        const int se = (col_tiles + t - 1) / t;
        const long long ctas = (long long)row_blocks * se;
        const long long waves = (ctas + sms - 1) / sms;
        const double cost = (double)waves * (t + overhead);
        if (cost < best - 1e-9) {
            best = cost;
            *splits = se;
            *tps = t;
        }
    }
}

fs_status encode_map(fs_handle *h, CUtensorMap *map, void *base, int rows_total, int box_rows) {
    auto fn = encode_fn();
    if (!fn) return fail(h, FS_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable from the driver");
    const CUtensorMapDataType dt = h->elem == 4 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32
                                   : (h->prec == FS_PREC_3XF16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16
                                                               : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16);
    cuuint64_t gdim[2] = {(cuuint64_t)(h->row_bytes / h->elem), (cuuint64_t)rows_total};
    cuuint64_t gstride[1] = {(cuuint64_t)h->row_bytes};
    cuuint32_t box[2] = {(cuuint32_t)(h->swz / h->elem), (cuuint32_t)box_rows};
    cuuint32_t estr[2] = {1, 1};
    const CUtensorMapSwizzle sw = h->swz == 128 ? CU_TENSOR_MAP_SWIZZLE_128B
                                  : h->swz == 64 ? CU_TENSOR_MAP_SWIZZLE_64B
                                                 : CU_TENSOR_MAP_SWIZZLE_32B;
    CUresult r = fn(map, dt, 2, base, gdim, gstride, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(h, FS_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
    return FS_OK;
}

// The factor from a base-2 bias to raw score units (1 / scale2), and the
// operand type of the bias rows (tf32 for the tf32 kinds, else bf16).
float mm_inv_c(const fs_handle *h) {
    return (float)(1.0 / (fs::kLog2ed / (double)h->desc.eps * (double)h->sscale));
}
int mm_tf32(const fs_handle *h) { return h->prec == FS_PREC_TF32 || h->prec == FS_PREC_3XTF32 ? 1 : 0; }

// The map of a side's bias rows: rows_total rows of 32 bytes (16 bf16 or 8 fp32),
// boxes of 256 rows, 32-byte swizzle (as the single-CTA pass's bias step reads them).
fs_status encode_bias_map(fs_handle *h, CUtensorMap *map, void *base, int rows_total) {
    auto fn = encode_fn();
    if (!fn) return fail(h, FS_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable from the driver");
    const bool tf32 = mm_tf32(h) != 0;
    cuuint64_t gdim[2] = {(cuuint64_t)(tf32 ? 8 : 16), (cuuint64_t)rows_total};
    cuuint64_t gstride[1] = {32};
    cuuint32_t box[2] = {(cuuint32_t)(tf32 ? 8 : 16), (cuuint32_t)kBlockCols};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(map, tf32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, base, gdim,
                    gstride, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_32B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(h, FS_ERR_CUDA, "cuTensorMapEncodeTiled failed for the bias rows (%d)", (int)r);
    return FS_OK;
}

fs::PassParams make_pass(const fs_handle *h, bool fdir, bool measure) {
    fs::PassParams p{};
    const fs_desc &D = h->desc;
    p.rows = fdir ? D.n : D.m;
    p.rows_pad = fdir ? h->n_pad : h->m_pad;
    p.rows_stride = fdir ? h->n_stride : h->m_stride;
    p.cols = fdir ? D.m : D.n;
    p.cols_rows = fdir ? h->m_pad : h->n_pad;
    p.cols_stride = fdir ? h->m_stride : h->n_stride;
    p.row_bytes = h->row_bytes;
    p.swz = h->swz;
    p.plane_bytes = h->plane_bytes;
    p.d = D.d;
    p.splits = fdir ? h->splits_f : h->splits_g;
    p.tiles_per_split = fdir ? h->tps_f : h->tps_g;
    p.col_tiles = (p.cols + kBlockCols - 1) / kBlockCols;
    p.stages = measure ? h->stages_meas : h->stages;
    // two MMA-issuing threads for one-pass operands and short split jobs (see fs_lse_tc.cu)
    const int npass = (h->prec == FS_PREC_3XTF32 || h->prec == FS_PREC_3XF16) ? 3 : 1;
    p.issuers = (npass == 1 || npass * (h->plane_bytes / 32) <= 4) ? 2 : 1;
    p.eps = (double)D.eps;
    p.scale2 = (float)(fs::kLog2ed / (double)D.eps * (double)h->sscale);
    p.sscale = h->sscale;
    p.mm_inv_c = mm_inv_c(h);
    p.mm_tf32 = mm_tf32(h);
    p.col_bias = fdir ? h->bias_col : h->bias_row;
    p.row_norm = fdir ? h->xn : h->yn;
    p.row_logw2 = fdir ? h->la2 : h->lb2;
    p.col_norm = fdir ? h->yn : h->xn;
    p.part = h->part;
    p.counters = h->counters;
    p.stats = h->stats;
    p.plain_rows = fdir ? h->packX : h->packY;
    p.plain_cols = fdir ? h->packY : h->packX;
    p.timeout_ns = h->timeout_ns;
    p.err = h->err;
    return p;
}

cudaError_t run_pass(fs_handle *h, const fs::PassParams &p, bool fdir, bool measure) {
    if (h->prec == FS_PREC_F32_SIMT) return fs::launch_lse_simt(p, h->desc.batch, measure, h->stream);
    if (h->pair)  // 128-row boxes for both roles: each CTA of a pair loads half of a 256-column tile
        return fs::launch_lse_tc2(p, h->desc.batch, measure, h->prec, fdir ? &h->mapX_r : &h->mapY_r,
                                  fdir ? &h->mapY_r : &h->mapX_r, measure ? h->smem_meas : h->smem, h->stream);
    const CUtensorMap *mr = fdir ? &h->mapX_r : &h->mapY_r;
    const CUtensorMap *mc = fdir ? &h->mapY_c : &h->mapX_c;
    const CUtensorMap *mb = fdir ? &h->mapBmm_col : &h->mapBmm_row;
    return fs::launch_lse_tc(p, h->desc.batch, measure, h->prec, h->qt, mr, mc, mb,
                             measure ? h->smem_meas : h->smem, h->stream);
}

// Bias of the pass that has `cnt`-side columns, from potential pot of that side.
cudaError_t run_bias(fs_handle *h, const float *pot, bool col_is_y) {
    const fs_desc &D = h->desc;
    const double scale2 = fs::kLog2ed / (double)D.eps;
    if (col_is_y)
        return fs::launch_bias(pot, D.batch, D.m, h->m_stride, h->yn, h->lb2, scale2, h->bias_col, h->bmm_col,
                               mm_inv_c(h), mm_tf32(h), h->stream);
    return fs::launch_bias(pot, D.batch, D.n, h->n_stride, h->xn, h->la2, scale2, h->bias_row, h->bmm_row,
                           mm_inv_c(h), mm_tf32(h), h->stream);
}

fs_status update(fs_handle *h, const float *in, float *out, bool fdir, bool write_next_bias) {
    FS_LAUNCH(h, run_bias(h, in, fdir));
    fs::PassParams p = make_pass(h, fdir, false);
    p.pot_out = out;
    p.next_bias = write_next_bias ? (fdir ? h->bias_row : h->bias_col) : nullptr;
    p.next_bias_mm = write_next_bias ? (fdir ? h->bmm_row : h->bmm_col) : nullptr;
    FS_LAUNCH(h, run_pass(h, p, fdir, false));
    return FS_OK;
}

fs_status check_flags(fs_handle *h) {
    FS_CUDA(h, cudaMemcpyAsync(h->host_err, h->err, sizeof(int), cudaMemcpyDeviceToHost, h->stream));
    FS_CUDA(h, cudaMemsetAsync(h->err, 0, sizeof(int), h->stream));
    FS_CUDA(h, cudaStreamSynchronize(h->stream));
    const int e = h->host_err[0];
    if (e & fs::kDevErrTimeout) return fail(h, FS_ERR_TIMEOUT, "a bounded device wait timed out");
    if (e & fs::kDevErrNonfinite) return fail(h, FS_ERR_NONFINITE, "non-finite value in a result or input");
    return FS_OK;
}

// Measure pass in direction fdir at potentials (f, g); results land in
// h->red[slot][batch][8].
fs_status measure(fs_handle *h, const float *f, const float *g, bool fdir, int slot, bool want_col_sum) {
    const fs_desc &D = h->desc;
    FS_LAUNCH(h, run_bias(h, fdir ? g : f, fdir));
    fs::PassParams p = make_pass(h, fdir, true);
    p.pot_in = fdir ? f : g;
    FS_LAUNCH(h, run_pass(h, p, fdir, true));
    const int row_blocks = p.rows_pad / kBlockRows;
    FS_LAUNCH(h, fs::launch_finalize(h->stats, D.batch, row_blocks, want_col_sum ? (fdir ? g : f) : nullptr,
                                   fdir ? h->lb2 : h->la2, p.cols, p.cols_stride, h->red + (size_t)slot * D.batch * 8,
                                   h->stream));
    return FS_OK;
}

}  // namespace

void fs::set_thread_error(const char *msg) { g_last_error = msg; }

namespace {
// Whether (f, g) are still the last alternating solve's output, bit for bit
// (the caller may have written them since): *same receives the answer.
// Synchronises the stream.
fs_status tail_matches(fs_handle *h, const float *f, const float *g, bool *same) {
    *same = false;
    if (!h->tail_ok || f != h->tail_f || g != h->tail_g) return FS_OK;
    const fs_desc &D = h->desc;
    int host = 1;
    FS_CUDA(h, cudaMemsetAsync(h->cmp, 0, sizeof(int), h->stream));
    FS_LAUNCH(h, fs::launch_differs(f, h->snap_f, (size_t)D.batch * D.n, h->cmp, h->stream));
    FS_LAUNCH(h, fs::launch_differs(g, h->snap_g, (size_t)D.batch * D.m, h->cmp, h->stream));
    FS_CUDA(h, cudaMemcpyAsync(&host, h->cmp, sizeof(int), cudaMemcpyDeviceToHost, h->stream));
    FS_CUDA(h, cudaStreamSynchronize(h->stream));
    *same = host == 0;
    return FS_OK;
}
}  // namespace
void fs::count_launches(unsigned count) {
    if (t_capturing)
        t_captured += (int)count;
    else
        g_launches.fetch_add(count, std::memory_order_relaxed);
}

namespace {
// fdir: out_i = sum_j P_ij V_j over the X side's rows (V indexed by Y's points);
// otherwise the transposed application out_j = sum_i P_ij V_i over Y's rows.
fs_status apply(fs_handle *h, const float *f, const float *g, const void *V, bool v_bf16, int dv, float *out,
                float *r, bool divide, bool fdir = true) {
    const fs_desc &D = h->desc;
    FS_CUDA(h, cudaSetDevice(h->device));
    FS_LAUNCH(h, run_bias(h, fdir ? g : f, fdir));  // the column bias of the pass in this direction
    fs::ApplyParams p{};
    p.rows = fdir ? D.n : D.m;
    p.rows_pad = fdir ? h->n_pad : h->m_pad;
    p.rows_stride = fdir ? h->n_stride : h->m_stride;
    p.cols = fdir ? D.m : D.n;
    p.cols_rows = fdir ? h->m_pad : h->n_pad;
    p.cols_stride = fdir ? h->m_stride : h->n_stride;
    p.d = D.d;
    p.d_p = h->d_p;
    p.row_elems = h->row_elems;
    p.pack_mode = h->pack_mode;
    p.dv = dv;
    // packed X holds qscale (x - t), packed Y kscale * 2 (y - t) (or the
    // normalised rows): unscaled, their dot product is S_ij either way round
    p.q_unscale = 1.f / (fdir ? h->qscale : h->kscale);
    p.k_unscale = 1.f / (fdir ? h->kscale : h->qscale);
    p.scale = fs::kLog2ed / (double)D.eps;
    p.packQ = fdir ? h->packX : h->packY;
    p.packK = fdir ? h->packY : h->packX;
    p.row_norm = fdir ? h->xn : h->yn;
    p.row_logw2 = fdir ? h->la2 : h->lb2;
    p.pot_row = fdir ? f : g;
    p.col_bias = fdir ? h->bias_col : h->bias_row;
    p.V = V;
    p.v_bf16 = v_bf16 ? 1 : 0;
    p.out = out;
    p.rsum = r;
    p.divide = divide ? 1 : 0;
    // Tensor cores for dv <= 256: on CTA pairs for the 512-byte operand rows
    // (and at every width with FS_APPLY_PAIR=1), on one CTA for rows of up to
    // 256 bytes where its plan fits -- two 128-row blocks per CTA sharing every
    // streamed tile where dv <= 128 and the grid still covers the SMs.  The
    // CUDA-core kernel otherwise, for the fp32 SIMT precision, or with
    // FS_APPLY_SIMT=1.
    const int vpl = v_bf16 ? 1 : 2;
    const char *force_simt = getenv("FS_APPLY_SIMT");
    const bool tc_ok = h->prec != FS_PREC_F32_SIMT && dv <= 256 && !(force_simt && atoi(force_simt) != 0);
    bool use_pair = h->pair;
    if (const char *env = getenv("FS_APPLY_PAIR")) use_pair = atoi(env) != 0;
    int dv_pad = use_pair ? (dv + 31) / 32 * 32 : (dv + 15) / 16 * 16;
    int kslots = 0, stages = 0;
    size_t smem = 0;
    bool use_q2 = false;
    int qb = 2;
    if (tc_ok && use_pair)
        smem = fs::apply_tc2_plan(h->row_bytes, dv_pad, vpl, &kslots, &stages);
    if (tc_ok && smem == 0 && !h->pair && h->row_bytes <= 256) {
        use_pair = false;
        dv_pad = (dv + 15) / 16 * 16;
        // Two 128-row blocks per CTA for narrow V where that still gives every SM
        // a CTA; else one block shared by both groups, which take alternate tiles
        // (twice the CTAs).  Measured at dv = 128 (n = m = 65536): 3.33 ms shared,
        // 3.41 two blocks; middim (dv = 64, 64 two-block CTAs): 0.299 shared, 0.352
        // the one-block kernel; dv = 3 and dv = 32: two blocks 1-3 % faster.
        // FS_ROW_BLOCKS=1 forces the one-block kernel of fs_apply_tc.cu, =2 two
        // blocks, =3 one shared block, wherever they fit.
        const char *env_rb = getenv("FS_ROW_BLOCKS");
        const int rbk = env_rb ? atoi(env_rb) : 0;
        const long long q2_ctas = (long long)D.batch * ((p.rows_pad + 255) / 256);
        if (rbk != 1) {
            qb = rbk == 2 ? 2 : (rbk == 3 ? 1 : (q2_ctas >= h->sms && dv < 64 ? 2 : 1));
            smem = fs::apply_q2_plan(h->row_bytes, dv_pad, vpl, qb, &kslots, &stages);
            use_q2 = smem != 0;
        }
        if (smem == 0) smem = fs::apply_tc_plan(h->row_bytes, dv_pad, vpl, &kslots, &stages);
    }
    if (smem == 0) {
        h->last_apply = 2;
        h->last_apply_parts = 1;
        FS_LAUNCH(h, fs::launch_apply_simt(p, D.batch, h->stream));
        return FS_OK;
    }
    h->last_apply = use_pair ? 3 : (use_q2 ? (qb == 2 ? 4 : 6) : 1);
    h->last_apply_parts = 1;
    p.row_bytes = h->row_bytes;
    p.swz = h->swz;
    p.plane_bytes = h->plane_bytes;
    p.dv_pad = dv_pad;
    p.kslots = kslots;
    p.stages = stages;
    p.sscale = h->sscale;
    p.timeout_ns = h->timeout_ns;
    p.err = h->err;
    // One row block per CTA (one CTA per SM): the row blocks past the last full
    // wave, where they fill at most half the SMs, are split over their column
    // tiles into k parts of at least two tiles (one per softmax group), so the
    // last wave takes 1/k of a CTA's time.  A second launch runs the parts, and
    // a merge kernel adds them.  Highdim (512 row blocks, 148 SMs): the last 68
    // in two parts each.  FS_APPLY_TAIL=0 keeps every row block whole.
    p.main_blocks = p.rows_pad / fs::kBlockRows;
    p.tail_k = 1;
    size_t tail_rows = 0;
    if (use_q2 && qb == 1 && D.batch == 1) {
        const char *env_tail = getenv("FS_APPLY_TAIL");
        const int blocks = p.rows_pad / fs::kBlockRows, rem = blocks % h->sms;
        const int ntiles = (p.cols + 127) / 128;
        int k = rem > 0 ? std::min(8, h->sms / rem) : 1;
        k = std::min(k, ntiles / 2);
        if (env_tail && atoi(env_tail) == 0) k = 1;
        if (k > 1) {
            p.tail_k = h->last_apply_parts = k;
            p.main_blocks = blocks - rem;
            tail_rows = (size_t)rem * fs::kBlockRows;
        }
    }
    // V~: V transposed, bf16 planes [batch][vpl][dv_pad][m_pad], from the pool for
    // this call, followed by the split row blocks' partial sums
    const size_t vt_bytes = ((size_t)D.batch * vpl * dv_pad * p.cols_rows * 2 + 255) / 256 * 256;
    const size_t tail_bytes = (size_t)p.tail_k * tail_rows * (dv + 1) * 4;
    cudaMemPool_t pool;
    void *vt = nullptr;
    FS_CUDA(h, device_pool(h->device, &pool));
    FS_CUDA(h, cudaMallocFromPoolAsync(&vt, vt_bytes + tail_bytes, pool, h->stream));
    if (p.tail_k > 1) {
        p.tail_o = reinterpret_cast<float *>(static_cast<char *>(vt) + vt_bytes);
        p.tail_rs = p.tail_o + (size_t)p.tail_k * tail_rows * dv;
    }
    cudaError_t e = fs::launch_vt_pack(V, v_bf16, D.batch, p.cols, dv, p.cols_rows, dv_pad, vpl, vt, h->stream);
    g_launches.fetch_add(1, std::memory_order_relaxed);
    CUtensorMap map_v{};
    fs_status st = FS_OK;
    if (e == cudaSuccess) {
        auto fn = encode_fn();
        cuuint64_t gdim[2] = {(cuuint64_t)p.cols_rows, (cuuint64_t)D.batch * vpl * dv_pad};
        cuuint64_t gstride[1] = {(cuuint64_t)p.cols_rows * 2};
        cuuint32_t box[2] = {64, (cuuint32_t)dv_pad};
        cuuint32_t estr[2] = {1, 1};
        if (use_pair) box[1] = (cuuint32_t)(dv_pad / 2);  // each CTA of a pair loads half the columns of V
        CUresult r2 = fn ? fn(&map_v, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, vt, gdim, gstride, box, estr,
                              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE)
                         : CUDA_ERROR_NOT_SUPPORTED;
        if (r2 != CUDA_SUCCESS) st = fail(h, FS_ERR_CUDA, "cuTensorMapEncodeTiled failed for V (%d)", (int)r2);
    }
    if (e == cudaSuccess && st == FS_OK) {
        if (use_pair) {
            // each CTA of a pair loads a 64-point half of every 128-column tile of K
            CUtensorMap map_k2{};
            st = encode_map(h, &map_k2, fdir ? h->packY : h->packX, D.batch * p.cols_rows, 64);
            if (st == FS_OK) {
                e = fs::launch_apply_tc2(p, D.batch, h->prec, vpl, fdir ? &h->mapX_r : &h->mapY_r, &map_k2, &map_v,
                                         smem, h->stream);
                g_launches.fetch_add(1, std::memory_order_relaxed);
            }
        } else if (use_q2) {
            e = fs::launch_apply_q2(p, D.batch, h->prec, vpl, qb, fdir ? &h->mapX_r : &h->mapY_r,
                                    fdir ? &h->mapY_r : &h->mapX_r, &map_v, smem, h->stream);
            g_launches.fetch_add(qb == 1 && p.tail_k > 1 ? (p.main_blocks > 0) + 2 : 1, std::memory_order_relaxed);
        } else {
            e = fs::launch_apply_tc(p, D.batch, h->prec, vpl, fdir ? &h->mapX_r : &h->mapY_r,
                                    fdir ? &h->mapY_r : &h->mapX_r, &map_v, smem, h->stream);
            g_launches.fetch_add(1, std::memory_order_relaxed);
        }
    }
    cudaFreeAsync(vt, h->stream);
    if (st != FS_OK) return st;
    FS_CUDA(h, e);
    return FS_OK;
}
// One-column transport application out = P v (fdir) or P^T v through the streamed
// LSE pass's vector mode: the softmax warps accumulate sum_j 2^(z_j - m) v_j next to
// the row's LSE state, so the column costs no P~ and no P V product, and the
// pass runs at the LSE pass's rate (a tensor-core application of one column costs
// as much as one of 128).  vpad: scratch of batch x (the column side's stride)
// floats.  r (may be null) receives the row sums.  Tensor-core handles only.
fs_status apply_vec(fs_handle *h, const float *f, const float *g, const float *v, bool fdir, float *out, float *r,
                    float *vpad, bool bias_ready = false) {
    const fs_desc &D = h->desc;
    fs::PassParams p = make_pass(h, fdir, true);
    FS_LAUNCH(h, fs::launch_pad_vec(v, D.batch, p.cols, p.cols_stride, vpad, h->stream));
    if (!bias_ready) FS_LAUNCH(h, run_bias(h, fdir ? g : f, fdir));
    p.pot_in = fdir ? f : g;
    p.col_vec = vpad;
    p.vec_out = out;
    p.vec_rsum = r;
    FS_LAUNCH(h, run_pass(h, p, fdir, true));
    return FS_OK;
}

// The launches of fs_solve, in order, on h->stream.
fs_status enqueue_solve(fs_handle *h, float *f, float *g, int iters, fs_schedule schedule) {
    if (schedule == FS_SCHED_ALTERNATING) {
        // One bias launch from the initial g; afterwards every pass's fused
        // epilogue writes the bias the next pass reads.
        FS_LAUNCH(h, run_bias(h, g, true));
        for (int it = 0; it < iters; ++it) {
            fs::PassParams pf = make_pass(h, true, false);
            pf.pot_out = f;
            pf.next_bias = h->bias_row;
            pf.next_bias_mm = h->bmm_row;
            FS_LAUNCH(h, run_pass(h, pf, true, false));
            fs::PassParams pg = make_pass(h, false, false);
            pg.pot_out = g;
            pg.next_bias = h->bias_col;
            pg.next_bias_mm = h->bmm_col;
            // the final g-pass also reduces the column marginal of the pair it leaves
            if (it == iters - 1) pg.tail_stats = h->tail_stats;
            FS_LAUNCH(h, run_pass(h, pg, false, false));
        }
        if (iters > 0) {
            const fs_desc &D = h->desc;
            FS_CUDA(h, cudaMemcpyAsync(h->snap_f, f, (size_t)D.batch * D.n * 4, cudaMemcpyDeviceToDevice, h->stream));
            FS_CUDA(h, cudaMemcpyAsync(h->snap_g, g, (size_t)D.batch * D.m * 4, cudaMemcpyDeviceToDevice, h->stream));
        }
    } else {
        for (int it = 0; it < iters; ++it) {
            FS_LAUNCH(h, run_bias(h, g, true));
            FS_LAUNCH(h, run_bias(h, f, false));
            fs::PassParams pf = make_pass(h, true, false);
            pf.pot_out = f;
            FS_LAUNCH(h, run_pass(h, pf, true, false));
            fs::PassParams pg = make_pass(h, false, false);
            pg.pot_out = g;
            FS_LAUNCH(h, run_pass(h, pg, false, false));
        }
    }
    return FS_OK;
}

// Capture enqueue_solve into h->gexec on the handle's private stream.  Returns
// false (with no error left pending and the stream usable) if the capture or
// the instantiation fails; the caller then launches directly.
// The handle's stream for graph captures (and its two events), created once.
bool ensure_graph_stream(fs_handle *h) {
    if (h->gstream) return true;
    if (cudaStreamCreateWithFlags(&h->gstream, cudaStreamNonBlocking) != cudaSuccess ||
        cudaEventCreateWithFlags(&h->gev_in, cudaEventDisableTiming) != cudaSuccess ||
        cudaEventCreateWithFlags(&h->gev_out, cudaEventDisableTiming) != cudaSuccess) {
        cudaGetLastError();
        return false;
    }
    return true;
}

bool capture_solve(fs_handle *h, float *f, float *g, int iters, fs_schedule schedule) {
    if (h->gexec) {
        cudaGraphExecDestroy(h->gexec);
        h->gexec = nullptr;
    }
    if (!ensure_graph_stream(h)) return false;
    if (cudaStreamBeginCapture(h->gstream, cudaStreamCaptureModeThreadLocal) != cudaSuccess) {
        cudaGetLastError();
        return false;
    }
    cudaStream_t user = h->stream;
    const std::string saved_error = h->last_error;  // a failed capture is not the caller's error
    h->stream = h->gstream;
    t_capturing = true;
    t_captured = 0;
    const fs_status st = enqueue_solve(h, f, g, iters, schedule);
    t_capturing = false;
    h->stream = user;
    h->last_error = saved_error;
    cudaGraph_t graph = nullptr;
    const cudaError_t ec = cudaStreamEndCapture(h->gstream, &graph);  // always ends the capture
    bool ok = st == FS_OK && ec == cudaSuccess && graph != nullptr &&
              cudaGraphInstantiate(&h->gexec, graph, 0) == cudaSuccess;
    if (graph) cudaGraphDestroy(graph);
    if (!ok) {
        cudaGetLastError();
        h->gexec = nullptr;
        return false;
    }
    h->gkey_f = f;
    h->gkey_g = g;
    h->gkey_iters = iters;
    h->gkey_sched = (int)schedule;
    h->gkernels = t_captured;
    return true;
}
// MV_i = sum_j P_ij (v_i . y_j) y_j in one pass over the plan (fs_hvp_tc.cu), batch 1,
// squared Euclidean cost; *done = false (and nothing enqueued) where the handle's
// operands have no fused form or its plan does not fit.
fs_status hvp_fused_term(fs_handle *h, const float *f, const float *g, const void *Y, const float *V, float *MV,
                         bool *done) {
    *done = false;
    const fs_desc &D = h->desc;
    if (h->prec == FS_PREC_F32_SIMT || h->pair || D.cost != FS_COST_SQEUCLIDEAN) return FS_OK;
    const int umode = fs::hvp_w_mode(h->prec, h->plane_bytes, h->row_bytes);
    if (umode == 0) return FS_OK;
    const bool bf16 = D.dtype == FS_BF16;
    const int vpl = bf16 ? 1 : 2;
    const int dv_pad = (D.d + 15) / 16 * 16;
    int kslots = 0, stages = 0;
    const size_t smem = fs::hvp_w_plan(h->row_bytes, umode, dv_pad, vpl, &kslots, &stages);
    if (smem == 0 || dv_pad > 256) return FS_OK;
    const int B = D.batch;
    size_t off = 0;
    auto carve = [&](size_t bytes) {
        const size_t o = off;
        off += align256(bytes);
        return o;
    };
    const size_t o_u = carve((umode == 2 ? 2 : 1) * (size_t)B * h->n_pad * h->row_bytes);
    const size_t o_norm = carve((size_t)B * h->n_stride * 4);
    const size_t o_vt = carve((size_t)B * vpl * dv_pad * h->m_pad * 2);
    const size_t o_mx = carve(16);
    cudaMemPool_t pool;
    uint8_t *blk = nullptr;
    FS_CUDA(h, device_pool(h->device, &pool));
    FS_CUDA(h, cudaMallocFromPoolAsync((void **)&blk, off, pool, h->stream));
    auto run = [&]() -> fs_status {
        cudaStream_t s = h->stream;
        FS_LAUNCH(h, run_bias(h, g, true));  // the f-direction column bias from g
        float uscale = 1.f;
        if (umode == 1) {
            if (h->pack_mode == fs::kPack3xF16) {  // U's own power-of-two scale, as for X and Y
                float *mx = reinterpret_cast<float *>(blk + o_mx);
                float host = 0.f;
                FS_LAUNCH(h, fs::launch_maxabs(V, false, D.n, D.d, B, nullptr, mx, s));
                FS_CUDA(h, cudaMemcpyAsync(&host, mx, sizeof(float), cudaMemcpyDeviceToHost, s));
                FS_CUDA(h, cudaStreamSynchronize(s));
                if (host > 0.f && std::isfinite(host))
                    uscale = std::ldexp(1.f, 14 - (int)std::ceil(std::log2((double)host)));
            }
            FS_LAUNCH(h, fs::launch_pack(V, false, D.n, h->n_pad, D.d, B, nullptr, uscale, h->pack_mode, h->d_p,
                                         h->row_elems, blk + o_u, reinterpret_cast<float *>(blk + o_norm), h->n_stride,
                                         h->err, s, false));
        } else {
            FS_LAUNCH(h, fs::launch_u_split(V, B, D.n, h->n_pad, D.d, h->row_elems, blk + o_u, s));
        }
        FS_LAUNCH(h, fs::launch_vt_pack(Y, bf16, B, D.m, D.d, h->m_pad, dv_pad, vpl, blk + o_vt, s));
        CUtensorMap map_u{}, map_v{};
        fs_status st = encode_map(h, &map_u, blk + o_u, (umode == 2 ? 2 : 1) * B * h->n_pad, kBlockRows);
        if (st != FS_OK) return st;
        auto fn = encode_fn();
        cuuint64_t gdim[2] = {(cuuint64_t)h->m_pad, (cuuint64_t)B * vpl * dv_pad};
        cuuint64_t gstride[1] = {(cuuint64_t)h->m_pad * 2};
        cuuint32_t box[2] = {64, (cuuint32_t)dv_pad};
        cuuint32_t estr[2] = {1, 1};
        const CUresult r2 = fn ? fn(&map_v, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, blk + o_vt, gdim, gstride, box, estr,
                                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE)
                               : CUDA_ERROR_NOT_SUPPORTED;
        if (r2 != CUDA_SUCCESS) return fail(h, FS_ERR_CUDA, "cuTensorMapEncodeTiled failed for Y~ (%d)", (int)r2);
        fs::ApplyParams p{};
        p.rows = D.n;
        p.rows_pad = h->n_pad;
        p.rows_stride = h->n_stride;
        p.cols = D.m;
        p.cols_rows = h->m_pad;
        p.cols_stride = h->m_stride;
        p.d = D.d;
        p.d_p = h->d_p;
        p.row_elems = h->row_elems;
        p.pack_mode = h->pack_mode;
        p.dv = D.d;
        p.scale = fs::kLog2ed / (double)D.eps;
        p.pot_row = f;
        p.row_norm = h->xn;
        p.row_logw2 = h->la2;
        p.col_bias = h->bias_col;
        p.out = MV;
        p.row_bytes = h->row_bytes;
        p.swz = h->swz;
        p.plane_bytes = h->plane_bytes;
        p.dv_pad = dv_pad;
        p.kslots = kslots;
        p.stages = stages;
        p.sscale = h->sscale;
        p.timeout_ns = h->timeout_ns;
        p.err = h->err;
        // K holds 2 kscale (y - t) and U holds uscale v: v . (y - t) = S' / (2 kscale uscale)
        const float cw = (float)(1.0 / (2.0 * (double)h->kscale * (double)uscale));
        FS_LAUNCH(h, fs::launch_hvp_w(p, B, h->prec, umode, vpl, cw, V, bf16 ? nullptr : h->center, &h->mapX_r, &map_u,
                                      &h->mapY_r, &map_v, smem, s));
        return FS_OK;
    };
    const fs_status st = run();
    cudaFreeAsync(blk, h->stream);
    if (st == FS_OK) *done = true;
    return st;
}

}  // namespace

// A single column on a tensor-core handle goes through the LSE pass's vector mode
// (apply_vec), unless FS_APPLY_VEC=0 or the CUDA-core path is asked for.
static bool vec_path(const fs_handle *h, int dv) {
    if (dv != 1 || h->prec == FS_PREC_F32_SIMT) return false;
    const char *e = getenv("FS_APPLY_VEC");
    if (e && atoi(e) == 0) return false;
    const char *s = getenv("FS_APPLY_SIMT");
    return !(s && atoi(s) != 0);
}
static fs_status apply_vec_alloc(fs_handle *h, const float *f, const float *g, const float *v, bool fdir,
                                 float *out, float *r) {
    const fs_desc &D = h->desc;
    FS_CUDA(h, cudaSetDevice(h->device));
    cudaMemPool_t pool;
    float *vpad = nullptr;
    FS_CUDA(h, device_pool(h->device, &pool));
    FS_CUDA(h, cudaMallocFromPoolAsync((void **)&vpad, (size_t)D.batch * (fdir ? h->m_stride : h->n_stride) * 4,
                                       pool, h->stream));
    const fs_status st = apply_vec(h, f, g, v, fdir, out, r, vpad);
    cudaFreeAsync(vpad, h->stream);
    if (st == FS_OK) {
        h->last_apply = 5;
        h->last_apply_parts = 1;
    }
    return st;
}

extern "C" {

// ---- transport application ("FlashSinkhorn: IO-aware EOT on GPU", Metodologia
// section 3: barycentric projection and gradient as plan-weighted averages) ----
fs_status fs_transport_apply(fs_handle *h, const float *f, const float *g, const float *V, int dv, float *out,
                             float *r) {
    if (!h || !f || !g || !V || !out || dv < 1) return fail(h, FS_ERR_INVALID_ARG, "bad argument");
    if (vec_path(h, dv)) return apply_vec_alloc(h, f, g, V, true, out, r);
    return apply(h, f, g, V, false, dv, out, r, false);
}

fs_status fs_barycentric_map(fs_handle *h, const float *f, const float *g, const void *Y, float *out) {
    if (!h || !f || !g || !Y || !out) return fail(h, FS_ERR_INVALID_ARG, "null argument");
    return apply(h, f, g, Y, h->desc.dtype == FS_BF16, h->desc.d, out, nullptr, true);
}

// Cosine-cost gradient with respect to the `own` cloud (X for the f direction):
// b = P (other)^ (the transport application of the other cloud's unit rows, from
// a pool scratch), then grad = -(b - (own^.b) own^) / |own|, row by row.
static fs_status cosine_grad(fs_handle *h, const float *f, const float *g, const void *own, const void *other, bool fdir,
                      float *grad) {
    const fs_desc &D = h->desc;
    const bool bf16 = D.dtype == FS_BF16;
    const size_t own_rows = (size_t)D.batch * (fdir ? D.n : D.m), other_rows = (size_t)D.batch * (fdir ? D.m : D.n);
    FS_CUDA(h, cudaSetDevice(h->device));
    cudaMemPool_t pool;
    float *unit = nullptr;
    FS_CUDA(h, device_pool(h->device, &pool));
    FS_CUDA(h, cudaMallocFromPoolAsync((void **)&unit, other_rows * D.d * 4, pool, h->stream));
    auto run = [&]() -> fs_status {
        FS_LAUNCH(h, fs::cos_unit_rows(other, bf16, other_rows, D.d, unit, h->stream));
        fs_status st = apply(h, f, g, unit, false, D.d, grad, nullptr, false, fdir);
        if (st != FS_OK) return st;
        FS_LAUNCH(h, fs::cos_grad(own, bf16, grad, own_rows, D.d, grad, h->stream));
        return FS_OK;
    };
    const fs_status st = run();
    cudaFreeAsync(unit, h->stream);
    return st;
}

fs_status fs_grad_x(fs_handle *h, const float *f, const float *g, const void *X, const void *Y, float *grad) {
    if (!h || !f || !g || !X || !Y || !grad) return fail(h, FS_ERR_INVALID_ARG, "null argument");
    if (h->desc.cost == FS_COST_COSINE) return cosine_grad(h, f, g, X, Y, true, grad);
    const fs_desc &D = h->desc;
    const bool bf16 = D.dtype == FS_BF16;
    fs_status st = apply(h, f, g, Y, bf16, D.d, grad, h->rsum, false);  // grad <- P Y, rsum <- P 1
    if (st != FS_OK) return st;
    FS_LAUNCH(h, fs::launch_grad_combine(X, bf16, h->rsum, grad, D.batch, D.n, D.d, grad, h->stream));
    return FS_OK;
}

fs_status fs_transport_apply_t(fs_handle *h, const float *f, const float *g, const float *U, int du, float *out,
                               float *c) {
    if (!h || !f || !g || !U || !out || du < 1) return fail(h, FS_ERR_INVALID_ARG, "bad argument");
    if (vec_path(h, du)) return apply_vec_alloc(h, f, g, U, false, out, c);
    return apply(h, f, g, U, false, du, out, c, false, false);
}

fs_status fs_grad_y(fs_handle *h, const float *f, const float *g, const void *X, const void *Y, float *grad) {
    if (!h || !f || !g || !X || !Y || !grad) return fail(h, FS_ERR_INVALID_ARG, "null argument");
    if (h->desc.cost == FS_COST_COSINE) return cosine_grad(h, f, g, Y, X, false, grad);
    const fs_desc &D = h->desc;
    const bool bf16 = D.dtype == FS_BF16;
    fs_status st = apply(h, f, g, X, bf16, D.d, grad, h->rsum, false, false);  // grad <- P^T X, rsum <- P^T 1
    if (st != FS_OK) return st;
    FS_LAUNCH(h, fs::launch_grad_combine(Y, bf16, h->rsum, grad, D.batch, D.m, D.d, grad, h->stream));
    return FS_OK;
}

fs_status fs_hvp_x(fs_handle *h, const float *f, const float *g, const void *X, const void *Y, const float *V,
                   float *out, int max_cg_iters, double cg_rtol, int *cg_iters_done) {
    if (!h || !f || !g || !X || !Y || !V || !out || max_cg_iters < 1 || !(cg_rtol > 0.0))
        return fail(h, FS_ERR_INVALID_ARG, "bad argument");
    const fs_desc &D = h->desc;
    if (D.batch > 65535) return fail(h, FS_ERR_UNSUPPORTED, "fs_hvp_x takes at most 65535 problems");
    FS_CUDA(h, cudaSetDevice(h->device));
    // Each problem of the batch is its own solve, laid out problem after problem:
    // the row-wise steps run over B n rows (B m columns) at once, the reductions
    // and the CG scalars are per problem.
    const int B = D.batch;
    const size_t n1 = (size_t)D.n, m1 = (size_t)D.m, d = (size_t)D.d;
    const size_t n = (size_t)B * n1, m = (size_t)B * m1;
    // The cosine cost runs the same sequence on the unit rows Y^ (fp32) and the
    // projected direction v~ (fs_cosine.cu), with its own first and last steps.
    const bool cosine = D.cost == FS_COST_COSINE;
    const bool bf16 = D.dtype == FS_BF16;
    // Columns of y folded into one transport-matrix product (width nq d, fp32):
    // as many as keep the width within 256 and, where the handle's operands
    // suit the tensor-core application, within its shared-memory plan.
    int nq = d >= 256 ? 1 : (int)(256 / d);
    if (h->prec != FS_PREC_F32_SIMT) {
        int ks = 0, stg = 0;
        if (h->pair)  // the CTA-pair application, fp32 columns in two bf16 planes
            while (nq > 1 && fs::apply_tc2_plan(h->row_bytes, (nq * (int)d + 31) / 32 * 32, 2, &ks, &stg) == 0) --nq;
        else if (h->row_bytes <= 256)
            while (nq > 1 && fs::apply_tc_plan(h->row_bytes, (nq * (int)d + 15) / 16 * 16, 2, &ks, &stg) == 0) --nq;
    }
    // scratch, O((n + m) d), from the pool for this call
    size_t off = 0;
    auto carve = [&](size_t count) {
        size_t o = off;
        off += (count * 4 + 255) / 256 * 256;
        return o;
    };
    const size_t oPY = carve(n * d), o_r = carve(n), o_c = carve(m), oW1 = carve(n * (d + 2)), oT = carve(m * (d + 2));
    const size_t o_u = carve(n), o_tn = carve(n), o_tm = carve(m), o_z = carve(m), o_x = carve(m);
    const size_t o_res = carve(m), o_p = carve(m), o_Ap = carve(m), o_df = carve(n);
    const size_t o_dgY = carve(m * (d + 1)), oQ1 = carve(n * (d + 1)), oMV = carve(n * d);
    const size_t oVc = carve(m * nq * d), oOc = carve(n * nq * d);
    const size_t o_part = carve((size_t)B * 2 * 4096), o_sc = carve((size_t)B * 2 * 5);
    const size_t o_Yh = carve(cosine ? m * d : 1), o_Vt = carve(cosine ? n * d : 1);
    const size_t o_vpad = carve((size_t)B * (h->n_stride > h->m_stride ? h->n_stride : h->m_stride));
    const size_t o_steps = carve((size_t)B);
    cudaMemPool_t pool;
    uint8_t *blk = nullptr;
    FS_CUDA(h, device_pool(h->device, &pool));
    FS_CUDA(h, cudaMallocFromPoolAsync((void **)&blk, off, pool, h->stream));
    auto F = [&](size_t o) { return reinterpret_cast<float *>(blk + o); };
    double *part = reinterpret_cast<double *>(blk + o_part);
    double *sc = reinterpret_cast<double *>(blk + o_sc);  // [k][B]: k = 0 rr, 1 p.Ap, 2 rr_new, 3 sum, 4 z.z
    double *rr_d = sc, *pap_d = sc + B, *rrn_d = sc + 2 * B, *sum_d = sc + 3 * B, *zz_d = sc + 4 * B;
    int *steps_d = reinterpret_cast<int *>(blk + o_steps);  // [B] CG steps each problem took
    const double tol2 = cg_rtol * cg_rtol;
    float *PY = F(oPY), *r = F(o_r), *c = F(o_c), *W1 = F(oW1), *Tm = F(oT), *u = F(o_u);
    float *tn = F(o_tn), *tm = F(o_tm), *z = F(o_z), *x = F(o_x), *res = F(o_res), *p = F(o_p), *Ap = F(o_Ap);
    float *df = F(o_df), *dgY = F(o_dgY), *Q1 = F(oQ1), *MV = F(oMV);
    float *Vc = F(oVc), *Oc = F(oOc), *Yh = F(o_Yh), *Vt = F(o_Vt), *vpad = F(o_vpad);
    // the CG's one-column products through the LSE pass's vector mode on tensor-core
    // handles; the CUDA-core validation path keeps the transport kernels
    const char *env_simt0 = getenv("FS_APPLY_SIMT");
    const bool use_vec = h->prec != FS_PREC_F32_SIMT && !(env_simt0 && atoi(env_simt0) != 0);
    // (inside the CG both directions' biases are already in place: f and g do not change)
    auto apply1 = [&](const float *vin, bool fdir, float *vout) -> fs_status {
        if (use_vec) return apply_vec(h, f, g, vin, fdir, vout, nullptr, vpad, true);
        return apply(h, f, g, vin, false, 1, vout, nullptr, false, fdir);
    };
    // the column cloud the transport products see (Y, or its unit rows), and the
    // direction the transport-matrix term contracts with (v, or v~)
    const void *Yop = cosine ? (const void *)Yh : Y;
    const bool ybf = cosine ? false : bf16;
    const float *Vop = cosine ? Vt : V;
    cudaStream_t s = h->stream;
    fs_status st = FS_OK;
    int it = 0;
    auto run = [&]() -> fs_status {
        // transport products that do not depend on the CG solution
        if (cosine) FS_LAUNCH(h, fs::cos_unit_rows(Y, bf16, m, (int)d, Yh, s));
        // (every application costs a full pass over the plan whatever its width, so
        // the vectors that share a direction go through one application together)
        fs_status s2 = apply(h, f, g, Yop, ybf, (int)d, PY, r, false, true);  // P Y (P Y^), r = P 1
        if (s2 != FS_OK) return s2;
        if (cosine)
            FS_LAUNCH(h, fs::cos_hvp_prep(X, bf16, V, PY, r, n, (int)d, u, W1, Vt, s));
        else
            FS_LAUNCH(h, fs::hvp_prep(X, bf16, V, PY, r, (int)n, (int)d, u, W1, s));
        // P^T [v | x.v | u/r] (P^T [v~ | 0 | u/r]) and its row sums c = P^T 1
        s2 = apply(h, f, g, W1, false, (int)d + 2, Tm, c, false, false);
        if (s2 != FS_OK) return s2;
        FS_LAUNCH(h, fs::hvp_w(Yop, ybf, Tm, (int)m, (int)d, cosine ? 1.f : 2.f, z, s));  // z = w - P^T (u / r)
        FS_LAUNCH(h, fs::hvp_dot(B, m1, z, nullptr, part, sum_d, s));
        FS_LAUNCH(h, fs::hvp_center(B, m1, sum_d, z, s));
        // CG on [diag(c) - P^T diag(1/r) P] dg = z, iterates kept orthogonal to 1;
        // a problem stops once rr <= tol2 z.z, the others run on
        FS_CUDA(h, cudaMemsetAsync(x, 0, m * 4, s));
        FS_CUDA(h, cudaMemsetAsync(steps_d, 0, (size_t)B * 4, s));
        FS_CUDA(h, cudaMemcpyAsync(res, z, m * 4, cudaMemcpyDeviceToDevice, s));
        FS_CUDA(h, cudaMemcpyAsync(p, z, m * 4, cudaMemcpyDeviceToDevice, s));
        FS_LAUNCH(h, fs::hvp_dot(B, m1, z, z, part, rr_d, s));
        FS_LAUNCH(h, fs::hvp_dot(B, m1, z, z, part, zz_d, s));
        std::vector<double> rr((size_t)B), zz((size_t)B);
        FS_CUDA(h, cudaMemcpyAsync(rr.data(), rr_d, (size_t)B * 8, cudaMemcpyDeviceToHost, s));
        FS_CUDA(h, cudaMemcpyAsync(zz.data(), zz_d, (size_t)B * 8, cudaMemcpyDeviceToHost, s));
        FS_CUDA(h, cudaStreamSynchronize(s));
        auto any_running = [&]() {
            for (int b = 0; b < B; ++b)
                if (rr[b] > tol2 * zz[b] && zz[b] > 0.0) return true;
            return false;
        };
        if (use_vec) {  // the biases of both directions, once for the whole CG
            FS_LAUNCH(h, run_bias(h, g, true));
            FS_LAUNCH(h, run_bias(h, f, false));
        }
        // k CG steps on h->stream (the stream the lambdas see)
        auto enqueue_steps = [&](int k) -> fs_status {
            const cudaStream_t st = h->stream;
            for (int q = 0; q < k; ++q) {
                fs_status s3 = apply1(p, true, tn);  // P p
                if (s3 != FS_OK) return s3;
                FS_LAUNCH(h, fs::hvp_vec(n, tn, r, 1.f, nullptr, 0.f, true, tn, st));  // / r
                s3 = apply1(tn, false, tm);  // P^T (P p / r)
                if (s3 != FS_OK) return s3;
                FS_LAUNCH(h, fs::hvp_vec(m, p, c, 1.f, tm, -1.f, false, Ap, st));  // c o p - ...
                FS_LAUNCH(h, fs::hvp_dot(B, m1, Ap, nullptr, part, sum_d, st));
                FS_LAUNCH(h, fs::hvp_center(B, m1, sum_d, Ap, st));
                FS_LAUNCH(h, fs::hvp_dot(B, m1, p, Ap, part, pap_d, st));
                FS_LAUNCH(h, fs::hvp_cg_step(B, m1, rr_d, pap_d, zz_d, tol2, p, Ap, x, res, steps_d, st));
                FS_LAUNCH(h, fs::hvp_dot(B, m1, res, res, part, rrn_d, st));
                FS_LAUNCH(h, fs::hvp_cg_dir(B, m1, rrn_d, rr_d, zz_d, tol2, res, p, st));
                FS_CUDA(h, cudaMemcpyAsync(rr_d, rrn_d, (size_t)B * 8, cudaMemcpyDeviceToDevice, st));
            }
            return FS_OK;
        };
        // Blocks of kCgBlock steps replay one CUDA graph, captured at the first
        // such block on the handle's graph stream (its buffers are this call's);
        // if the capture fails they are launched directly.
        constexpr int kCgBlock = 8;
        cudaGraphExec_t cg_exec = nullptr;
        int cg_kernels = 0;
        bool cg_tried = false;
        auto capture_block = [&]() -> bool {
            cg_tried = true;
            if (!ensure_graph_stream(h)) return false;
            if (cudaStreamBeginCapture(h->gstream, cudaStreamCaptureModeThreadLocal) != cudaSuccess) {
                cudaGetLastError();
                return false;
            }
            const cudaStream_t user = h->stream;
            const std::string saved_error = h->last_error;
            h->stream = h->gstream;
            t_capturing = true;
            t_captured = 0;
            const fs_status s3 = enqueue_steps(kCgBlock);
            t_capturing = false;
            h->stream = user;
            h->last_error = saved_error;
            cudaGraph_t graph = nullptr;
            const cudaError_t ec = cudaStreamEndCapture(h->gstream, &graph);
            const bool good = s3 == FS_OK && ec == cudaSuccess && graph != nullptr &&
                              cudaGraphInstantiate(&cg_exec, graph, 0) == cudaSuccess;
            if (graph) cudaGraphDestroy(graph);
            if (!good) {
                cudaGetLastError();
                cg_exec = nullptr;
                return false;
            }
            cg_kernels = t_captured;
            return true;
        };
        // The host reads the stopping test back after every k steps: k = 1 for the
        // first 16 steps, then up to 8 as the count grows, so at most an eighth
        // more steps run than needed.  A problem that has converged keeps its
        // iterates (the step kernels skip it), so the extra steps change nothing.
        int enqueued = 0;
        fs_status cg_st = FS_OK;
        while (enqueued < max_cg_iters && any_running()) {
            const int k = std::min(max_cg_iters - enqueued, std::max(1, std::min(kCgBlock, enqueued / 8)));
            if (k == kCgBlock && (cg_exec || (!cg_tried && capture_block()))) {
                if (cudaGraphLaunch(cg_exec, s) != cudaSuccess) {
                    cg_st = fail(h, FS_ERR_CUDA, "CUDA graph launch of the CG steps failed");
                    break;
                }
                g_launches.fetch_add((unsigned long long)cg_kernels, std::memory_order_relaxed);
            } else {
                cg_st = enqueue_steps(k);
                if (cg_st != FS_OK) break;
            }
            enqueued += k;
            if (cudaMemcpyAsync(rr.data(), rr_d, (size_t)B * 8, cudaMemcpyDeviceToHost, s) != cudaSuccess ||
                cudaStreamSynchronize(s) != cudaSuccess) {
                cg_st = fail(h, FS_ERR_CUDA, "CG stopping test: %s", cudaGetErrorString(cudaGetLastError()));
                break;
            }
        }
        if (cg_exec) cudaGraphExecDestroy(cg_exec);
        if (cg_st != FS_OK) return cg_st;
        {  // the most steps any problem took
            std::vector<int> steps((size_t)B);
            FS_CUDA(h, cudaMemcpyAsync(steps.data(), steps_d, (size_t)B * 4, cudaMemcpyDeviceToHost, s));
            FS_CUDA(h, cudaStreamSynchronize(s));
            for (int b = 0; b < B; ++b) it = std::max(it, steps[b]);
        }
        // Q1 = P [dg o Y | dg] in one application; df = (u - P dg) / r
        FS_LAUNCH(h, fs::hvp_dgy(Yop, ybf, x, (int)m, (int)d, dgY, s));
        s2 = apply(h, f, g, dgY, false, (int)d + 1, Q1, nullptr, false, true);
        if (s2 != FS_OK) return s2;
        FS_LAUNCH(h, fs::hvp_df(n, (int)d, u, Q1, r, df, s));
        // sum_j P_ij (y_j.v_i) y_j: in one fused pass where the handle's operands
        // allow it (tensor cores), else nq columns of y at a time
        bool fused = false;
        const char *env_fused = getenv("FS_HVP_FUSED"), *env_simt = getenv("FS_APPLY_SIMT");
        if (!(env_fused && atoi(env_fused) == 0) && !(env_simt && atoi(env_simt) != 0)) {
            s2 = hvp_fused_term(h, f, g, Y, V, MV, &fused);
            if (s2 != FS_OK) return s2;
        }
        h->last_hvp_fused = fused ? 1 : 0;
        if (!fused) {
            FS_CUDA(h, cudaMemsetAsync(MV, 0, n * d * 4, s));
            for (int k0 = 0; k0 < (int)d; k0 += nq) {
                const int q = (int)d - k0 < nq ? (int)d - k0 : nq;
                FS_LAUNCH(h, fs::hvp_ychunk(Yop, ybf, (int)m, (int)d, k0, q, Vc, s));
                s2 = apply(h, f, g, Vc, false, q * (int)d, Oc, nullptr, false, true);
                if (s2 != FS_OK) return s2;
                FS_LAUNCH(h, fs::hvp_mv_acc(Vop, Oc, (int)n, (int)d, k0, q, MV, s));
            }
        }
        if (cosine)
            FS_LAUNCH(h, fs::cos_hvp_final(X, bf16, V, PY, df, Q1, MV, n, (int)d, D.eps, out, s));
        else
            FS_LAUNCH(h, fs::hvp_final(X, bf16, V, PY, r, df, Q1, MV, (int)n, (int)d, D.eps, out, s));
        return FS_OK;
    };
    st = run();
    cudaFreeAsync(blk, s);
    if (cg_iters_done) *cg_iters_done = it;
    return st;
}

fs_status fs_selftest_wait(fs_handle *h, int timeout_ms) {
    if (!h || timeout_ms < 1) return fail(h, FS_ERR_INVALID_ARG, "bad argument");
    FS_CUDA(h, cudaSetDevice(h->device));
    FS_LAUNCH(h, fs::launch_wait_probe((unsigned long long)timeout_ms * 1000000ull, h->err, h->stream));
    return check_flags(h);
}

unsigned long long fs_kernel_launches(void) { return g_launches.load(std::memory_order_relaxed); }

const char *fs_last_error(const fs_handle *h) { return h ? h->last_error.c_str() : g_last_error.c_str(); }

fs_status fs_destroy(fs_handle *h) {
    if (!h) return FS_OK;
    cudaSetDevice(h->device);
    // an in-flight replay completes first; these release on completion
    if (h->gexec) cudaGraphExecDestroy(h->gexec);
    if (h->gev_in) cudaEventDestroy(h->gev_in);
    if (h->gev_out) cudaEventDestroy(h->gev_out);
    if (h->gstream) cudaStreamDestroy(h->gstream);
    if (h->block) cudaFreeAsync(h->block, h->stream);  // stream-ordered: no device-wide sync
    delete h;
    return FS_OK;
}

fs_status fs_create(const fs_desc *desc, const void *X, const void *Y, const float *a, const float *b,
                    void *stream, fs_handle **out) {
    if (out) *out = nullptr;
    if (!desc || !X || !Y || !out) return fail(nullptr, FS_ERR_INVALID_ARG, "null argument");
    const fs_desc D = *desc;
    if (D.batch < 1 || D.n < 1 || D.m < 1 || D.d < 1)
        return fail(nullptr, FS_ERR_INVALID_ARG, "sizes must be >= 1 (batch=%d n=%d m=%d d=%d)", D.batch, D.n, D.m,
                    D.d);
    if (!(D.eps > 0.f) || !std::isfinite(D.eps))
        return fail(nullptr, FS_ERR_INVALID_ARG, "eps must be finite and > 0");
    if (D.dtype != FS_F32 && D.dtype != FS_BF16) return fail(nullptr, FS_ERR_INVALID_ARG, "unknown dtype");
    if (D.cost != FS_COST_SQEUCLIDEAN && D.cost != FS_COST_COSINE)
        return fail(nullptr, FS_ERR_INVALID_ARG, "unknown cost");
    if (D.prec != FS_PREC_AUTO && D.prec != FS_PREC_BF16 && D.prec != FS_PREC_TF32 && D.prec != FS_PREC_3XTF32 &&
        D.prec != FS_PREC_3XF16 && D.prec != FS_PREC_F32_SIMT)
        return fail(nullptr, FS_ERR_INVALID_ARG, "unknown precision");
    if ((long long)D.batch * (D.n + 127) > (1LL << 31) || (long long)D.batch * (D.m + 127) > (1LL << 31))
        return fail(nullptr, FS_ERR_UNSUPPORTED, "batch * rows exceeds 2^31");

    fs_handle *h = new fs_handle();
    h->desc = D;
    h->stream = static_cast<cudaStream_t>(stream);
    {
        int major = 0, minor = 0;
        cudaError_t e = cudaGetDevice(&h->device);
        if (e == cudaSuccess) e = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, h->device);
        if (e == cudaSuccess) e = cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, h->device);
        if (e == cudaSuccess) e = cudaDeviceGetAttribute(&h->sms, cudaDevAttrMultiProcessorCount, h->device);
        if (e != cudaSuccess) {
            fail(nullptr, FS_ERR_CUDA, "no CUDA device: %s", cudaGetErrorString(e));
            delete h;
            return FS_ERR_CUDA;
        }
        if (major != 10) {
            fail(nullptr, FS_ERR_UNSUPPORTED, "device is sm_%d%d; this library is built for sm_100a", major, minor);
            delete h;
            return FS_ERR_UNSUPPORTED;
        }
    }
    if (const char *env = getenv("FS_WAIT_TIMEOUT_MS")) {
        // at least 100 ms: the same limit bounds the waits with which a timed-out
        // kernel drains its own copies and MMAs before freeing shared memory and TMEM
        const long long ms = atoll(env);
        if (ms > 0) h->timeout_ns = (unsigned long long)(ms < 100 ? 100 : ms) * 1000000ull;
    }

    // ---- precision and packed layout ----
    int prec = D.prec;
    const bool cosine = D.cost == FS_COST_COSINE;
    if (prec == FS_PREC_AUTO)  // normalised rows are fp32 values, whatever the input dtype
        prec = (D.dtype == FS_BF16 && !cosine) ? FS_PREC_BF16 : (D.d <= 128 ? FS_PREC_3XF16 : FS_PREC_F32_SIMT);
    h->prec = prec;
    if (prec == FS_PREC_F32_SIMT) {
        if (D.d > 256) {
            fail(nullptr, FS_ERR_UNSUPPORTED, "the fp32 SIMT path supports d <= 256");
            delete h;
            return FS_ERR_UNSUPPORTED;
        }
        h->elem = 4;
        h->planes = 1;
        h->d_p = D.d;
        h->row_bytes = D.d * 4;
        h->swz = 0;
        h->plane_bytes = D.d * 4;
        h->pack_mode = fs::kPackPlain;
        h->row_elems = D.d;
    } else {
        h->elem = (prec == FS_PREC_BF16 || prec == FS_PREC_3XF16) ? 2 : 4;
        h->planes = (prec == FS_PREC_3XTF32 || prec == FS_PREC_3XF16) ? 2 : 1;
        const int kstep = 32 / h->elem;  // elements per 32-byte MMA K slice
        h->d_p = round_up(D.d, kstep);
        h->plane_bytes = h->d_p * h->elem;
        const int used = h->planes * h->plane_bytes;
        if (used <= 32) {
            h->row_bytes = 32;
            h->swz = 32;
        } else if (used <= 64) {
            h->row_bytes = 64;
            h->swz = 64;
        } else {
            h->row_bytes = round_up(used, 128);
            h->swz = 128;
        }
        h->pack_mode = prec == FS_PREC_BF16    ? fs::kPackBf16
                       : prec == FS_PREC_TF32  ? fs::kPackTf32
                       : prec == FS_PREC_3XF16 ? fs::kPack3xF16
                                               : fs::kPack3xTf32;
        h->row_elems = h->row_bytes / h->elem;
        // CTA pairs halve the shared memory each CTA spends on column tiles; they
        // serve the rows too wide for the single-CTA ring (512-byte rows), and
        // any width when FS_CTA_PAIR=1.
        h->pair = fs::tc_max_stages(h->row_bytes, 1, true) == 0;
        if (const char *env = getenv("FS_CTA_PAIR")) h->pair = atoi(env) != 0;
        if (h->row_bytes > 512) {  // four swizzle atoms: the kernels' per-tile descriptor table
            fail(nullptr, FS_ERR_UNSUPPORTED,
                 "d=%d needs %d-byte operand rows; the tensor-core pass supports rows up to 512 bytes "
                 "(bf16 d<=256, tf32 and 3xF16 d<=128, 3xTF32 d<=64)",
                 D.d, h->row_bytes);
            delete h;
            return FS_ERR_UNSUPPORTED;
        }
        // Two resident 128-row blocks per CTA when their Q tiles and a K ring of
        // at least one tile plus one slot fit in shared memory: every K tile
        // then serves 256 rows.  FS_ROW_BLOCKS=1 forces one.
        h->qt = fs::tc_max_stages(h->row_bytes, 2, true) > 0 ? 2 : 1;
        if (const char *env = getenv("FS_ROW_BLOCKS")) h->qt = atoi(env) == 1 ? 1 : h->qt;
        h->stages = h->pair ? fs::tc2_max_stages(h->row_bytes, false) : fs::tc_max_stages(h->row_bytes, h->qt, false);
        h->stages_meas =
            h->pair ? fs::tc2_max_stages(h->row_bytes, true) : fs::tc_max_stages(h->row_bytes, h->qt, true);
        if (h->stages < 2 || h->stages_meas < 2) {
            fail(nullptr, FS_ERR_UNSUPPORTED,
                 "d=%d needs %d-byte operand rows; no K ring of at least one tile plus one slot fits in "
                 "shared memory",
                 D.d, h->row_bytes);
            delete h;
            return FS_ERR_UNSUPPORTED;
        }
        h->smem = h->pair ? fs::tc2_smem_bytes(h->row_bytes, h->stages, false)
                          : fs::tc_smem_bytes(h->row_bytes, h->qt, h->stages, false);
        h->smem_meas = h->pair ? fs::tc2_smem_bytes(h->row_bytes, h->stages_meas, true)
                               : fs::tc_smem_bytes(h->row_bytes, h->qt, h->stages_meas, true);
    }
    // Both clouds serve as rows (128-row blocks) and as columns (256-column tiles).
    h->n_pad = round_up(D.n, 256);
    h->m_pad = round_up(D.m, 256);
    h->n_stride = h->n_pad + 256;
    h->m_stride = h->m_pad + 256;
    {
        // CTAs along the rows: one per 128-row block, or per 256 rows on the two-block pass.
        const int rows_per_cta = (prec == FS_PREC_F32_SIMT || h->pair) ? kBlockRows : kBlockRows * h->qt;
        const int tile = kBlockCols;
        plan_splits(D.batch * (h->n_pad / rows_per_cta), (D.m + tile - 1) / tile, h->sms, &h->splits_f, &h->tps_f);
        plan_splits(D.batch * (h->m_pad / rows_per_cta), (D.n + tile - 1) / tile, h->sms, &h->splits_g, &h->tps_g);
    }

    // ---- one device allocation, carved ----
    const size_t B = (size_t)D.batch;
    const size_t max_pad = (size_t)(h->n_pad > h->m_pad ? h->n_pad : h->m_pad);
    const int max_splits = h->splits_f > h->splits_g ? h->splits_f : h->splits_g;
    const size_t max_rb = max_pad / kBlockRows;
    size_t off = 0;
    auto carve = [&](size_t bytes) {
        size_t o = off;
        off += align256(bytes);
        return o;
    };
    const size_t o_packX = carve(B * h->n_pad * h->row_bytes);
    const size_t o_packY = carve(B * h->m_pad * h->row_bytes);
    const size_t o_xn = carve(B * h->n_stride * 4), o_yn = carve(B * h->m_stride * 4);
    const size_t o_la2 = carve(B * h->n_stride * 4), o_lb2 = carve(B * h->m_stride * 4);
    const size_t o_brow = carve(B * h->n_stride * 4), o_bcol = carve(B * h->m_stride * 4);
    const size_t o_bmrow = carve(B * h->n_stride * 32), o_bmcol = carve(B * h->m_stride * 32);
    const size_t o_center = carve(B * D.d * 4);
    const size_t o_rsum = carve(B * max_pad * 4);
    const size_t o_part = carve(max_splits > 1 ? B * max_splits * max_pad * 16 : 16);
    const size_t o_ctr = carve(B * max_rb * 4);
    const size_t o_stats = carve(B * max_rb * 4 * 8);
    const size_t o_red = carve(2 * B * 8 * 8);
    const size_t o_wstat = carve(2 * B * 2 * 8 + 16);
    const size_t o_err = carve(16);
    const size_t o_tail = carve(B * max_rb * 4 * 8);
    const size_t o_snapf = carve(B * D.n * 4), o_snapg = carve(B * D.m * 4);
    const size_t o_cmp = carve(16);
    h->bytes = off;
    {
        cudaMemPool_t pool = nullptr;
        cudaError_t e = device_pool(h->device, &pool);
        if (e == cudaSuccess) e = cudaMallocFromPoolAsync(&h->block, h->bytes, pool, h->stream);
        if (e != cudaSuccess) {
            h->block = nullptr;
            fail(nullptr, e == cudaErrorMemoryAllocation ? FS_ERR_OOM : FS_ERR_CUDA, "allocation of %zu bytes: %s",
                 h->bytes, cudaGetErrorString(e));
            fs_destroy(h);
            return e == cudaErrorMemoryAllocation ? FS_ERR_OOM : FS_ERR_CUDA;
        }
        h->host_red.assign(2 * B * 8 + 4 * B, 0.0);
    }
    char *base = static_cast<char *>(h->block);
    h->packX = base + o_packX;
    h->packY = base + o_packY;
    h->xn = reinterpret_cast<float *>(base + o_xn);
    h->yn = reinterpret_cast<float *>(base + o_yn);
    h->la2 = reinterpret_cast<float *>(base + o_la2);
    h->lb2 = reinterpret_cast<float *>(base + o_lb2);
    h->bias_row = reinterpret_cast<float *>(base + o_brow);
    h->rsum = reinterpret_cast<float *>(base + o_rsum);
    h->bias_col = reinterpret_cast<float *>(base + o_bcol);
    h->bmm_row = base + o_bmrow;
    h->bmm_col = base + o_bmcol;
    h->center = reinterpret_cast<float *>(base + o_center);
    h->part = reinterpret_cast<float4 *>(base + o_part);
    h->counters = reinterpret_cast<unsigned *>(base + o_ctr);
    h->stats = reinterpret_cast<double *>(base + o_stats);
    h->red = reinterpret_cast<double *>(base + o_red);
    h->wstat = reinterpret_cast<double *>(base + o_wstat);
    h->err = reinterpret_cast<int *>(base + o_err);
    h->tail_stats = reinterpret_cast<double *>(base + o_tail);
    h->snap_f = reinterpret_cast<float *>(base + o_snapf);
    h->snap_g = reinterpret_cast<float *>(base + o_snapg);
    h->cmp = reinterpret_cast<int *>(base + o_cmp);

    // ---- set-up kernels ----
    fs_status st = FS_OK;
    auto run = [&]() -> fs_status {
        const bool bf16 = D.dtype == FS_BF16;
        FS_CUDA(h, cudaMemsetAsync(h->counters, 0, B * max_rb * 4, h->stream));
        FS_CUDA(h, cudaMemsetAsync(h->err, 0, 16, h->stream));
        const float *t = nullptr;
        const bool cosine = D.cost == FS_COST_COSINE;  // normalised rows; C is not translation-invariant
        if (!bf16 && !cosine) {
            FS_LAUNCH(h, fs::launch_center(X, Y, bf16, D.batch, D.n, D.m, D.d, h->center, h->stream));
            t = h->center;
        }
        if (h->pack_mode == fs::kPack3xF16) {
            // Power-of-two scales putting each cloud's largest |value| (Y side
            // counted with its factor 2) at most 2^14: exact, and far from the
            // fp16 overflow; the MMA's raw score is divided back by their product.
            float hm[2] = {1.f, 0.5f};  // normalised rows: |value| <= 1 on both sides (Y counted x2 below)
            if (!cosine) {
                float *mx = reinterpret_cast<float *>(h->wstat + 4 * B);
                FS_LAUNCH(h, fs::launch_maxabs(X, bf16, D.n, D.d, D.batch, t, mx, h->stream));
                FS_LAUNCH(h, fs::launch_maxabs(Y, bf16, D.m, D.d, D.batch, t, mx + 1, h->stream));
                FS_CUDA(h, cudaMemcpyAsync(hm, mx, sizeof(hm), cudaMemcpyDeviceToHost, h->stream));
                FS_CUDA(h, cudaStreamSynchronize(h->stream));
            }
            auto pow2_scale = [](float maxabs) {
                if (!(maxabs > 0.f) || !std::isfinite(maxabs)) return 1.f;
                return std::ldexp(1.f, 14 - (int)std::ceil(std::log2((double)maxabs)));
            };
            h->qscale = pow2_scale(hm[0]);
            h->kscale = pow2_scale(2.f * hm[1]);
            h->sscale = 1.f / (h->qscale * h->kscale);
        }
        FS_CUDA(h, cudaMemsetAsync(h->xn, 0, B * h->n_stride * 4, h->stream));
        FS_CUDA(h, cudaMemsetAsync(h->yn, 0, B * h->m_stride * 4, h->stream));
        // K = 2(Y - t) for the squared Euclidean cost, K = Y/|Y| for the cosine cost
        FS_LAUNCH(h, fs::launch_pack(X, bf16, D.n, h->n_pad, D.d, D.batch, t, h->qscale, h->pack_mode, h->d_p,
                                     h->row_elems, h->packX, h->xn, h->n_stride, h->err, h->stream, cosine));
        FS_LAUNCH(h, fs::launch_pack(Y, bf16, D.m, h->m_pad, D.d, D.batch, t, (cosine ? 1.f : 2.f) * h->kscale,
                                     h->pack_mode, h->d_p, h->row_elems, h->packY, h->yn, h->m_stride, h->err,
                                     h->stream, cosine));
        FS_LAUNCH(h, fs::launch_weights(a, D.batch, D.n, h->n_stride, h->la2, h->wstat, h->stream));
        FS_LAUNCH(h, fs::launch_weights(b, D.batch, D.m, h->m_stride, h->lb2, h->wstat + 2 * B, h->stream));
        FS_LAUNCH(h, fs::launch_fill(h->bias_row, B * h->n_stride, -INFINITY, h->stream));
        FS_LAUNCH(h, fs::launch_fill(h->bias_col, B * h->m_stride, -INFINITY, h->stream));
        FS_LAUNCH(h, fs::launch_fill_bias_mm(h->bmm_row, B * h->n_stride, mm_tf32(h), h->stream));
        FS_LAUNCH(h, fs::launch_fill_bias_mm(h->bmm_col, B * h->m_stride, mm_tf32(h), h->stream));
        double *hw = h->host_red.data() + 2 * B * 8;
        FS_CUDA(h, cudaMemcpyAsync(hw, h->wstat, 4 * B * 8, cudaMemcpyDeviceToHost, h->stream));
        FS_CUDA(h, cudaMemcpyAsync(h->host_err, h->err, sizeof(int), cudaMemcpyDeviceToHost, h->stream));
        FS_CUDA(h, cudaMemsetAsync(h->err, 0, 16, h->stream));
        FS_CUDA(h, cudaStreamSynchronize(h->stream));
        for (size_t k = 0; k < 2 * B; ++k) {
            const bool is_a = k < B;
            const double s = hw[2 * k], bad = hw[2 * k + 1];
            if (bad > 0 || !(std::fabs(s - 1.0) <= 1e-5))
                return fail(h, FS_ERR_INVALID_ARG, "weights %s of problem %zu must be positive and sum to 1 (sum=%.9g)",
                            is_a ? "a" : "b", is_a ? k : k - B, s);
        }
        if (h->host_err[0] & fs::kDevErrNonfinite) return fail(h, FS_ERR_NONFINITE, "non-finite value in X or Y");
        if (h->host_err[0] & fs::kDevErrZeroRow)
            return fail(h, FS_ERR_INVALID_ARG, "the cosine cost is undefined for a zero row of X or Y");
        if (prec != FS_PREC_F32_SIMT) {
            fs_status s2 = encode_map(h, &h->mapX_r, h->packX, D.batch * h->n_pad, kBlockRows);
            if (s2 == FS_OK) s2 = encode_map(h, &h->mapX_c, h->packX, D.batch * h->n_pad, kBlockCols);
            if (s2 == FS_OK) s2 = encode_map(h, &h->mapY_r, h->packY, D.batch * h->m_pad, kBlockRows);
            if (s2 == FS_OK) s2 = encode_map(h, &h->mapY_c, h->packY, D.batch * h->m_pad, kBlockCols);
            if (s2 == FS_OK) s2 = encode_bias_map(h, &h->mapBmm_row, h->bmm_row, D.batch * h->n_stride);
            if (s2 == FS_OK) s2 = encode_bias_map(h, &h->mapBmm_col, h->bmm_col, D.batch * h->m_stride);
            if (s2 != FS_OK) return s2;
        }
        return FS_OK;
    };
    st = run();
    if (st != FS_OK) {
        g_last_error = h->last_error;
        fs_destroy(h);
        return st;
    }
    *out = h;
    return FS_OK;
}

fs_status fs_update_f(fs_handle *h, const float *g, float *f) {
    if (!h || !g || !f) return fail(h, FS_ERR_INVALID_ARG, "null argument");
    FS_CUDA(h, cudaSetDevice(h->device));
    return update(h, g, f, true, false);
}

fs_status fs_update_g(fs_handle *h, const float *f, float *g) {
    if (!h || !f || !g) return fail(h, FS_ERR_INVALID_ARG, "null argument");
    FS_CUDA(h, cudaSetDevice(h->device));
    return update(h, f, g, false, false);
}

fs_status fs_solve(fs_handle *h, float *f, float *g, int iters, fs_schedule schedule) {
    if (!h || !f || !g || iters < 0) return fail(h, FS_ERR_INVALID_ARG, "bad argument");
    if (schedule != FS_SCHED_ALTERNATING && schedule != FS_SCHED_SYMMETRIC)
        return fail(h, FS_ERR_INVALID_ARG, "unknown schedule");
    if (iters == 0) return FS_OK;
    h->tail_ok = false;
    h->meas_ok = false;
    FS_CUDA(h, cudaSetDevice(h->device));
    // The whole loop as one CUDA graph where launch latency is a visible part
    // of a pass: batch * n * m up to 2^26 entries (FS_SOLVE_GRAPH=1 forces the
    // graph at every size, FS_SOLVE_GRAPH=0 forbids it).  It is kept for the
    // next call with the same buffers, count and schedule.
    // When the caller is itself capturing the handle's stream, the launches go
    // straight into the caller's graph.
    const char *env = getenv("FS_SOLVE_GRAPH");
    const fs_desc &D = h->desc;
    cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(h->stream, &cap) != cudaSuccess) {  // unknown: launch directly
        cudaGetLastError();
        cap = cudaStreamCaptureStatusActive;
    }
    // A loop of more than 1024 iterations launches directly: its graph would take
    // seconds to capture and hold millions of nodes.
    const bool want_graph = cap == cudaStreamCaptureStatusNone && iters <= 1024 &&
                            (env && *env ? atoi(env) != 0 : (double)D.batch * D.n * D.m <= 67108864.0);
    const bool have = h->gexec && h->gkey_f == f && h->gkey_g == g && h->gkey_iters == iters &&
                      h->gkey_sched == (int)schedule;
    if (want_graph && (have || capture_solve(h, f, g, iters, schedule))) {
        FS_CUDA(h, cudaEventRecord(h->gev_in, h->stream));
        FS_CUDA(h, cudaStreamWaitEvent(h->gstream, h->gev_in, 0));
        FS_CUDA(h, cudaGraphLaunch(h->gexec, h->gstream));
        FS_CUDA(h, cudaEventRecord(h->gev_out, h->gstream));
        FS_CUDA(h, cudaStreamWaitEvent(h->stream, h->gev_out, 0));
        g_launches.fetch_add((unsigned long long)h->gkernels, std::memory_order_relaxed);
        h->last_solve_graph = 1;
    } else {
        h->last_solve_graph = 2;
        const fs_status st = enqueue_solve(h, f, g, iters, schedule);
        if (st != FS_OK) {
            h->tail_ok = false;
            return st;
        }
    }
    h->tail_ok = schedule == FS_SCHED_ALTERNATING;
    h->tail_f = f;
    h->tail_g = g;
    h->meas_ok = false;
    return FS_OK;
}

fs_status fs_marginal_err(fs_handle *h, const float *f, const float *g, double *err_row, double *err_col) {
    if (!h || !f || !g) return fail(h, FS_ERR_INVALID_ARG, "null argument");
    FS_CUDA(h, cudaSetDevice(h->device));
    const size_t B = (size_t)h->desc.batch;
    bool fused = false;
    fs_status s = tail_matches(h, f, g, &fused);
    if (s != FS_OK) return s;
    // fs_ot_cost may have measured this very pair since the solve
    const bool row_cached = err_row && fused && h->meas_ok;
    if (err_row && !row_cached) {
        // with the column sums too, so that fs_ot_cost at the same pair can reuse it
        s = measure(h, f, g, true, 0, true);
        if (s != FS_OK) return s;
    }
    if (err_col) {
        if (fused)  // the solve's final g-pass reduced the column marginal already
            FS_LAUNCH(h, fs::launch_finalize(h->tail_stats, h->desc.batch, h->m_pad / kBlockRows, nullptr, h->lb2,
                                           h->desc.m, h->m_stride, h->red + B * 8, h->stream));
        else {
            s = measure(h, f, g, false, 1, false);
            if (s != FS_OK) return s;
        }
    }
    FS_CUDA(h, cudaMemcpyAsync(h->host_red.data(), h->red, 2 * B * 8 * 8, cudaMemcpyDeviceToHost, h->stream));
    s = check_flags(h);
    if (s != FS_OK) return s;
    for (size_t k = 0; k < B; ++k) {
        if (err_row) err_row[k] = row_cached ? h->meas_cache[k * 8 + 0] : h->host_red[k * 8 + 0];
        if (err_col) err_col[k] = h->host_red[(B + k) * 8 + 0];
    }
    if (fused && err_row && !row_cached) {
        h->meas_cache.assign(h->host_red.begin(), h->host_red.begin() + B * 8);
        h->meas_ok = true;
    }
    h->last_measure_fused = fused ? 1 : 0;
    return FS_OK;
}

fs_status fs_ot_cost(fs_handle *h, const float *f, const float *g, double *dual, double *primal) {
    if (!h || !f || !g) return fail(h, FS_ERR_INVALID_ARG, "null argument");
    FS_CUDA(h, cudaSetDevice(h->device));
    const size_t B = (size_t)h->desc.batch;
    bool fused = false;
    fs_status s = tail_matches(h, f, g, &fused);
    if (s != FS_OK) return s;
    const double *res = nullptr;
    if (fused && h->meas_ok) {  // fs_marginal_err measured this very pair since the solve
        res = h->meas_cache.data();
    } else {
        s = measure(h, f, g, true, 0, true);
        if (s != FS_OK) return s;
        FS_CUDA(h, cudaMemcpyAsync(h->host_red.data(), h->red, B * 8 * 8, cudaMemcpyDeviceToHost, h->stream));
        s = check_flags(h);
        if (s != FS_OK) return s;
        res = h->host_red.data();
        if (fused) {
            h->meas_cache.assign(res, res + B * 8);
            h->meas_ok = true;
        }
    }
    const double eps = (double)h->desc.eps;
    for (size_t k = 0; k < B; ++k) {
        const double *r = res + k * 8;  // [|r-a|, sum r, sum r*meanC, <a,f>, <b,g>]
        if (dual) dual[k] = r[3] + r[4] - eps * (r[1] - 1.0);
        if (primal) primal[k] = r[2];
    }
    h->last_measure_fused = fused ? 1 : 0;
    return FS_OK;
}

fs_status fs_sync(fs_handle *h) {
    if (!h) return fail(nullptr, FS_ERR_INVALID_ARG, "null handle");
    FS_CUDA(h, cudaSetDevice(h->device));
    return check_flags(h);
}

fs_status fs_get_info(const fs_handle *h, fs_info *info) {
    if (!h || !info) return FS_ERR_INVALID_ARG;
    info->prec = h->prec;
    info->d_pad = h->d_p;
    info->row_bytes = h->row_bytes;
    info->swizzle_bytes = h->swz;
    info->stages = h->stages;
    info->block_rows = (h->prec == FS_PREC_F32_SIMT || h->pair) ? kBlockRows : kBlockRows * h->qt;
    info->block_cols = kBlockCols;
    info->splits_f = h->splits_f;
    info->splits_g = h->splits_g;
    info->launches_update = 2;
    info->launches_solve_iter = 2;
    info->device_bytes = h->bytes;
    info->cta_pair = (h->prec != FS_PREC_F32_SIMT && h->pair) ? 1 : 0;
    info->last_apply_path = h->last_apply;
    info->last_solve_graph = h->last_solve_graph;
    info->last_measure_fused = h->last_measure_fused;
    info->last_hvp_fused = h->last_hvp_fused;
    info->last_apply_parts = h->last_apply_parts;
    return FS_OK;
}

fs_status fs_solve_host(const fs_desc *desc, const void *X_host, const void *Y_host, const float *a_host,
                        const float *b_host, float *f_host, float *g_host, int iters, fs_schedule schedule,
                        double *err_row, double *err_col, double *dual, double *primal, void *stream) {
    if (!desc || !X_host || !Y_host || !f_host || !g_host || iters < 0)
        return fail(nullptr, FS_ERR_INVALID_ARG, "null or bad argument");
    const fs_desc D = *desc;
    if (D.batch < 1 || D.n < 1 || D.m < 1 || D.d < 1)
        return fail(nullptr, FS_ERR_INVALID_ARG, "sizes must be >= 1");
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const size_t B = (size_t)D.batch, es = D.dtype == FS_BF16 ? 2 : 4;
    const size_t bx = B * D.n * D.d * es, by = B * D.m * D.d * es, bf = B * D.n * 4, bg = B * D.m * 4;
    const size_t total = align256(bx) + align256(by) + 2 * align256(bf) + 2 * align256(bg);
    char *blk = nullptr;
    int dev = 0;
    cudaMemPool_t pool = nullptr;
    cudaError_t e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = device_pool(dev, &pool);
    if (e == cudaSuccess) e = cudaMallocFromPoolAsync((void **)&blk, total, pool, s);
    if (e != cudaSuccess)
        return fail(nullptr, e == cudaErrorMemoryAllocation ? FS_ERR_OOM : FS_ERR_CUDA, "cudaMallocAsync: %s",
                    cudaGetErrorString(e));
    char *dX = blk, *dY = dX + align256(bx);
    float *da = reinterpret_cast<float *>(dY + align256(by));
    float *df = reinterpret_cast<float *>(reinterpret_cast<char *>(da) + align256(bf));
    float *db = reinterpret_cast<float *>(reinterpret_cast<char *>(df) + align256(bf));
    float *dg = reinterpret_cast<float *>(reinterpret_cast<char *>(db) + align256(bg));
    fs_handle *h = nullptr;
    fs_status st = FS_OK;
    auto body = [&]() -> fs_status {
        FS_CUDA(nullptr, cudaMemcpyAsync(dX, X_host, bx, cudaMemcpyHostToDevice, s));
        FS_CUDA(nullptr, cudaMemcpyAsync(dY, Y_host, by, cudaMemcpyHostToDevice, s));
        if (a_host) FS_CUDA(nullptr, cudaMemcpyAsync(da, a_host, bf, cudaMemcpyHostToDevice, s));
        if (b_host) FS_CUDA(nullptr, cudaMemcpyAsync(db, b_host, bg, cudaMemcpyHostToDevice, s));
        FS_CUDA(nullptr, cudaMemcpyAsync(dg, g_host, bg, cudaMemcpyHostToDevice, s));
        fs_status r = fs_create(&D, dX, dY, a_host ? da : nullptr, b_host ? db : nullptr, s, &h);
        if (r != FS_OK) return r;
        r = fs_solve(h, df, dg, iters, schedule);
        if (r == FS_OK && (err_row || err_col)) r = fs_marginal_err(h, df, dg, err_row, err_col);
        if (r == FS_OK && (dual || primal)) r = fs_ot_cost(h, df, dg, dual, primal);
        if (r != FS_OK) {
            g_last_error = h->last_error;
            return r;
        }
        FS_CUDA(h, cudaMemcpyAsync(f_host, df, bf, cudaMemcpyDeviceToHost, s));
        FS_CUDA(h, cudaMemcpyAsync(g_host, dg, bg, cudaMemcpyDeviceToHost, s));
        return fs_sync(h);
    };
    st = body();
    if (st != FS_OK && h) g_last_error = h->last_error;
    fs_destroy(h);
    cudaFreeAsync(blk, s);
    cudaStreamSynchronize(s);
    return st;
}

}  // extern "C"
