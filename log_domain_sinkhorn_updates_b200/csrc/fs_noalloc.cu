// fs_update_f_noalloc: one f-update that allocates nothing.
//
// Who needs it: callers that cannot allocate device memory at the moment
// they need an update.  Examples are plug-ins whose host framework owns all
// device memory and forbids allocations by third-party code, services that
// reserve a fixed memory budget up front, and latency-critical loops where
// an allocation, with the synchronisation it can imply, is not acceptable.
// The handle API cannot serve them: fs_create allocates the handle's buffers
// and synchronises.
//
// This entry point takes the raw fp32 clouds and potentials and writes f.
// Its only scratch is one file-scope device array of kScratchFloats floats
// (4 MiB).  Every GPU that loads this library holds it until the process
// exits.  The array holds the centring sums and the common centre, the
// squared norms of both centred clouds, and the column bias of the pass.
// Consequences for the caller:
//  * d <= 256 and n_pad + m + m_pad <= kScratchFloats - kReserved
//    (n_pad, m_pad: n, m rounded up to 128; kReserved floats hold the
//    centring sums); larger problems are rejected with FS_ERR_INVALID_ARG;
//  * every call on a device shares the array, and the array keeps the last
//    call's contents, so calls whose kernels overlap on the GPU (different
//    streams, or different host threads, without ordering between them)
//    race and corrupt each other's results; order them on one stream or
//    synchronise between them;
//  * the first call on each device looks up the array's device address
//    (cudaGetSymbolAddress) and sets the kernel's shared-memory limit.  The address is kept
//    per device index for the life of the process; after cudaDeviceReset the
//    kept address refers to the old context, so do not use this entry point
//    after resetting a device.
// The arithmetic is the library's plain-fp32 pass (FMA dot products on CUDA
// cores, online base-2 LSE, accurate exp2f) on inputs shifted by the common
// centre t = (mean X + mean Y)/2, as the handle path does: C_ij is
// translation-invariant, and the shift keeps |x - t|^2, |y - t|^2 and
// 2 (x - t).(y - t) small when both clouds sit far from the origin.
#include <mutex>

#include "flashsinkhorn.h"
#include "fs_internal.cuh"

namespace {

constexpr size_t kScratchFloats = size_t(1) << 20;  // 4 MiB
constexpr int kMaxDevices = 64;
constexpr int kCols = 32;          // columns staged in shared memory per step
constexpr int kMaxD = 256;         // shared-memory tiles of 128 + 32 rows of d floats
constexpr int kCenterBlocks = 64;  // blocks of the centring sums
// Floats reserved ahead of the per-point arrays: the centring partial sums
// (kCenterBlocks x 2 clouds x kMaxD doubles) and the centre t (kMaxD floats).
constexpr size_t kReserved = (size_t)kCenterBlocks * 2 * kMaxD * 2 + kMaxD;

static __device__ __align__(256) float g_scratch[kScratchFloats];

// Per block b: sums over the rows b, b + G, ... of X and of Y, dimension k
// per thread, in double -> part[b][0][k], part[b][1][k].
__global__ void __launch_bounds__(kMaxD) noalloc_center_partial(const float *X, int n, const float *Y, int m, int d,
                                                               double *part) {
    const int k = threadIdx.x;
    if (k >= d) return;
    double sx = 0.0, sy = 0.0;
    for (int r = blockIdx.x; r < n; r += gridDim.x) sx += (double)X[(size_t)r * d + k];
    for (int r = blockIdx.x; r < m; r += gridDim.x) sy += (double)Y[(size_t)r * d + k];
    part[((size_t)blockIdx.x * 2 + 0) * kMaxD + k] = sx;
    part[((size_t)blockIdx.x * 2 + 1) * kMaxD + k] = sy;
}

// t_k = (mean X + mean Y)_k / 2 from the partial sums, added in block order.
__global__ void __launch_bounds__(kMaxD) noalloc_center_final(const double *part, int blocks, int n, int m, int d,
                                                             float *t) {
    const int k = threadIdx.x;
    if (k >= d) return;
    double sx = 0.0, sy = 0.0;
    for (int b = 0; b < blocks; ++b) {
        sx += part[((size_t)b * 2 + 0) * kMaxD + k];
        sy += part[((size_t)b * 2 + 1) * kMaxD + k];
    }
    t[k] = (float)(0.5 * (sx / n + sy / m));
}

// |p_r - t|^2 for r < rows (double accumulation, one warp per row).
__global__ void noalloc_norms(const float *P, const float *t, int rows, int d, float *out) {
    const int lane = threadIdx.x & 31;
    const long long w0 = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const long long nw = ((long long)gridDim.x * blockDim.x) >> 5;
    for (long long r = w0; r < rows; r += nw) {
        double acc = 0.0;
        for (int k = lane; k < d; k += 32) {
            const double v = (double)(P[(size_t)r * d + k] - t[k]);
            acc += v * v;
        }
        for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
        if (lane == 0) out[r] = (float)acc;
    }
}

// beta_j = (g_j - |y_j - t|^2) log2(e)/eps + log2 b_j, -inf for j >= m.
__global__ void noalloc_bias(const float *g, const float *b, const float *ynorm, int m, int m_pad, double scale2,
                             float *bias) {
    const double ulog = -log2((double)m);
    for (int j = blockIdx.x * blockDim.x + threadIdx.x; j < m_pad; j += gridDim.x * blockDim.x) {
        float v = -INFINITY;
        if (j < m)
            v = (float)__fma_rn((double)g[j] - (double)ynorm[j], scale2, b ? log2((double)b[j]) : ulog);
        bias[j] = v;
    }
}

// f_i = |x_i - t|^2 - eps ln2 log2 sum_j 2^(2 (x_i - t).(y_j - t) log2(e)/eps + beta_j),
// one thread per row.
__global__ void __launch_bounds__(fs::kBlockRows)
    noalloc_lse(const float *X, const float *Y, const float *t, int n, int m, int d, const float *bias,
                const float *xnorm, float scale2x2, double eps, float *f) {
    extern __shared__ float sm[];
    const int ld = d + 1;
    float *srow = sm;                               // [128][d+1]
    float *scol = srow + fs::kBlockRows * ld;       // [32][d]
    float *sbias = scol + kCols * d;                // [32]
    const int rl = threadIdx.x;
    const int row0 = blockIdx.x * fs::kBlockRows;
    for (int e = rl; e < fs::kBlockRows * d; e += fs::kBlockRows) {
        const int r = row0 + e / d;
        srow[(e / d) * ld + (e % d)] = r < n ? X[(size_t)row0 * d + e] - t[e % d] : 0.f;
    }
    float mx = -INFINITY, l = 0.f;
    for (int c0 = 0; c0 < m; c0 += kCols) {
        __syncthreads();
        for (int e = rl; e < kCols * d; e += fs::kBlockRows)
            scol[e] = (c0 + e / d) < m ? Y[(size_t)c0 * d + e] - t[e % d] : 0.f;
        if (rl < kCols) sbias[rl] = bias[c0 + rl];  // bias is padded to a multiple of 128 with -inf
        __syncthreads();
        float z[kCols];
        float tmax = -INFINITY;
        for (int j = 0; j < kCols; ++j) {
            float s = 0.f;
            for (int k = 0; k < d; ++k) s = fmaf(srow[rl * ld + k], scol[j * d + k], s);
            z[j] = fmaf(s, scale2x2, sbias[j]);
            tmax = fmaxf(tmax, z[j]);
        }
        const float mnew = fmaxf(mx, tmax);
        if (mnew == -INFINITY) continue;
        float acc = 0.f;
        for (int j = 0; j < kCols; ++j) acc += exp2f(z[j] - mnew);
        l = l * exp2f(mx - mnew) + acc;
        mx = mnew;
    }
    const int row = row0 + rl;
    if (row < n) f[row] = (float)((double)xnorm[row] - eps * fs::kLn2d * ((double)mx + log2((double)l)));
}

size_t lse_smem_bytes(int d) { return sizeof(float) * ((size_t)fs::kBlockRows * (d + 1) + (size_t)kCols * d + kCols); }

std::mutex g_mu;
float *g_scratch_ptr[kMaxDevices] = {};

// Once per device, with that device current: the device address of the
// scratch array (host code only sees a stand-in for it) and the kernel's
// shared-memory limit.
cudaError_t scratch_for_device(int dev, float **out) {
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_scratch_ptr[dev]) {
        float *p = nullptr;
        cudaError_t e = cudaGetSymbolAddress(reinterpret_cast<void **>(&p), g_scratch);
        if (e != cudaSuccess) return e;
        e = cudaFuncSetAttribute(noalloc_lse, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)lse_smem_bytes(kMaxD));
        if (e != cudaSuccess) return e;
        g_scratch_ptr[dev] = p;
    }
    *out = g_scratch_ptr[dev];
    return cudaSuccess;
}

// Errors are reported like every other call without a handle: the message
// is what fs_last_error(NULL) returns on this thread.
fs_status reject(fs_status st, const char *msg) {
    fs::set_thread_error(msg);
    return st;
}

}  // namespace

extern "C" {

fs_status fs_update_f_noalloc(int n, int m, int d, float eps, const float *X, const float *Y, const float *b,
                              const float *g, float *f, void *stream) {
    if (!X || !Y || !g || !f) return reject(FS_ERR_INVALID_ARG, "null argument");
    if (n < 1 || m < 1 || d < 1) return reject(FS_ERR_INVALID_ARG, "sizes must be >= 1");
    if (!(eps > 0.f) || !isfinite(eps)) return reject(FS_ERR_INVALID_ARG, "eps must be finite and > 0");
    if (d > kMaxD) return reject(FS_ERR_INVALID_ARG, "d exceeds 256, the limit of the allocation-free update");
    const size_t n_pad = ((size_t)n + fs::kBlockRows - 1) / fs::kBlockRows * fs::kBlockRows;
    const size_t m_pad = ((size_t)m + fs::kBlockRows - 1) / fs::kBlockRows * fs::kBlockRows;
    if (n_pad + (size_t)m + m_pad > kScratchFloats - kReserved)
        return reject(FS_ERR_INVALID_ARG,
                      "n + 2m (each rounded up to 128) exceeds the 982784 floats left for points in the 4 MiB "
                      "static scratch of the allocation-free update");
    int dev = 0, major = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
    if (e != cudaSuccess) return reject(FS_ERR_CUDA, cudaGetErrorString(e));
    if (major != 10) return reject(FS_ERR_UNSUPPORTED, "this library is built for sm_100a");
    if (dev >= kMaxDevices) return reject(FS_ERR_UNSUPPORTED, "device index beyond 63");
    float *scratch = nullptr;
    e = scratch_for_device(dev, &scratch);
    if (e != cudaSuccess) return reject(FS_ERR_CUDA, cudaGetErrorString(e));

    double *part = reinterpret_cast<double *>(scratch);           // [kCenterBlocks][2][kMaxD]
    float *t = scratch + (size_t)kCenterBlocks * 2 * kMaxD * 2;    // [kMaxD]
    float *xnorm = scratch + kReserved;                            // [n_pad]
    float *ynorm = xnorm + n_pad;                                  // [m]
    float *bias = ynorm + m;                                       // [m_pad]
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const int nb = (int)((((size_t)n > (size_t)m ? n : m) * 32 + 255) / 256);
    // Every value these kernels read from the scratch is written earlier in
    // the same call, so nothing a previous call left there is used.
    noalloc_center_partial<<<kCenterBlocks, kMaxD, 0, s>>>(X, n, Y, m, d, part);
    noalloc_center_final<<<1, kMaxD, 0, s>>>(part, kCenterBlocks, n, m, d, t);
    noalloc_norms<<<nb < 4096 ? nb : 4096, 256, 0, s>>>(X, t, n, d, xnorm);
    noalloc_norms<<<nb < 4096 ? nb : 4096, 256, 0, s>>>(Y, t, m, d, ynorm);
    noalloc_bias<<<(int)((m_pad + 255) / 256), 256, 0, s>>>(g, b, ynorm, m, (int)m_pad, fs::kLog2ed / (double)eps,
                                                           bias);
    noalloc_lse<<<(int)(n_pad / fs::kBlockRows), fs::kBlockRows, lse_smem_bytes(d), s>>>(
        X, Y, t, n, m, d, bias, xnorm, (float)(2.0 * fs::kLog2ed / (double)eps), (double)eps, f);
    e = cudaGetLastError();
    if (e != cudaSuccess) return reject(FS_ERR_CUDA, cudaGetErrorString(e));
    fs::count_launches(6);
    return FS_OK;
}

}  // extern "C"
