// fs_update_f_noalloc: one f-update that allocates nothing.
//
// For callers that cannot allocate device memory at the moment they need
// an update -- code running while a CUDA graph is being captured (cudaMalloc
// is not a capturable operation), plug-ins whose host framework owns all
// device memory and forbids driver allocations, and latency-critical loops
// where an allocation (and the synchronisation it can imply) is not
// acceptable.  The handle API cannot serve them: fs_create allocates the
// handle's buffers and synchronises.
//
// This entry point takes the raw fp32 clouds and potentials and writes f.
// Its only scratch -- the squared norms of both clouds and the column bias
// of the pass -- lives in one file-scope device array of kScratchFloats
// floats (4 MiB), which every GPU that loads this library holds until the
// process exits.  Consequences for the caller:
//  * n_pad + m + m_pad <= kScratchFloats (n_pad, m_pad: n, m rounded up to
//    128); larger problems are rejected with FS_ERR_INVALID_ARG;
//  * every call on a device shares the array, so calls whose kernels
//    overlap on the GPU (different streams, or different host threads,
//    without ordering between them) race and corrupt each other's results;
//    order them on one stream or synchronise between them;
//  * the first call on each device looks up the array's device address
//    (cudaGetSymbolAddress) and sets the kernel's shared-memory limit; make
//    that first call before any stream capture begins.
// The arithmetic is the library's plain-fp32 pass (FMA dot products on CUDA
// cores, online base-2 LSE, accurate exp2f) on uncentred inputs.
#include <mutex>

#include "flashsinkhorn.h"
#include "fs_internal.cuh"

namespace {

constexpr size_t kScratchFloats = size_t(1) << 20;  // 4 MiB
constexpr int kMaxDevices = 64;
constexpr int kCols = 32;   // columns staged in shared memory per step
constexpr int kMaxD = 256;  // shared-memory tiles of 128 + 32 rows of d floats

static __device__ __align__(256) float g_scratch[kScratchFloats];

// |p_r|^2 for r < rows (double accumulation, one warp per row).
__global__ void noalloc_norms(const float *P, int rows, int d, float *out) {
    const int lane = threadIdx.x & 31;
    const long long w0 = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const long long nw = ((long long)gridDim.x * blockDim.x) >> 5;
    for (long long r = w0; r < rows; r += nw) {
        double acc = 0.0;
        for (int k = lane; k < d; k += 32) {
            const double v = P[(size_t)r * d + k];
            acc += v * v;
        }
        for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
        if (lane == 0) out[r] = (float)acc;
    }
}

// beta_j = (g_j - |y_j|^2) log2(e)/eps + log2 b_j, -inf for j >= m.
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

// f_i = |x_i|^2 - eps ln2 log2 sum_j 2^(2 x_i.y_j log2(e)/eps + beta_j), one thread per row.
__global__ void __launch_bounds__(fs::kBlockRows)
    noalloc_lse(const float *X, const float *Y, int n, int m, int d, const float *bias, const float *xnorm,
                float scale2x2, double eps, float *f) {
    extern __shared__ float sm[];
    const int ld = d + 1;
    float *srow = sm;                               // [128][d+1]
    float *scol = srow + fs::kBlockRows * ld;       // [32][d]
    float *sbias = scol + kCols * d;                // [32]
    const int rl = threadIdx.x;
    const int row0 = blockIdx.x * fs::kBlockRows;
    for (int e = rl; e < fs::kBlockRows * d; e += fs::kBlockRows) {
        const int r = row0 + e / d;
        srow[(e / d) * ld + (e % d)] = r < n ? X[(size_t)row0 * d + e] : 0.f;
    }
    float mx = -INFINITY, l = 0.f;
    for (int c0 = 0; c0 < m; c0 += kCols) {
        __syncthreads();
        for (int e = rl; e < kCols * d; e += fs::kBlockRows)
            scol[e] = (c0 + e / d) < m ? Y[(size_t)c0 * d + e] : 0.f;
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
    if (n_pad + (size_t)m + m_pad > kScratchFloats)
        return reject(FS_ERR_INVALID_ARG,
                      "n + 2m (each rounded up to 128) exceeds the 1048576-float static scratch of the "
                      "allocation-free update");
    int dev = 0, major = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
    if (e != cudaSuccess) return reject(FS_ERR_CUDA, cudaGetErrorString(e));
    if (major != 10) return reject(FS_ERR_UNSUPPORTED, "this library is built for sm_100a");
    if (dev >= kMaxDevices) return reject(FS_ERR_UNSUPPORTED, "device index beyond 63");
    float *scratch = nullptr;
    e = scratch_for_device(dev, &scratch);
    if (e != cudaSuccess) return reject(FS_ERR_CUDA, cudaGetErrorString(e));

    float *xnorm = scratch;             // [n_pad]
    float *ynorm = xnorm + n_pad;       // [m]
    float *bias = ynorm + m;            // [m_pad]
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const int nb = (int)((((size_t)n > (size_t)m ? n : m) * 32 + 255) / 256);
    noalloc_norms<<<nb < 4096 ? nb : 4096, 256, 0, s>>>(X, n, d, xnorm);
    noalloc_norms<<<nb < 4096 ? nb : 4096, 256, 0, s>>>(Y, m, d, ynorm);
    noalloc_bias<<<(int)((m_pad + 255) / 256), 256, 0, s>>>(g, b, ynorm, m, (int)m_pad, fs::kLog2ed / (double)eps,
                                                           bias);
    noalloc_lse<<<(int)(n_pad / fs::kBlockRows), fs::kBlockRows, lse_smem_bytes(d), s>>>(
        X, Y, n, m, d, bias, xnorm, (float)(2.0 * fs::kLog2ed / (double)eps), (double)eps, f);
    e = cudaGetLastError();
    if (e != cudaSuccess) return reject(FS_ERR_CUDA, cudaGetErrorString(e));
    return FS_OK;
}

}  // extern "C"
