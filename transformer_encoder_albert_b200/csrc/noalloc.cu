// noalloc.cu -- the residual + LayerNorm GEMM behind an entry point that
// allocates no device memory.
//
// Some hosts must not call cudaMalloc once they are running: a real-time audio
// thread that feeds the encoder's features to a speech decoder cannot absorb
// the device-wide synchronization and unbounded latency an allocation may
// bring, and runtimes that plan all device memory up front (an arena laid out
// before the first request) forbid allocations behind their back.  For them,
// albert_gemm_residual_ln_noalloc runs the same kernel as the rest of the
// library (Y = LN(A W^T + bias + R; gamma, beta)) with its scratch memory --
// the per-row statistics and epoch flags that the LayerNorm epilogue's column
// tiles exchange, the row-count word and the status word -- in file-scope
// __device__ arrays instead of memory the call allocates.
#include <cuda_runtime.h>

#include <atomic>
#include <mutex>

#include "albert.h"
#include "kernels.h"

namespace albert {
namespace {

// The static arrays hold the LayerNorm exchange buffers for up to this many
// rows: 8192 rows x 3 tiles of (mean, M2) fp32 = 192 KiB of statistics plus
// 64 row blocks x 4 lane quadrants x 3 tiles epoch flags (3 KiB).
constexpr int kNoAllocMaxRows = 8192;
constexpr size_t kNoAllocStats = (size_t)kNoAllocMaxRows * (gemm::LN_N / gemm::BN);
constexpr size_t kNoAllocFlags = (size_t)(kNoAllocMaxRows / gemm::BM) * 4 * (gemm::LN_N / gemm::BN);

static __device__ __align__(256) float2 g_ln_stats[kNoAllocStats];
static __device__ __align__(256) int g_ln_flags[kNoAllocFlags];
static __device__ __align__(256) int g_ln_words[2];  // [0] rows to process, [1] status

// Flags hold the epoch of the call that wrote them; every call uses a larger one.
std::atomic<int> g_epoch{0};

constexpr int kMaxDevices = 128;
std::mutex g_setup_mu;
float2 *g_stats_dev[kMaxDevices] = {};
int *g_flags_dev[kMaxDevices] = {};
int *g_words_dev[kMaxDevices] = {};

__global__ void reset_words_kernel(int *words, int rows) {
    words[0] = rows;
    words[1] = 0;  // the status word must start at zero on every call
}

// Device addresses of the static arrays on the current device, looked up once.
int setup_device(int dev, float2 **stats, int **flags, int **words) {
    if (dev < 0 || dev >= kMaxDevices) return ALBERT_ERR_CONFIG;
    std::lock_guard<std::mutex> lock(g_setup_mu);
    if (!g_stats_dev[dev]) {
        void *s = nullptr, *f = nullptr, *w = nullptr;
        if (cudaGetSymbolAddress(&s, g_ln_stats) != cudaSuccess) return ALBERT_ERR_CUDA;
        if (cudaGetSymbolAddress(&f, g_ln_flags) != cudaSuccess) return ALBERT_ERR_CUDA;
        if (cudaGetSymbolAddress(&w, g_ln_words) != cudaSuccess) return ALBERT_ERR_CUDA;
        g_stats_dev[dev] = static_cast<float2 *>(s);
        g_flags_dev[dev] = static_cast<int *>(f);
        g_words_dev[dev] = static_cast<int *>(w);
    }
    *stats = g_stats_dev[dev];
    *flags = g_flags_dev[dev];
    *words = g_words_dev[dev];
    return ALBERT_OK;
}

}  // namespace
}  // namespace albert

using namespace albert;

extern "C" int albert_gemm_residual_ln_noalloc(const void *A, const void *W, const float *bias, const void *R,
                                              const float *ln_g, const float *ln_b, float eps, void *Y, int M,
                                              int K, void *stream) {
    if (!A || !W || !bias || !R || !ln_g || !ln_b || !Y) return ALBERT_ERR_NULL;
    if (M < 1 || M > kNoAllocMaxRows || K < gemm::BK || K % gemm::BK) return ALBERT_ERR_SHAPE;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return ALBERT_ERR_CUDA;
    float2 *stats = nullptr;
    int *flags = nullptr, *words = nullptr;
    int rc = setup_device(dev, &stats, &flags, &words);
    if (rc) return rc;
    int sms = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return ALBERT_ERR_CUDA;

    const int N = gemm::LN_N;
    const int rows_cap = (M + gemm::BM - 1) / gemm::BM * gemm::BM;
    const int grid = gemm_grid(kEpiLN, rows_cap, N, sms);
    CUtensorMap ta, tb, to, tr;
    if (make_tmap_bf16(&ta, A, M, K, gemm::BM) || make_tmap_bf16(&tb, W, N, K, gemm::BN) ||
        make_tmap_bf16_tile32(&to, Y, M, N) || make_tmap_bf16_tile32(&tr, R, M, N))
        return ALBERT_ERR_CUDA;

    reset_words_kernel<<<1, 1, 0, s>>>(words, M);
    if (cudaGetLastError() != cudaSuccess) return ALBERT_ERR_CUDA;
    GemmArgs a{};
    a.N = N;
    a.K = K;
    a.rows_cap = rows_cap;
    a.n_rows = words;
    a.bias = bias;
    a.resid = static_cast<const bf16 *>(R);
    a.ld_resid = N;
    a.ln_g = ln_g;
    a.ln_b = ln_b;
    a.eps = eps;
    a.out = static_cast<bf16 *>(Y);
    a.ld_out = N;
    a.ln_stats = stats;
    a.ln_flags = flags;
    a.epoch = ++g_epoch;
    a.status = words + 1;
    if (launch_gemm(kEpiLN, ta, tb, to, tr, a, grid, s) != cudaSuccess) return ALBERT_ERR_CUDA;
    int st = 0;
    if (cudaMemcpyAsync(&st, words + 1, sizeof(int), cudaMemcpyDeviceToHost, s) != cudaSuccess) return ALBERT_ERR_CUDA;
    if (cudaStreamSynchronize(s) != cudaSuccess) return ALBERT_ERR_CUDA;
    return st;
}
