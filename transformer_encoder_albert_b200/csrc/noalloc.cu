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
// the per-CTA fp32 row slots of the LayerNorm epilogue, the row-count word and
// the status word -- in a file-scope __device__ array instead of memory the
// call allocates.
#include <cuda_runtime.h>

#include <mutex>

#include "albert.h"
#include "kernels.h"

namespace albert {
namespace {

// The static array holds the LayerNorm scratch of this many CTAs, one CTA per
// 128-row block: 16 x 128 x 768 fp32 = 6 MiB, so M <= 2048 rows.
constexpr int kNoAllocSlots = 16;
constexpr int kNoAllocMaxRows = kNoAllocSlots * gemm::BM;
constexpr size_t kNoAllocScratchFloats = (size_t)kNoAllocSlots * gemm::BM * gemm::LN_N;

static __device__ __align__(256) float g_ln_scratch[kNoAllocScratchFloats];
static __device__ __align__(256) int g_ln_words[2];  // [0] rows to process, [1] status

constexpr int kMaxDevices = 128;
std::mutex g_setup_mu;
float *g_scratch_dev[kMaxDevices] = {};
int *g_words_dev[kMaxDevices] = {};

__global__ void reset_words_kernel(int *words, int rows) {
    words[0] = rows;
    words[1] = 0;  // the status word must start at zero on every call
}

// Device addresses of the static array on the current device, looked up once.
int setup_device(int dev, float **scratch, int **words) {
    if (dev < 0 || dev >= kMaxDevices) return ALBERT_ERR_CONFIG;
    std::lock_guard<std::mutex> lock(g_setup_mu);
    if (!g_scratch_dev[dev]) {
        void *s = nullptr, *w = nullptr;
        if (cudaGetSymbolAddress(&s, g_ln_scratch) != cudaSuccess) return ALBERT_ERR_CUDA;
        if (cudaGetSymbolAddress(&w, g_ln_words) != cudaSuccess) return ALBERT_ERR_CUDA;
        g_scratch_dev[dev] = static_cast<float *>(s);
        g_words_dev[dev] = static_cast<int *>(w);
    }
    *scratch = g_scratch_dev[dev];
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
    float *scratch = nullptr;
    int *words = nullptr;
    int rc = setup_device(dev, &scratch, &words);
    if (rc) return rc;

    const int N = gemm::LN_N;
    const int rows_cap = (M + gemm::BM - 1) / gemm::BM * gemm::BM;
    const int grid = rows_cap / gemm::BM;  // one CTA per row block: <= kNoAllocSlots scratch slots
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
    a.scratch = scratch;
    a.status = words + 1;
    if (launch_gemm(kEpiLN, ta, tb, to, tr, a, grid, s) != cudaSuccess) return ALBERT_ERR_CUDA;
    int st = 0;
    if (cudaMemcpyAsync(&st, words + 1, sizeof(int), cudaMemcpyDeviceToHost, s) != cudaSuccess) return ALBERT_ERR_CUDA;
    if (cudaStreamSynchronize(s) != cudaSuccess) return ALBERT_ERR_CUDA;
    return st;
}
