// noalloc.cu -- the residual + LayerNorm GEMM behind an entry point that
// allocates no device memory.
//
// Some hosts must not call cudaMalloc once they are running: a real-time audio
// thread that feeds the encoder's features to a speech decoder cannot absorb
// the device-wide synchronization and unbounded latency an allocation may
// bring, and runtimes that plan all device memory up front (an arena laid out
// before the first request) forbid allocations behind their back.  For them,
// albert_gemm_residual_ln_noalloc computes Y = LN(A W^T + bias + R; gamma, beta)
// with the same two kernels as the rest of the library -- the GEMM whose
// epilogue forms z = A W^T + bias + R, writes z * gamma and per-row partial
// statistics, then the row normalization -- and keeps their scratch memory
// (z * gamma, the statistics, the row-count word and the status word) in
// file-scope __device__ arrays instead of memory the call allocates.
#include <cuda_runtime.h>

#include "albert.h"
#include "kernels.h"

namespace albert {
namespace {

// The static arrays hold the intermediates of up to this many rows:
// z * gamma, 2048 x 768 bf16 (3 MiB), and 2048 x 6 (mean, M2) fp32 pairs (96 KiB).
constexpr int kNoAllocMaxRows = 2048;
constexpr size_t kNoAllocZg = (size_t)kNoAllocMaxRows * gemm::LN_N;
constexpr size_t kNoAllocStats = (size_t)kNoAllocMaxRows * gemm::LN_PARTS;

static __device__ __align__(256) bf16 g_ln_zg[kNoAllocZg];
static __device__ __align__(256) float2 g_ln_stats[kNoAllocStats];
static __device__ __align__(256) int g_ln_words[2];  // [0] rows to process, [1] status

__global__ void reset_words_kernel(int *words, int rows) {
    words[0] = rows;
    words[1] = 0;  // the status word must start at zero on every call
}

// Device addresses of the static arrays on the current device.  In host code
// the arrays' names stand for host-side shadows, so their device addresses are
// looked up with the device current.  The lookup runs on every call: it is
// cheap and allocates nothing once the library's module is loaded on the
// device, and a cached address would go stale if the device's primary context
// were reset and the module loaded again elsewhere.
int lookup_scratch(bf16 **zg, float2 **stats, int **words) {
    void *z = nullptr, *st = nullptr, *w = nullptr;
    if (cudaGetSymbolAddress(&z, g_ln_zg) != cudaSuccess) return ALBERT_ERR_CUDA;
    if (cudaGetSymbolAddress(&st, g_ln_stats) != cudaSuccess) return ALBERT_ERR_CUDA;
    if (cudaGetSymbolAddress(&w, g_ln_words) != cudaSuccess) return ALBERT_ERR_CUDA;
    *zg = static_cast<bf16 *>(z);
    *stats = static_cast<float2 *>(st);
    *words = static_cast<int *>(w);
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
    // the epilogue reads bias and ln_g as float4
    if ((reinterpret_cast<uintptr_t>(bias) | reinterpret_cast<uintptr_t>(ln_g)) & 15) return ALBERT_ERR_CONFIG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return ALBERT_ERR_CUDA;
    bf16 *zg = nullptr;
    float2 *stats = nullptr;
    int *words = nullptr;
    int rc = lookup_scratch(&zg, &stats, &words);
    if (rc) return rc;
    int sms = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return ALBERT_ERR_CUDA;

    const int N = gemm::LN_N;
    const int rows_cap = (M + gemm::BM - 1) / gemm::BM * gemm::BM;
    // one CTA for a single 128-row block, else the pair: two kernel instances, both
    // loaded by a warm-up call of each kind (the narrow tile is not used here)
    const int variant = rows_cap > gemm::BM ? kGemmPair : kGemmSingle;
    const int grid = gemm_grid(kEpiResStats, rows_cap, N, sms, variant);
    CUtensorMap ta, tb, to, tr;
    if (make_tmap_bf16(&ta, A, M, K, gemm::BM) || make_tmap_bf16(&tb, W, N, K, gemm::B_BOX) ||
        make_tmap_bf16_tile32(&to, zg, rows_cap, N) || make_tmap_bf16_tile32(&tr, R, M, N))
        return ALBERT_ERR_CUDA;

    reset_words_kernel<<<1, 1, 0, s>>>(words, M);
    if (cudaGetLastError() != cudaSuccess) return ALBERT_ERR_CUDA;
    GemmArgs a{};
    a.N = N;
    a.K = K;
    a.rows_cap = rows_cap;
    a.n_rows = words;
    a.bias = bias;
    a.out_g = ln_g;
    a.out_stats = stats;
    a.eps = eps;
    a.status = words + 1;
    if (launch_gemm(kEpiResStats, ta, tb, to, tr, a, grid, sms, s, variant) != cudaSuccess) return ALBERT_ERR_CUDA;
    if (launch_ln_rows(zg, stats, ln_g, ln_b, eps, static_cast<bf16 *>(Y), nullptr, M, rows_cap, words, words + 1, s) !=
        cudaSuccess)
        return ALBERT_ERR_CUDA;
    // The call returns only once its kernels are done with the shared arrays:
    // callers may rely on this to serialize calls with a host-side lock alone.
    int st = 0;
    if (cudaMemcpyAsync(&st, words + 1, sizeof(int), cudaMemcpyDeviceToHost, s) != cudaSuccess) return ALBERT_ERR_CUDA;
    if (cudaStreamSynchronize(s) != cudaSuccess) return ALBERT_ERR_CUDA;
    return st;
}
