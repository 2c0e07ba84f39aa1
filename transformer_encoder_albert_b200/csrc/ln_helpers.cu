// ln_helpers.cu -- small kernels around the deferred LayerNorm.
//
// The post-LN LayerNorms of the shared layer ("ALBERT: How Kokoro's Phoneme
// Encoder Works", section "Inside One Real ALBERT Layer", steps 5 and 6:
// LN(x) = (x - mean) / sqrt(var + eps) * gamma + beta over the 768 features)
// are applied by the GEMMs that consume their output.  These kernels prepare
// the folded constants of those GEMMs once per weight set, and normalize rows
// where a LayerNorm output leaves the library (hidden-state outputs and the
// single-kernel entry points).
#include "kernels.h"
#include "sm100_ptx.cuh"

namespace albert {
namespace {

// One warp per output feature j of W [N, K]: s_j = sum_k gamma_k W_jk,
// c_j = sum_k beta_k W_jk + b_j, fp32, fixed order (lane-strided, then a
// butterfly reduction).
__global__ void fold_ln_kernel(const bf16 *__restrict__ W, int N, int K, const float *__restrict__ gamma,
                               const float *__restrict__ beta, const float *__restrict__ b, float *s_out,
                               float *c_out) {
    const int j = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
    if (j >= N) return;
    const bf16 *w = W + (size_t)j * K;
    float s = 0.f, c = 0.f;
    for (int k = lane; k < K; k += 32) {
        const float x = __bfloat162float(w[k]);
        s = fmaf(gamma[k], x, s);
        c = fmaf(beta[k], x, c);
    }
    for (int o = 16; o; o >>= 1) {
        s += __shfl_xor_sync(0xffffffffu, s, o);
        c += __shfl_xor_sync(0xffffffffu, c, o);
    }
    if (lane == 0) {
        s_out[j] = s;
        c_out[j] = c + (b ? b[j] : 0.f);
    }
}

// One warp per row: merge the six partial (mean, M2) pairs, then
// out = rstd * zg - rstd * mu * gamma + beta over 768 columns (bf16).
__global__ void __launch_bounds__(256)
ln_rows_kernel(const bf16 *__restrict__ zg, const float2 *__restrict__ stats, const float *__restrict__ gamma,
               const float *__restrict__ beta, float eps, bf16 *__restrict__ out, const int *__restrict__ row_dst,
               int out_rows, const int *n_rows, int *status) {
    // last kernel of a forward: no early trigger, so that whatever follows in the
    // stream waits for its completion (and, through the chain, the whole forward's)
    griddep_wait();               // the previous kernel has completed

    if (*reinterpret_cast<const volatile int *>(status) != 0) return;
    const int r = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
    if (r >= *n_rows) return;
    const int dst = row_dst ? row_dst[r] : r;
    if (dst < 0) return;
    if (dst >= out_rows) {  // never expected: record it instead of writing out of bounds
        set_status(status, kStatusShape);
        return;
    }
    constexpr int P = gemm::LN_PARTS;
    float2 q[P];
#pragma unroll
    for (int i = 0; i < P; ++i) q[i] = stats[(size_t)r * P + i];
    float m = 0.f;
#pragma unroll
    for (int i = 0; i < P; ++i) m += q[i].x;
    m *= 1.0f / P;
    float m2 = 0.f;
#pragma unroll
    for (int i = 0; i < P; ++i) {
        const float d = q[i].x - m;
        m2 += q[i].y + (float)(kHidden / P) * d * d;
    }
    const float rstd = rsqrtf(m2 * (1.0f / kHidden) + eps), nmu = -rstd * m;
    const uint4 *src = reinterpret_cast<const uint4 *>(zg + (size_t)r * kHidden);
    uint4 *o = reinterpret_cast<uint4 *>(out + (size_t)dst * kHidden);
    for (int c = lane; c < kHidden / 8; c += 32) {
        const uint4 w = src[c];
        const uint32_t in[4] = {w.x, w.y, w.z, w.w};
        uint32_t res[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int col = c * 8 + 2 * e;
            const float2 f = unpack_bf16x2(in[e]);
            const float y0 = fmaf(rstd, f.x, fmaf(nmu, gamma[col], beta[col]));
            const float y1 = fmaf(rstd, f.y, fmaf(nmu, gamma[col + 1], beta[col + 1]));
            res[e] = pack_bf16x2(y0, y1);
        }
        o[c] = make_uint4(res[0], res[1], res[2], res[3]);
    }
}

__global__ void vec_add_kernel(const float *a, const float *b, float *out, int n) {
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i < n) out[i] = a[i] + b[i];
}

}  // namespace

cudaError_t launch_fold_ln(const bf16 *W, int N, int K, const float *gamma, const float *beta, const float *b,
                           float *s_out, float *c_out, cudaStream_t s) {
    fold_ln_kernel<<<(N + 7) / 8, 256, 0, s>>>(W, N, K, gamma, beta, b, s_out, c_out);
    return cudaGetLastError();
}

cudaError_t launch_ln_rows(const bf16 *zg, const float2 *stats, const float *gamma, const float *beta, float eps,
                           bf16 *out, const int *row_dst, int out_rows, int rows_cap, const int *n_rows, int *status,
                           cudaStream_t s) {
    return launch_pdl(ln_rows_kernel, dim3((rows_cap + 7) / 8), dim3(256), 0, s, zg, stats, gamma, beta, eps, out,
                      row_dst, out_rows, n_rows, status);
}

cudaError_t launch_vec_add(const float *a, const float *b, float *out, int n, cudaStream_t s) {
    vec_add_kernel<<<(n + 255) / 256, 256, 0, s>>>(a, b, out, n);
    return cudaGetLastError();
}

}  // namespace albert
