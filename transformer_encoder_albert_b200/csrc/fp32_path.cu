// fp32_path.cu -- the all-fp32 variant of the path (SIMT FMA; tcgen05 has no
// fp32 input kind and TF32 would not meet a 1e-4 relative bound).  Used for
// small workloads that need fp32 agreement with the oracle.
//
// Linear layer: y_j = b_j + sum_i x_i W_{j,i}, W stored [out, in] ("Qwen3-TTS
// and Kokoro", section A); epilogues: bias, tanh-GELU (page "ALBERT: How
// Kokoro's Phoneme Encoder Works", step 6), residual add (steps 5-6), row
// scatter.  LayerNorm over 768 columns: textbook (biased variance, eps inside
// the square root), affine gamma/beta.
#include "kernels.h"
#include "sm100_ptx.cuh"

namespace albert {
namespace {

constexpr int TM = 64, TN = 64, TK = 16;

template <int EPI>
__global__ void __launch_bounds__(256)
gemm_f32_kernel(const GemmF32Args a) {
    if (*reinterpret_cast<const volatile int *>(a.status) != 0) return;
    const int n_rows = *a.n_rows;
    const int m0 = blockIdx.y * TM, n0 = blockIdx.x * TN;
    if (m0 >= n_rows) return;
    __shared__ float As[TK][TM + 4];
    __shared__ float Ws[TK][TN + 4];
    const int tid = threadIdx.x;
    const int ty = tid >> 4, tx = tid & 15;
    float acc[4][4] = {};
    const int lr = tid >> 2, lk = (tid & 3) * 4;  // loader: row, k offset (float4)
    for (int k0 = 0; k0 < a.K; k0 += TK) {
        const int ar = m0 + lr;
        float4 av = make_float4(0.f, 0.f, 0.f, 0.f);
        if (ar < n_rows) av = *reinterpret_cast<const float4 *>(a.A + (size_t)ar * a.K + k0 + lk);
        As[lk + 0][lr] = av.x; As[lk + 1][lr] = av.y; As[lk + 2][lr] = av.z; As[lk + 3][lr] = av.w;
        const float4 wv = *reinterpret_cast<const float4 *>(a.W + (size_t)(n0 + lr) * a.K + k0 + lk);
        Ws[lk + 0][lr] = wv.x; Ws[lk + 1][lr] = wv.y; Ws[lk + 2][lr] = wv.z; Ws[lk + 3][lr] = wv.w;
        __syncthreads();
#pragma unroll
        for (int k = 0; k < TK; ++k) {
            float x[4], w[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) { x[i] = As[k][ty * 4 + i]; w[i] = Ws[k][tx * 4 + i]; }
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(x[i], w[j], acc[i][j]);
        }
        __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int r = m0 + ty * 4 + i;
        if (r >= n_rows) continue;
        int dst = r;
        if (EPI == kF32Scatter) {
            dst = __ldg(a.row_dst + r);
            if (dst < 0) continue;
        }
        float v[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int c = n0 + tx * 4 + j;
            v[j] = acc[i][j] + __ldg(a.bias + c);
            if (EPI == kF32Gelu) v[j] = 0.5f * v[j] * (1.0f + tanhf(0.7978845608028654f * (v[j] + 0.044715f * v[j] * v[j] * v[j])));
            if (EPI == kF32Resid) v[j] += a.resid[(size_t)r * a.N + c];
        }
        *reinterpret_cast<float4 *>(a.out + (size_t)dst * a.ld_out + n0 + tx * 4) = make_float4(v[0], v[1], v[2], v[3]);
    }
}

// One warp per row of 768: two-pass mean / variance in registers.
__global__ void __launch_bounds__(256)
layer_norm_f32_kernel(const float *__restrict__ x, float *__restrict__ y, const float *__restrict__ g,
                      const float *__restrict__ b, float eps, const int *n_rows, const int *status) {
    if (*reinterpret_cast<const volatile int *>(status) != 0) return;
    const int r = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
    if (r >= *n_rows) return;
    constexpr int PER = kHidden / 32;  // 24
    float v[PER];
    const float *xr = x + (size_t)r * kHidden;
    float s = 0.f;
#pragma unroll
    for (int i = 0; i < PER; ++i) { v[i] = xr[lane + 32 * i]; s += v[i]; }
    for (int o = 16; o; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    const float mu = s / kHidden;
    float q = 0.f;
#pragma unroll
    for (int i = 0; i < PER; ++i) { const float d = v[i] - mu; q = fmaf(d, d, q); }
    for (int o = 16; o; o >>= 1) q += __shfl_xor_sync(0xffffffffu, q, o);
    const float inv = 1.0f / sqrtf(q / kHidden + eps);
    float *yr = y + (size_t)r * kHidden;
#pragma unroll
    for (int i = 0; i < PER; ++i) {
        const int c = lane + 32 * i;
        yr[c] = (v[i] - mu) * inv * g[c] + b[c];
    }
}

}  // namespace

cudaError_t launch_gemm_f32(int epi, const GemmF32Args &a, cudaStream_t s) {
    dim3 grid(a.N / TN, (a.rows_cap + TM - 1) / TM);
    switch (epi) {
        case kF32Bias: gemm_f32_kernel<kF32Bias><<<grid, 256, 0, s>>>(a); break;
        case kF32Gelu: gemm_f32_kernel<kF32Gelu><<<grid, 256, 0, s>>>(a); break;
        case kF32Resid: gemm_f32_kernel<kF32Resid><<<grid, 256, 0, s>>>(a); break;
        case kF32Scatter: gemm_f32_kernel<kF32Scatter><<<grid, 256, 0, s>>>(a); break;
        default: return cudaErrorInvalidValue;
    }
    return cudaGetLastError();
}

cudaError_t launch_layer_norm_f32(const float *x, float *y, const float *g, const float *b,
                                  float eps, int rows_cap, const int *n_rows, const int *status,
                                  cudaStream_t s) {
    layer_norm_f32_kernel<<<(rows_cap + 7) / 8, 256, 0, s>>>(x, y, g, b, eps, n_rows, status);
    return cudaGetLastError();
}

}  // namespace albert
