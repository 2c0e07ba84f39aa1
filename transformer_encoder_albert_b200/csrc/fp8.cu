// fp8.cu -- the FP8 (E4M3) variant's quantization and folded LayerNorm constants.
//
// The pages evaluate a quantized build of the encoder against its FP32 outputs
// ("Kokoro-82M-encoder-hailo10h" model card, section "Eval results": per-sample
// cosine and MSE on random post-embedding-LayerNorm inputs).  Here both
// operands of the layer GEMMs are E4M3 with one fp32 scale per row along the
// reduction dimension (per token for activations, per output channel for
// weights), so the tcgen05 product (kind::f8f6f4) sums q_x q_w exactly in fp32
// and the epilogue multiplies by s_x s_w:
//   amax = max |x|,  s = amax / 448,  q = E4M3(fp32(x * (448 / amax)))
// (one rounding of the fp32 product to E4M3, to nearest even, saturating; a
// row of zeros has s = 0 and q = 0).
// A row's scale needs the whole row, which the GEMM epilogues that produce the
// activations do not have (their tiles are 256 columns wide), so activations
// are quantized by a separate pass per GEMM: one warp per row at a time.
#include "kernels.h"
#include "sm100_ptx.cuh"

namespace albert {
namespace {

constexpr int Q_WARPS = 8;

// Two fp32 -> two E4M3 bytes (lo at the lower address): one rounding to nearest,
// ties to even, saturating at +-448, the sign kept (also on zero).  The
// conversion instruction's results were checked bit for bit against this
// definition on the GPU, every E4M3 midpoint included.
__device__ __forceinline__ uint16_t cvt_e4m3x2(float lo, float hi) {
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
    return r;
}

// x [rows, K] bf16 -> q [rows, K] E4M3, scale [rows] fp32, K = 256 * RUNS: each
// lane holds RUNS runs of 8 consecutive values of a row.  A warp walks rows
// with a grid stride and loads its next row while it converts the current
// one, so that two rows per warp are in flight (one row per warp left the
// loads of a wave to finish before the next wave started).
template <int RUNS>
__device__ __forceinline__ void quant_load(const bf16 *__restrict__ x, int row, int lane, uint4 (&v)[RUNS]) {
    const uint4 *src = reinterpret_cast<const uint4 *>(x + (size_t)row * (RUNS * 256));
#pragma unroll
    for (int i = 0; i < RUNS; ++i) v[i] = src[i * 32 + lane];
}

template <int RUNS>
__device__ __forceinline__ void quant_store(const uint4 (&v)[RUNS], int row, int lane, uint8_t *__restrict__ q,
                                            float *__restrict__ scale) {
    float amax = 0.f;
#pragma unroll
    for (int i = 0; i < RUNS; ++i) {
        const uint32_t w[4] = {v[i].x, v[i].y, v[i].z, v[i].w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const float2 f = unpack_bf16x2(w[e]);
            amax = fmaxf(amax, fmaxf(fabsf(f.x), fabsf(f.y)));
        }
    }
    // non-negative floats order like their bit patterns
    amax = __uint_as_float(__reduce_max_sync(0xffffffffu, __float_as_uint(amax)));
    const bool nz = amax > 0.f;
    const float inv = nz ? __fdiv_rn(448.0f, amax) : 0.f;
    if (lane == 0) scale[row] = nz ? __fdiv_rn(amax, 448.0f) : 0.f;
    uint2 *dst = reinterpret_cast<uint2 *>(q + (size_t)row * (RUNS * 256));
#pragma unroll
    for (int i = 0; i < RUNS; ++i) {
        const uint32_t w[4] = {v[i].x, v[i].y, v[i].z, v[i].w};
        uint16_t b[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const float2 f = unpack_bf16x2(w[e]);
            b[e] = cvt_e4m3x2(__fmul_rn(f.x, inv), __fmul_rn(f.y, inv));
        }
        dst[i * 32 + lane] = make_uint2((uint32_t)b[0] | ((uint32_t)b[1] << 16), (uint32_t)b[2] | ((uint32_t)b[3] << 16));
    }
}

template <int RUNS>
__global__ void __launch_bounds__(32 * Q_WARPS)
quant_rows_e4m3_kernel(const bf16 *__restrict__ x, int rows, const int *n_rows, uint8_t *__restrict__ q,
                       float *__restrict__ scale, const int *status, int trigger) {
    if (trigger) griddep_launch_dependents();
    griddep_wait();
    if (status && *reinterpret_cast<const volatile int *>(status) != 0) return;
    const int lane = threadIdx.x & 31;
    int nr = n_rows ? *reinterpret_cast<const volatile int *>(n_rows) : rows;
    nr = nr < rows ? nr : rows;
    const int stride = gridDim.x * Q_WARPS;
    int row = blockIdx.x * Q_WARPS + (threadIdx.x >> 5);
    uint4 a[RUNS], b[RUNS];
    if (row < nr) quant_load<RUNS>(x, row, lane, a);
    // two rows per iteration, alternating the register sets
    while (row < nr) {
        const int r1 = row + stride;
        if (r1 < nr) quant_load<RUNS>(x, r1, lane, b);
        quant_store<RUNS>(a, row, lane, q, scale);
        if (r1 >= nr) break;
        const int r2 = r1 + stride;
        if (r2 < nr) quant_load<RUNS>(x, r2, lane, a);
        quant_store<RUNS>(b, r1, lane, q, scale);
        row = r2;
    }
}

__device__ __forceinline__ float e4m3_to_f32(uint8_t b) {
    // sign, 4 exponent bits (bias 7), 3 mantissa bits; no infinities; 0x7f / 0xff are NaN
    const float sgn = (b & 0x80) ? -1.f : 1.f;
    const int e = (b >> 3) & 15, m = b & 7;
    if ((b & 0x7f) == 0x7f) return __int_as_float(0x7fc00000);
    const float mag = e == 0 ? ldexpf((float)m, -9) : ldexpf((float)(8 + m), e - 10);
    return sgn * mag;
}

// Folded LayerNorm constants of an E4M3 weight W_q [N, K] with row scales sw:
// s_j = sw_j sum_k gamma_k q_jk,  c_j = sw_j sum_k beta_k q_jk + b_j (one warp per j).
__global__ void fold_ln_e4m3_kernel(const uint8_t *__restrict__ Wq, const float *__restrict__ sw, int N, int K,
                                    const float *__restrict__ gamma, const float *__restrict__ beta,
                                    const float *__restrict__ b, float *s_out, float *c_out) {
    const int j = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
    if (j >= N) return;
    const uint8_t *w = Wq + (size_t)j * K;
    float s = 0.f, c = 0.f;
    for (int k = lane; k < K; k += 32) {
        const float x = e4m3_to_f32(w[k]);
        s = fmaf(gamma[k], x, s);
        c = fmaf(beta[k], x, c);
    }
    for (int o = 16; o; o >>= 1) {
        s += __shfl_xor_sync(0xffffffffu, s, o);
        c += __shfl_xor_sync(0xffffffffu, c, o);
    }
    if (lane == 0) {
        s_out[j] = s * sw[j];
        c_out[j] = c * sw[j] + (b ? b[j] : 0.f);
    }
}

}  // namespace

template <int RUNS>
cudaError_t launch_quant_runs(const bf16 *x, int rows, const int *n_rows, uint8_t *q, float *scale, const int *status,
                              cudaStream_t s, bool pdl, bool trigger) {
    int dev = 0, sms = 0, per_sm = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e == cudaSuccess)
        e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, quant_rows_e4m3_kernel<RUNS>, 32 * Q_WARPS, 0);
    if (e != cudaSuccess) return e;
    // a grid that is resident at once, rows by grid stride
    const int need = (rows + Q_WARPS - 1) / Q_WARPS;
    const int cap = (per_sm > 0 ? per_sm : 1) * sms;
    const int blocks = need < cap ? need : cap;
    if (blocks < 1) return cudaSuccess;
    if (!pdl) {
        quant_rows_e4m3_kernel<RUNS><<<blocks, 32 * Q_WARPS, 0, s>>>(x, rows, n_rows, q, scale, status, trigger ? 1 : 0);
        return cudaGetLastError();
    }
    return launch_pdl(quant_rows_e4m3_kernel<RUNS>, dim3(blocks), dim3(32 * Q_WARPS), 0, s, x, rows, n_rows, q, scale,
                      status, trigger ? 1 : 0);
}

cudaError_t launch_quant_rows_e4m3(const bf16 *x, int K, int rows, const int *n_rows, uint8_t *q, float *scale,
                                   const int *status, cudaStream_t s, bool pdl, bool trigger) {
    switch (K) {
        case 256: return launch_quant_runs<1>(x, rows, n_rows, q, scale, status, s, pdl, trigger);
        case 512: return launch_quant_runs<2>(x, rows, n_rows, q, scale, status, s, pdl, trigger);
        case 768: return launch_quant_runs<3>(x, rows, n_rows, q, scale, status, s, pdl, trigger);
        case 1024: return launch_quant_runs<4>(x, rows, n_rows, q, scale, status, s, pdl, trigger);
        case 1280: return launch_quant_runs<5>(x, rows, n_rows, q, scale, status, s, pdl, trigger);
        case 1536: return launch_quant_runs<6>(x, rows, n_rows, q, scale, status, s, pdl, trigger);
        case 1792: return launch_quant_runs<7>(x, rows, n_rows, q, scale, status, s, pdl, trigger);
        case 2048: return launch_quant_runs<8>(x, rows, n_rows, q, scale, status, s, pdl, trigger);
    }
    return cudaErrorInvalidValue;
}

cudaError_t launch_fold_ln_e4m3(const uint8_t *Wq, const float *sw, int N, int K, const float *gamma,
                                const float *beta, const float *b, float *s_out, float *c_out, cudaStream_t s) {
    fold_ln_e4m3_kernel<<<(N + 7) / 8, 256, 0, s>>>(Wq, sw, N, K, gamma, beta, b, s_out, c_out);
    return cudaGetLastError();
}

}  // namespace albert
