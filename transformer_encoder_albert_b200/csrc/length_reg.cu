// length_reg.cu -- length regulation: token durations, frame offsets and the
// frame-level expansion of the encoder's features.
//
// "How Kokoro TTS Works and Where CKE Stands", section "The time axis is where
// a circuit becomes difficult": per token the sigmoid duration channels are
// summed, divided by the speed, rounded and clamped to at least one frame; their
// sum A is the number of aligned frames; token features are repeated by the
// duration vector.  "Qwen3-TTS and Kokoro: Two Routes from Text to Speech",
// section "Path one": durations 2, 1, 3 -> p1 p1 p2 p3 p3 p3.
//
// Three launches on the caller's stream (the second and third chained with
// programmatic dependent launch), bounded by HBM traffic:
//   durations : a warp per token, 32 tokens (warps) per block, so every token's
//               loads and fp64 chain are in flight at once; fp64 sigmoid sum over the
//               channels (the decision is an integer, taken in fp64), rint, floor
//               of 1; then the block's exclusive prefix (local starts) and sum;
//   scan      : one block over the block sums; validates cu_seqlens, checks the
//               capacity, writes the per-sequence frame offsets;
//   expand    : a warp per token; frame start = block start + local start; reads
//               its feature row once (16-byte lanes) and writes it d[t] times
//               into consecutive frame rows.
#include <climits>
#include <cmath>

#include "albert.h"
#include "kernels.h"
#include "sm100_ptx.cuh"

namespace albert {
namespace {

constexpr int LR_THREADS = 256;      // expansion kernel
constexpr int LR_TOK = 32;           // tokens per block of the durations kernel, one warp each
constexpr int LR_DUR_THREADS = 32 * LR_TOK;
constexpr int SCAN_THREADS = 1024;

// Durations of LR_TOK consecutive tokens (warp w takes token w), then their
// exclusive prefix inside the block (local frame start) and the block sum.
__global__ void __launch_bounds__(LR_DUR_THREADS)
lr_durations_kernel(const float *__restrict__ logits, int C, double speed, int n_tok, int *__restrict__ dur,
                    int *__restrict__ local_start, long long *__restrict__ block_sum, int *status) {
    __shared__ int sd[LR_TOK];
    if (blockIdx.x == 0 && threadIdx.x == 0) *status = 0;
    griddep_launch_dependents();  // the scan (launched with PDL) may take SMs as this grid frees them
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int t0 = blockIdx.x * LR_TOK;
    for (int i = warp; i < LR_TOK; i += LR_DUR_THREADS / 32) {
        const int t = t0 + i;
        int d = 0;
        if (t < n_tok) {
            const float *z = logits + (size_t)t * C;
            double s = 0.0;
            for (int c = lane; c < C; c += 32) s += 1.0 / (1.0 + exp(-(double)__ldg(z + c)));
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
            const double q = rint(s / speed);
            // durations beyond INT_MAX / 2 cannot fit any frame buffer: the scan flags them
            d = q < 1.0 ? 1 : (q > (double)(INT_MAX / 2) ? INT_MAX / 2 : (int)q);
            if (lane == 0) dur[t] = d;
        }
        if (lane == 0) sd[i] = d;
    }
    __syncthreads();
    if (warp == 0) {
        const long long v = sd[lane];  // LR_TOK == 32: one token per lane
        long long x = v;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const long long y = __shfl_up_sync(0xffffffffu, x, o);
            if (lane >= o) x += y;
        }
        if (t0 + lane < n_tok) local_start[t0 + lane] = (int)(x - v);
        if (lane == 31) block_sum[blockIdx.x] = x;
    }
}

// Block-wide exclusive scan helper: returns the exclusive prefix of v and the total.
__device__ long long block_exclusive_scan(long long v, long long &total) {
    __shared__ long long warp_sums[SCAN_THREADS / 32];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    long long x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const long long y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) warp_sums[warp] = x;
    __syncthreads();
    if (warp == 0) {
        long long w = lane < SCAN_THREADS / 32 ? warp_sums[lane] : 0;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const long long y = __shfl_up_sync(0xffffffffu, w, o);
            if (lane >= o) w += y;
        }
        if (lane < SCAN_THREADS / 32) warp_sums[lane] = w;
    }
    __syncthreads();
    const long long before = (warp > 0 ? warp_sums[warp - 1] : 0) + x - v;
    total = warp_sums[SCAN_THREADS / 32 - 1];
    __syncthreads();
    return before;
}

// One block: validates cu_seqlens, scans the block sums (frame start of every
// block of LR_TOK tokens), checks the capacity and writes the sequence offsets.
__global__ void __launch_bounds__(SCAN_THREADS)
lr_scan_kernel(const long long *__restrict__ block_sum, int n_blocks, const int *__restrict__ local_start,
               const int *__restrict__ cu, int nseq, int n_tok, int max_frames, long long *__restrict__ block_start,
               int *__restrict__ cu_frames, int *status) {
    griddep_launch_dependents();  // the expansion (launched with PDL) may take SMs as this grid frees them
    griddep_wait();               // durations and block sums are complete
    __shared__ int bad;
    if (threadIdx.x == 0) bad = (cu[0] != 0 || cu[nseq] != n_tok) ? 1 : 0;
    __syncthreads();
    for (int b = threadIdx.x; b < nseq; b += SCAN_THREADS)
        if (cu[b + 1] < cu[b]) bad = 1;
    __syncthreads();
    if (bad) {
        if (threadIdx.x == 0) set_status(status, kStatusSeqlens);
        return;
    }
    const int per = (n_blocks + SCAN_THREADS - 1) / SCAN_THREADS;
    const int b0 = threadIdx.x * per, b1 = min(n_blocks, b0 + per);
    long long local = 0;
    for (int b = b0; b < b1; ++b) local += block_sum[b];
    long long total = 0;
    long long run = block_exclusive_scan(local, total);
    if (total > (long long)max_frames) {
        if (threadIdx.x == 0) set_status(status, kStatusShape);
        return;
    }
    for (int b = b0; b < b1; ++b) {
        block_start[b] = run;
        run += block_sum[b];
    }
    __syncthreads();
    for (int b = threadIdx.x; b <= nseq; b += SCAN_THREADS) {
        const int t = cu[b];
        cu_frames[b] = t < n_tok ? (int)(block_start[t / LR_TOK] + local_start[t]) : (int)total;
    }
}

// One warp per token: frame start = its block's start + its start inside the
// block; the feature row (16-byte lanes) is written d[t] times.
__global__ void __launch_bounds__(LR_THREADS)
lr_expand_kernel(const uint4 *__restrict__ feats, int chunks, const int *__restrict__ dur,
                 const int *__restrict__ local_start, const long long *__restrict__ block_start, int n_tok,
                 int *__restrict__ frame_start, uint4 *__restrict__ frames, const int *status) {
    // last kernel of the operation: no early trigger (whatever follows waits for it)
    griddep_wait();               // frame offsets are complete
    if (*reinterpret_cast<const volatile int *>(status) != 0) return;
    const int lane = threadIdx.x & 31;
    const int warps = gridDim.x * (LR_THREADS / 32);
    for (int t = blockIdx.x * (LR_THREADS / 32) + (threadIdx.x >> 5); t < n_tok; t += warps) {
        const int d = dur[t];
        const int f0 = (int)(block_start[t / LR_TOK] + local_start[t]);
        if (lane == 0) frame_start[t] = f0;
        uint4 *dst = frames + (size_t)f0 * chunks;
        for (int c = lane; c < chunks; c += 32) {
            const uint4 v = __ldg(feats + (size_t)t * chunks + c);
            for (int k = 0; k < d; ++k) dst[(size_t)k * chunks + c] = v;
        }
    }
}

}  // namespace
}  // namespace albert

using namespace albert;

// Scratch: local starts [n_tok] int32, then block sums and block starts
// [n_blocks] int64 each (8-byte aligned).
static size_t lr_scratch_layout(int n_tok, size_t *off_sum, size_t *off_start) {
    const size_t n_blocks = ((size_t)n_tok + LR_TOK - 1) / LR_TOK;
    *off_sum = ((size_t)n_tok * 4 + 7) & ~(size_t)7;
    *off_start = *off_sum + n_blocks * 8;
    return *off_start + n_blocks * 8;
}

extern "C" size_t albert_length_regulate_scratch_bytes(int n_tok) {
    size_t a, b;
    return n_tok < 1 ? 0 : lr_scratch_layout(n_tok, &a, &b);
}

extern "C" int albert_length_regulate(const float *logits, int C, float speed, const void *feats, int D,
                                      const int32_t *cu_seqlens, int nseq, int n_tok, int32_t *durations,
                                      int32_t *frame_start, int32_t *cu_frames, void *frames, int max_frames,
                                      void *scratch, int32_t *status, void *stream) {
    if (!logits || !feats || !cu_seqlens || !durations || !frame_start || !cu_frames || !frames || !scratch ||
        !status)
        return ALBERT_ERR_NULL;
    if (C < 1 || D < 8 || D % 8 || nseq < 1 || n_tok < 1 || max_frames < 0) return ALBERT_ERR_SHAPE;
    if (!(speed > 0.f) || !std::isfinite(speed)) return ALBERT_ERR_CONFIG;
    if (reinterpret_cast<uintptr_t>(feats) % 16 || reinterpret_cast<uintptr_t>(frames) % 16 ||
        reinterpret_cast<uintptr_t>(scratch) % 8)
        return ALBERT_ERR_CONFIG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const int n_blocks = (n_tok + LR_TOK - 1) / LR_TOK;
    size_t off_sum, off_start;
    lr_scratch_layout(n_tok, &off_sum, &off_start);
    int *local_start = static_cast<int *>(scratch);
    long long *block_sum = reinterpret_cast<long long *>(static_cast<char *>(scratch) + off_sum);
    long long *block_start = reinterpret_cast<long long *>(static_cast<char *>(scratch) + off_start);
    lr_durations_kernel<<<n_blocks, LR_DUR_THREADS, 0, s>>>(logits, C, (double)speed, n_tok, durations, local_start,
                                                        block_sum, status);
    cudaError_t e = launch_pdl(lr_scan_kernel, dim3(1), dim3(SCAN_THREADS), 0, s, block_sum, n_blocks, local_start,
                               cu_seqlens, nseq, n_tok, max_frames, block_start, cu_frames, status);
    const int chunks = D * 2 / 16;
    const int warps_needed = n_tok, blocks = (warps_needed + LR_THREADS / 32 - 1) / (LR_THREADS / 32);
    if (e == cudaSuccess)
        e = launch_pdl(lr_expand_kernel, dim3(blocks < 148 * 8 ? blocks : 148 * 8), dim3(LR_THREADS), 0, s,
                       static_cast<const uint4 *>(feats), chunks, durations, local_start, block_start, n_tok,
                       frame_start, static_cast<uint4 *>(frames), status);
    if (e != cudaSuccess) return ALBERT_ERR_CUDA;
    return cudaGetLastError() == cudaSuccess ? ALBERT_OK : ALBERT_ERR_CUDA;
}
