// length_reg.cu -- length regulation: token durations, frame offsets and the
// frame-level expansion of the encoder's features.
//
// "ALBERT: How Kokoro's Phoneme Encoder Works", section "The time axis is where
// a circuit becomes difficult": per token the sigmoid duration channels are
// summed, divided by the speed, rounded and clamped to at least one frame; their
// sum A is the number of aligned frames; token features are repeated by the
// duration vector.  "How Kokoro TTS Works and Where CKE Stands", section "Path
// one": durations 2, 1, 3 -> p1 p1 p2 p3 p3 p3.
//
// Three launches on the caller's stream, all bounded by HBM traffic:
//   durations : one warp per token; fp64 sigmoid sum over the channels (the
//               decision is an integer, taken in fp64), rint, floor of 1;
//   scan      : one block; validates cu_seqlens, exclusive prefix sum of the
//               durations (frame start of every token, sequences back to back),
//               per-sequence frame offsets, capacity check;
//   expand    : one warp per token; reads its feature row once (16-byte lanes)
//               and writes it d[t] times into consecutive frame rows.
#include <climits>
#include <cmath>

#include "albert.h"
#include "kernels.h"
#include "sm100_ptx.cuh"

namespace albert {
namespace {

constexpr int LR_THREADS = 256;
constexpr int SCAN_THREADS = 1024;

__global__ void __launch_bounds__(LR_THREADS)
lr_durations_kernel(const float *__restrict__ logits, int C, double speed, int n_tok, int *__restrict__ dur,
                    int *status) {
    if (blockIdx.x == 0 && threadIdx.x == 0) *status = 0;
    const int lane = threadIdx.x & 31;
    const int t = blockIdx.x * (LR_THREADS / 32) + (threadIdx.x >> 5);
    if (t >= n_tok) return;
    const float *z = logits + (size_t)t * C;
    double s = 0.0;
    for (int c = lane; c < C; c += 32) s += 1.0 / (1.0 + exp(-(double)__ldg(z + c)));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    if (lane == 0) {
        const double q = rint(s / speed);
        // durations beyond INT_MAX / 2 cannot fit any frame buffer: the scan flags them
        dur[t] = q < 1.0 ? 1 : (q > (double)(INT_MAX / 2) ? INT_MAX / 2 : (int)q);
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

__global__ void __launch_bounds__(SCAN_THREADS)
lr_scan_kernel(const int *__restrict__ dur, const int *__restrict__ cu, int nseq, int n_tok, int max_frames,
               int *__restrict__ frame_start, int *__restrict__ cu_frames, int *status) {
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
    // each thread scans a contiguous slice of tokens
    const int per = (n_tok + SCAN_THREADS - 1) / SCAN_THREADS;
    const int t0 = threadIdx.x * per, t1 = min(n_tok, t0 + per);
    long long local = 0;
    for (int t = t0; t < t1; ++t) local += dur[t];
    long long total = 0;
    long long run = block_exclusive_scan(local, total);
    if (total > (long long)max_frames) {
        if (threadIdx.x == 0) set_status(status, kStatusShape);
        return;
    }
    for (int t = t0; t < t1; ++t) {
        frame_start[t] = (int)run;
        run += dur[t];
    }
    __syncthreads();
    for (int b = threadIdx.x; b <= nseq; b += SCAN_THREADS)
        cu_frames[b] = cu[b] < n_tok ? frame_start[cu[b]] : (int)total;
}

__global__ void __launch_bounds__(LR_THREADS)
lr_expand_kernel(const uint4 *__restrict__ feats, int chunks, const int *__restrict__ dur,
                 const int *__restrict__ frame_start, int n_tok, uint4 *__restrict__ frames, const int *status) {
    if (*reinterpret_cast<const volatile int *>(status) != 0) return;
    const int lane = threadIdx.x & 31;
    const int warps = gridDim.x * (LR_THREADS / 32);
    for (int t = blockIdx.x * (LR_THREADS / 32) + (threadIdx.x >> 5); t < n_tok; t += warps) {
        const int d = dur[t];
        uint4 *dst = frames + (size_t)frame_start[t] * chunks;
        for (int c = lane; c < chunks; c += 32) {
            const uint4 v = __ldg(feats + (size_t)t * chunks + c);
            for (int k = 0; k < d; ++k) dst[(size_t)k * chunks + c] = v;
        }
    }
}

}  // namespace
}  // namespace albert

using namespace albert;

extern "C" int albert_length_regulate(const float *logits, int C, float speed, const void *feats, int D,
                                      const int32_t *cu_seqlens, int nseq, int n_tok, int32_t *durations,
                                      int32_t *frame_start, int32_t *cu_frames, void *frames, int max_frames,
                                      int32_t *status, void *stream) {
    if (!logits || !feats || !cu_seqlens || !durations || !frame_start || !cu_frames || !frames || !status)
        return ALBERT_ERR_NULL;
    if (C < 1 || D < 8 || D % 8 || nseq < 1 || n_tok < 1 || max_frames < 0) return ALBERT_ERR_SHAPE;
    if (!(speed > 0.f) || !std::isfinite(speed)) return ALBERT_ERR_CONFIG;
    if (reinterpret_cast<uintptr_t>(feats) % 16 || reinterpret_cast<uintptr_t>(frames) % 16) return ALBERT_ERR_CONFIG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const int blocks = (n_tok + LR_THREADS / 32 - 1) / (LR_THREADS / 32);
    lr_durations_kernel<<<blocks, LR_THREADS, 0, s>>>(logits, C, (double)speed, n_tok, durations, status);
    lr_scan_kernel<<<1, SCAN_THREADS, 0, s>>>(durations, cu_seqlens, nseq, n_tok, max_frames, frame_start, cu_frames,
                                              status);
    const int chunks = D * 2 / 16;
    lr_expand_kernel<<<blocks < 148 * 8 ? blocks : 148 * 8, LR_THREADS, 0, s>>>(
        static_cast<const uint4 *>(feats), chunks, durations, frame_start, n_tok, static_cast<uint4 *>(frames), status);
    return cudaGetLastError() == cudaSuccess ? ALBERT_OK : ALBERT_ERR_CUDA;
}
