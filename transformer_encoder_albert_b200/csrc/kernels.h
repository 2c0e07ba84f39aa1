// kernels.h -- launchers of the library's kernels (internal to the .so).
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cstdint>

namespace albert {

using bf16 = __nv_bfloat16;

// Fixed architecture of the kernels.
constexpr int kEmb = 128, kHidden = 768, kHeads = 12, kHeadDim = 64, kFfn = 2048;
constexpr int kQKV = 3 * kHidden;
constexpr int kMaxPos = 512;

// ------------------------------------------------------------- tcgen05 GEMM --
enum GemmEpi : int { kEpiBias = 0, kEpiGelu = 1, kEpiLN = 2, kEpiScatter = 3 };

namespace gemm {
constexpr int BM = 128, BN = 256, BK = 64, STAGES = 4;
constexpr int A_BYTES = BM * BK * 2;
constexpr int B_BYTES = BN * BK * 2;
constexpr int EPI_WARPS = 8;
constexpr int THREADS = 32 * (2 + EPI_WARPS);
constexpr int TMEM_COLS = 512;
constexpr int LN_N = 768;  // the LayerNorm epilogue normalizes rows of this width
constexpr int STG_BYTES = 32 * 32 * 2;  // one 32x32 bf16 epilogue staging tile per epilogue warp
constexpr int SMEM_BYTES = 2048 + STAGES * (A_BYTES + B_BYTES) + EPI_WARPS * STG_BYTES + 1024 + 2 * 2 * BM * 8;
}  // namespace gemm

struct GemmArgs {
    int N, K;
    int rows_cap;              // rows of the A / out buffers (multiple of 128)
    const int *n_rows;         // device: rows that hold data (<= rows_cap)
    const float *bias;         // [N]
    const bf16 *resid;         // LN: [rows, N]
    int ld_resid;
    const float *ln_g, *ln_b;  // LN: [N]
    float eps;
    bf16 *out;                 // [rows, ld_out] (scatter: destination rows)
    int ld_out;
    float2 *ln_stats;          // LN: per-row (mean, M2) of each 256-column tile, [rows_cap][N/256]
    int *ln_flags;             // LN: per (row block, lane quadrant, column tile) epoch flags
    int epoch;                 // LN: value this launch writes to ln_flags (> every earlier one)
    const int *row_dst;        // scatter: destination row or -1
    int *status;               // device status word
};

// Encode a 2-D bf16 row-major [rows, cols] tensor map with a {64, box_rows}
// box and the 128-byte swizzle.  Returns 0 on success.
int make_tmap_bf16(CUtensorMap *tm, const void *base, uint64_t rows, uint64_t cols,
                   uint32_t box_rows);
// Map of a bf16 row-major [rows, cols] tensor with a 32x32 box and the 64-byte
// swizzle: the epilogue's output stores and residual loads.
int make_tmap_bf16_tile32(CUtensorMap *tm, const void *base, uint64_t rows, uint64_t cols);

// Grid the GEMM uses for this many rows (persistent: <= number of SMs).
int gemm_grid(int epi, int rows_cap, int N, int num_sms);
// Cross-tile LayerNorm buffers for rows_cap rows of width LN_N.
inline size_t gemm_ln_stats_count(int rows_cap) { return (size_t)rows_cap * (gemm::LN_N / gemm::BN); }
inline size_t gemm_ln_flags_count(int rows_cap) {
    return (size_t)((rows_cap + gemm::BM - 1) / gemm::BM) * 4 * (gemm::LN_N / gemm::BN);
}

// tmOut: tile32 map of the output (unused by the scatter epilogue); tmRes: tile32
// map of the residual (LayerNorm epilogue only; pass any valid map otherwise).
cudaError_t launch_gemm(int epi, const CUtensorMap &tmA, const CUtensorMap &tmB, const CUtensorMap &tmOut,
                        const CUtensorMap &tmRes, const GemmArgs &args, int grid, cudaStream_t s);

// ---------------------------------------------------------------- attention --
// Masked bidirectional attention, bf16 tensor-core kernel (mma.sync m16n8k16).
cudaError_t launch_attention_bf16(const bf16 *qkv, bf16 *ctx, const int *seq_start,
                                  const int *seq_len, int nseq, int max_len,
                                  const int *status, cudaStream_t s);
cudaError_t launch_attention_f32(const float *qkv, float *ctx, const int *seq_start,
                                 const int *seq_len, int nseq, int max_len,
                                 const int *status, cudaStream_t s);

// ---------------------------------------------------- prep / embed / output --
// max_rows: the handle's max_tokens; a larger total sets ALBERT_ERR_SHAPE.
cudaError_t launch_prep_padded(const uint8_t *mask, int B, int T, int pack, int max_rows,
                               int *seq_start, int *seq_len, int *n_rows, int *status,
                               cudaStream_t s);
cudaError_t launch_prep_varlen(const int32_t *cu, int nseq, int max_len, int max_rows,
                               int *seq_start, int *seq_len, int *n_rows, int *status,
                               cudaStream_t s);

struct EmbedArgs {
    const int64_t *ids;
    int ids_padded;     // 1: ids[b*T + t]; 0: ids[row]
    int T;
    const int *seq_start, *seq_len;
    int nseq;
    const int *n_rows;
    int rows_cap;
    const float *word, *pos, *type, *g, *b;
    float eps;
    int vocab;
    void *E;            // bf16 or fp32 [rows, 128]
    int out_f32;
    int *row_dst;       // destination row in `out` (b*T + t or the row itself) or -1
    int dst_padded;
    int *status;
};
cudaError_t launch_embed(const EmbedArgs &a, cudaStream_t s);

// out[(b*T + t)] = 0 for padding slots t >= seq_len[b]; D columns of elem_bytes.
cudaError_t launch_zero_pad(void *out, int B, int T, int D, int elem_bytes, const int *seq_len,
                            const int *status, cudaStream_t s);
// out[row_dst[r]] = X[r] for r < n_rows with row_dst[r] >= 0.
cudaError_t launch_scatter_rows(const void *X, void *out, int D, int elem_bytes, int rows_cap,
                                const int *n_rows, const int *row_dst, const int *status,
                                cudaStream_t s);

// fp32 -> bf16 conversion of a parameter block.
cudaError_t launch_f32_to_bf16(const float *src, bf16 *dst, size_t n, cudaStream_t s);

// ---------------------------------------------------------------- fp32 path --
enum F32Epi : int { kF32Bias = 0, kF32Gelu = 1, kF32Resid = 2, kF32Scatter = 3 };
struct GemmF32Args {
    const float *A;     // [rows, K]
    const float *W;     // [N, K]
    const float *bias;  // [N]
    const float *resid; // [rows, N]
    float *out;         // [rows, ld_out]
    int ld_out;
    int N, K, rows_cap;
    const int *n_rows;
    const int *row_dst;
    const int *status;
};
cudaError_t launch_gemm_f32(int epi, const GemmF32Args &a, cudaStream_t s);
cudaError_t launch_layer_norm_f32(const float *x, float *y, const float *g, const float *b,
                                  float eps, int rows_cap, const int *n_rows, const int *status,
                                  cudaStream_t s);

}  // namespace albert
