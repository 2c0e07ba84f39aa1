// kernels.h -- launchers of the library's kernels (internal to the .so).
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <atomic>
#include <cstdint>

namespace albert {

using bf16 = __nv_bfloat16;

// Raise a kernel's dynamic shared-memory limit on the current device, once per
// device: the attribute belongs to the kernel as loaded on one device, so a
// process that drives several devices sets it on each.  `done` holds one bit
// per device ordinal (0..63; above that the attribute is set on every call).
// Two threads making their first call together may both set it, which is
// harmless; the bit is published only after the attribute is in place.
inline cudaError_t ensure_smem_attr(const void *func, int bytes, std::atomic<unsigned long long> &done) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const unsigned long long bit = (dev >= 0 && dev < 64) ? (1ull << dev) : 0ull;
    if (bit && (done.load(std::memory_order_acquire) & bit)) return cudaSuccess;
    e = cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e == cudaSuccess && bit) done.fetch_or(bit, std::memory_order_acq_rel);
    return e;
}

// Launch with programmatic stream serialization: the kernel may begin while
// the previous kernel in the stream runs; it must call griddep_wait() before
// using that kernel's results (every kernel launched this way does).  Used only
// where the previous operation in the stream is one of this library's kernels:
// a kernel that follows a copy or an event is launched plainly.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                              Args... args) {
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

// Fixed architecture of the kernels.
constexpr int kEmb = 128, kHidden = 768, kHeads = 12, kHeadDim = 64, kFfn = 2048;
constexpr int kQKV = 3 * kHidden;
constexpr int kMaxPos = 512;

// ------------------------------------------------------------- tcgen05 GEMM --
// Epilogues.  "LN input" operands hold z * gamma of a row z that a LayerNorm
// (width 768) still has to normalize; its per-row statistics come as six
// partial (mean, M2) pairs over 128-column slices, [rows][6] float2.  Since
// LN(z) W^T = rstd * (z*gamma) W^T - rstd * mu * (W gamma) + W beta, a GEMM on
// z*gamma applies the LayerNorm in its epilogue with fold_s = W gamma and
// bias = W beta + b.
enum GemmEpi : int {
    kEpiBias = 0,         // Y = acc + bias
    kEpiGelu = 1,         // Y = GELU_tanh(acc + bias)
    kEpiResStats = 2,     // z = acc + bias + residual; Y = z * out_g; out_stats = partial stats of z
    kEpiScatter = 3,      // Y[row_dst[r]] = acc + bias (row_dst[r] < 0: skipped)
    kEpiLnIn = 4,         // Y = rstd * acc - rstd * mu * fold_s + bias
    kEpiLnInGelu = 5,     // Y = GELU_tanh(rstd * acc - rstd * mu * fold_s + bias)
    kEpiLnInScatter = 6,  // Y[row_dst[r]] = rstd * acc - rstd * mu * fold_s + bias
};

namespace gemm {
constexpr int BM = 128, BN = 256, BK = 64;
// The ring uses STAGES - 1 (PAIR_STAGES - 1) stages: one stage's worth of shared
// memory goes to the epilogue's staging tiles.
constexpr int STAGES = 4;       // one CTA per tile: {A 128x64, B 256x64} per stage
constexpr int PAIR_STAGES = 6;  // CTA pair per 256x256 tile: {A 128x64, B 128x64} per CTA and stage
constexpr int B_BOX = 128;      // rows of B per TMA box (weight tensor maps)
constexpr int A_BYTES = BM * BK * 2;
constexpr int B_BYTES = BN * BK * 2;
constexpr int B_HALF_BYTES = B_BOX * BK * 2;
constexpr int EPI_WARPS = 8;
constexpr int THREADS = 32 * (2 + EPI_WARPS);
constexpr int TMEM_COLS = 512;
constexpr int LN_N = 768;     // LayerNorm row width
constexpr int LN_PARTS = 6;   // partial statistics per row (128 columns each)
constexpr int STG_BYTES = 32 * 32 * 2;  // one 32x32 bf16 staging tile

}  // namespace gemm

struct GemmArgs {
    int N, K;
    int rows_cap;              // rows of the A / out buffers (multiple of 128)
    const int *n_rows;         // device: rows that hold data (<= rows_cap)
    const float *bias;         // [N]
    // kEpiLnIn*: statistics of the LayerNorm input held (times gamma) in A
    const float2 *in_stats;    // [rows][6]
    const float *fold_s;       // [N] = W gamma
    // kEpiResStats: residual tile (tmRes) is plain (res_stats == nullptr) or a
    // LayerNorm input z*gamma with statistics res_stats, rebuilt as
    // rstd * r - rstd * mu * res_g + (its beta, folded into bias)
    const float2 *res_stats;   // [rows][6] or nullptr
    const float *res_g;        // [N]
    const float *out_g;        // [N]: Y = z * out_g
    float2 *out_stats;         // [rows][6]: partial (mean, M2) of z per 128 columns
    float eps;
    bf16 *out;                 // scatter epilogues: [*, ld_out] destination rows
    int ld_out;
    const int *row_dst;        // scatter: destination row or -1
    int *status;               // device status word
    int trigger;               // the next kernel in the stream is one of ours, launched with PDL:
                               // let it start early (0 for a last kernel, or before a copy)
    unsigned long long wait_ns;  // limit of the bounded waits (0 = kWaitLimitNs, 2 s)
    int withhold_loads;        // fault injection for tests: the TMA producer issues no loads, so
                               // the MMA issuer's first wait cannot complete and runs out
    // E4M3 operands (A and W as row-scaled E4M3 codes, maps from make_tmap_e4m3; K a
    // multiple of 128): the epilogue starts from acc * a_scale[row] * w_scale[col]
    int e4m3;
    const float *a_scale;      // [rows_cap]
    const float *w_scale;      // [N]
};

// Encode a 2-D bf16 row-major [rows, cols] tensor map with a {64, box_rows}
// box and the 128-byte swizzle (box_rows = BM for A operands, B_BOX for
// weights).  Returns 0 on success.
int make_tmap_bf16(CUtensorMap *tm, const void *base, uint64_t rows, uint64_t cols,
                   uint32_t box_rows);
// Map of an E4M3 (byte) row-major [rows, cols] tensor with a {128, box_rows} box
// and the 128-byte swizzle: the operands of the E4M3 GEMM variant.
int make_tmap_e4m3(CUtensorMap *tm, const void *base, uint64_t rows, uint64_t cols, uint32_t box_rows);
// Map of a bf16 row-major [rows, cols] tensor with a 32x32 box and the 64-byte
// swizzle: the epilogue's output stores and residual loads.
int make_tmap_bf16_tile32(CUtensorMap *tm, const void *base, uint64_t rows, uint64_t cols);

// Kernel variant: one CTA per 128x256 tile, a CTA pair (cluster of 2,
// tcgen05.mma cta_group::2) per 256x256 tile, or one CTA per 128x128 tile.
// Auto (gemm_resolve): the single CTA for one 128-row block; the narrow tile
// when pairs would leave clusters idle and every narrow tile runs at once;
// else the pair.
enum GemmVariant { kGemmAuto = 0, kGemmSingle = 1, kGemmPair = 2, kGemmNarrow = 3 };
int gemm_resolve(int rows_cap, int N, int num_sms, int variant);

// Grid (CTAs) the GEMM uses for this many rows: persistent, at most one CTA per
// SM, and for the pair variant an even count within the co-resident clusters.
int gemm_grid(int epi, int rows_cap, int N, int num_sms, int variant = kGemmAuto);

// The epilogue reads its per-column vectors as float4: each must be 16-byte aligned.
inline bool gemm_vectors_aligned(const GemmArgs &a) {
    auto ok = [](const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; };
    return ok(a.bias) && ok(a.fold_s) && ok(a.res_g) && ok(a.out_g) && ok(a.w_scale);
}

// tmOut: tile32 map of the output (unused by the scatter epilogues); tmRes: tile32
// map of the residual (kEpiResStats only; pass any valid map otherwise).
// grid: from gemm_grid with the same rows_cap, N, num_sms and variant.
cudaError_t launch_gemm(int epi, const CUtensorMap &tmA, const CUtensorMap &tmB, const CUtensorMap &tmOut,
                        const CUtensorMap &tmRes, const GemmArgs &args, int grid, int num_sms, cudaStream_t s,
                        int variant = kGemmAuto, bool pdl = true);

// ------------------------------------------------- small-batch whole forward --
// The whole forward for at most 128 token rows in one cooperative persistent
// kernel (forward_small.cu).  A-operand maps have {64, 64} boxes with the
// 128-byte swizzle over the workspace rows; weight maps {64, 64} boxes.
// Statistics are twelve 64-column (mean, M2) partials per row.
constexpr int kSmallParts = 24;  // 32-column statistics slices of a small-batch row
constexpr int kSmallMaxRows = 128;
struct SmallFwdArgs {
    CUtensorMap tmE, tmX, tmC, tmX1, tmZ, tmH;  // E [rows,128]; X, C, X1 = z1*g1, Z = z2*g2 [rows,768];
                                                // H [rows,2048]; {64 cols, 64 rows} boxes
    CUtensorMap tmQKV, tmQKV64;                 // [rows, 2304] with {64,128} / {64,64} boxes
    CUtensorMap tmWin, tmWqkv, tmW1, tmWout;    // {64 cols, 64 rows} boxes
    CUtensorMap tmWo, tmW2;                     // {64 cols, 32 rows} boxes (32-column jobs)
    bf16 *X, *QKV, *C, *X1, *Z, *H;
    float2 *st1, *st2;                          // [128][24]: per-row (mean, M2) of 32-column slices
    const float *b_in;
    const float *bqkv0, *bqkv, *s_qkv;          // first execution: plain bias; later: folded LN2
    const float *bo0, *bo;                      // out-proj bias (later executions: + beta2)
    const float *ln1_g, *s_1, *c_1, *bias_21;   // LN1 gamma; W1 folds; b2 + beta1
    const float *ln2_g, *ln2_b, *s_out, *c_out;
    bf16 *out;
    int out_dim;                                // 512, or 0: the hidden states LN2(z2)
    const int *row_dst;
    int out_rows;
    const int *seq_start, *seq_len;
    int nseq;
    const int *n_rows;
    int *status;
    int *bar;                                   // grid-barrier counter (zeroed by the launcher)
    int n_exec;                                 // >= 1
    float eps;
    unsigned long long wait_ns;
    int withhold_loads;                         // fault injection for tests (see GemmArgs)
};
int small_forward_grid(int num_sms);
// Zeroes the barrier counter, then a cooperative launch on stream s.
cudaError_t launch_forward_small(const SmallFwdArgs &a, int grid, cudaStream_t s);

// ---------------------------------------------------------------- attention --
// Masked bidirectional attention, bf16 tensor-core kernel (mma.sync m16n8k16).
// trigger: the next kernel in the stream is one of ours launched with PDL (see GemmArgs).
cudaError_t launch_attention_bf16(const bf16 *qkv, bf16 *ctx, const int *seq_start,
                                  const int *seq_len, int nseq, int max_len,
                                  const int *status, cudaStream_t s, bool trigger);
// Same operation on tcgen05 for max_len <= 128.  One item = one (group, head); a
// group is one sequence, or two sequences of at most kAttnHalfRows tokens placed
// in the two 64-row halves of one 128-row tile (each query attends only to the
// keys of its own sequence).  groups[g] = {start, length, partner start, partner
// length (0: no partner)} for g < *n_groups (device; written by the prep
// kernels), at most max_groups.  tmQKV / tmQKV64: bf16 maps of the packed
// [rows, 3*768] buffer with a {64, 128} / {64, 64} box and the 128-byte swizzle.
constexpr int kAttnTcMaxLen = 128;
constexpr int kAttnHalfRows = 64;
// wait_ns: limit of the kernel's bounded waits (0 = kWaitLimitNs, 2 s).
cudaError_t launch_attention_tc(const CUtensorMap &tmQKV, const CUtensorMap &tmQKV64, bf16 *ctx, const int4 *groups,
                                const int *n_groups, int max_groups, int *status, int num_sms, cudaStream_t s,
                                bool trigger, unsigned long long wait_ns = 0);
// Same operation on tcgen05 for 128 < max_len <= 512 (one item = one (sequence,
// 128-query block, head); keys in 64-key blocks with a running maximum, two items
// in flight per CTA); tmQKV as above, tmQKV64 with a {64, 64} box.
constexpr int kAttnTcLongMaxLen = 512;
cudaError_t launch_attention_tc_long(const CUtensorMap &tmQKV, const CUtensorMap &tmQKV64, bf16 *ctx,
                                     const int *seq_start, const int *seq_len, int nseq, int *status, int num_sms,
                                     cudaStream_t s, bool trigger, unsigned long long wait_ns = 0);
cudaError_t launch_attention_f32(const float *qkv, float *ctx, const int *seq_start,
                                 const int *seq_len, int nseq, int max_len,
                                 const int *status, cudaStream_t s);

// ---------------------------------------------------- prep / embed / output --
// max_rows: the handle's max_tokens; a larger total sets ALBERT_ERR_SHAPE.
// Besides the per-sequence rows, both build the attention groups of
// launch_attention_tc (groups: room for one per sequence; n_groups: one int).
cudaError_t launch_prep_padded(const uint8_t *mask, int B, int T, int pack, int max_rows,
                               int *seq_start, int *seq_len, int *n_rows, int *status,
                               int4 *groups, int *n_groups, cudaStream_t s, bool trigger);
cudaError_t launch_prep_varlen(const int32_t *cu, int nseq, int max_len, int max_rows,
                               int *seq_start, int *seq_len, int *n_rows, int *status,
                               int4 *groups, int *n_groups, cudaStream_t s, bool trigger);

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
    int trigger;        // the next launch is one of ours with PDL (see GemmArgs)
    const float *emb_in;  // non-null: rows [n_rows, 128] fp32 taken as E (no gather, no LayerNorm)
};
cudaError_t launch_embed(const EmbedArgs &a, cudaStream_t s);
// The embedding and the input projection in one kernel (bf16): X = E W_in^T + b_in
// with E = the rows launch_embed would write, kept in shared memory (a.E and
// a.out_f32 unused).  tmWin: W_in [768, 128] bf16 with a {64, 128} box and the
// 128-byte swizzle; a.rows_cap a multiple of 128; X: [rows_cap, 768] bf16.
// withhold_w (failure-path tests): W_in is never loaded, so the wait for it runs out.
cudaError_t launch_embed_proj(const CUtensorMap &tmWin, const EmbedArgs &a, const float *b_in, bf16 *X, int num_sms,
                              cudaStream_t s, unsigned long long wait_ns = 0, bool withhold_w = false);
// out[b][d][t] = t < seq_len[b] ? src[(b*T + t)*D + d] : 0 (elem_bytes 2 or 4),
// the last kernel of a forward with the transposed output layout.
cudaError_t launch_transpose_out(const void *src, void *out, int B, int T, int D, int elem_bytes,
                                 const int *seq_len, const int *status, cudaStream_t s);

// out[(b*T + t)] = 0 for padding slots t >= seq_len[b]; D columns of elem_bytes.
cudaError_t launch_zero_pad(void *out, int B, int T, int D, int elem_bytes, const int *seq_len,
                            const int *status, cudaStream_t s);
// out[row_dst[r]] = X[r] for r < n_rows with row_dst[r] >= 0.
cudaError_t launch_scatter_rows(const void *X, void *out, int D, int elem_bytes, int rows_cap,
                                const int *n_rows, const int *row_dst, const int *status,
                                cudaStream_t s);

// Folded LayerNorm constants of a linear layer W [N, K] (bf16) that consumes
// LN(z) = (z - mu) * rstd * gamma + beta:  s = W gamma,  c = W beta + b.
cudaError_t launch_fold_ln(const bf16 *W, int N, int K, const float *gamma, const float *beta,
                           const float *b, float *s_out, float *c_out, cudaStream_t s);
// out[row_dst[r]] = LN(z) = rstd * zg - rstd * mu * gamma + beta for r < n_rows
// (zg = z * gamma, [rows, 768] bf16; stats [rows][6]); row_dst == nullptr: out[r].
// out_rows bounds row_dst (a larger destination is recorded as ALBERT_ERR_SHAPE).
cudaError_t launch_ln_rows(const bf16 *zg, const float2 *stats, const float *gamma, const float *beta,
                           float eps, bf16 *out, const int *row_dst, int out_rows, int rows_cap,
                           const int *n_rows, int *status, cudaStream_t s);
// out[i] = a[i] + b[i]
cudaError_t launch_vec_add(const float *a, const float *b, float *out, int n, cudaStream_t s);

// ---------------------------------------------------------------- E4M3 path --
// x [rows, K] bf16 -> q [rows, K] E4M3 and scale [rows] (fp8.cu); rows past *n_rows
// (if given) are left alone; K a multiple of 256, at most 2048.
cudaError_t launch_quant_rows_e4m3(const bf16 *x, int K, int rows, const int *n_rows, uint8_t *q, float *scale,
                                   const int *status, cudaStream_t s, bool pdl, bool trigger);
// Folded LayerNorm constants of an E4M3 weight with row scales (see launch_fold_ln).
cudaError_t launch_fold_ln_e4m3(const uint8_t *Wq, const float *sw, int N, int K, const float *gamma,
                                const float *beta, const float *b, float *s_out, float *c_out, cudaStream_t s);

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
