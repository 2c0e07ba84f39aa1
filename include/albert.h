/*
 * albert.h -- C ABI of the B200 (sm_100a) forward pass of Kokoro's ALBERT
 * phoneme encoder.
 *
 * What the library computes ("ALBERT: How Kokoro's Phoneme Encoder Works, and
 * Where CKE Has Reached It", section "Inside One Real ALBERT Layer", steps 1-6
 * and the paragraph after them):
 *   E  = LN_128(word[id] + pos[t] + type[0])            (three-table embedding)
 *   X  = E W_in^T + b_in                                 (128 -> 768)
 *   repeat n_exec times with ONE shared weight set:
 *     [Q|K|V] = X [Wq;Wk;Wv]^T + b
 *     C  = per head h (64 columns each): softmax(Q_h K_h^T / 8 + mask) V_h
 *     X1 = LN(X + C Wo^T + bo)
 *     X  = LN(X1 + GELU_tanh(X1 W1^T + b1) W2^T + b2)
 *   Y  = X W_out^T + b_out                               (768 -> 512)
 * The mask is a key-padding mask: slot u of sequence b takes part only if
 * u < L_b ("How Kokoro TTS Works and Where CKE Stands", section "What ALBERT
 * does here": softmax(QK^T/sqrt(d) + mask) V).  Positions are slot indices
 * 0..T-1 (right padding); token type 0.
 *
 * Conventions (from "How Kokoro TTS Works and Where CKE Stands", sections on
 * checked kernels and the compiler side: integer status, validate before
 * writing, caller-owned memory planned up front):
 *   - every call returns an int status, ALBERT_OK (0) on success;
 *   - host-detected errors return before anything is enqueued, so `out` is
 *     untouched;
 *   - device-detected errors (bad id, bad mask, bad sequence lengths, an
 *     expired bounded wait) are recorded in a device status word; every later
 *     kernel of the same forward then exits without writing, so `out` is left
 *     as it was.  albert_get_status() reports that word;
 *   - all memory the forward pass needs is allocated by albert_create();
 *     albert_forward() and albert_forward_varlen() allocate nothing.
 *
 * All device pointers are CUDA device addresses on the device that was current
 * when the handle was created.  `stream` is a cudaStream_t passed as void*
 * (NULL = legacy default stream).  A handle may be used from one stream at a
 * time; two forwards that overlap on different streams race on its workspace.
 */
#ifndef ALBERT_B200_H
#define ALBERT_B200_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* ---- status codes ---- */
#define ALBERT_OK           0
#define ALBERT_ERR_NULL     1  /* a required pointer is NULL                        */
#define ALBERT_ERR_CONFIG   2  /* unsupported albert_config                         */
#define ALBERT_ERR_SHAPE    3  /* B, T, nseq, max_len or token count out of range   */
#define ALBERT_ERR_ID       4  /* device: a valid slot holds an id outside [0,vocab) */
#define ALBERT_ERR_MASK     5  /* device: a mask row is not a non-empty 1..1 0..0 prefix */
#define ALBERT_ERR_SEQLENS  6  /* device: cu_seqlens not 0-based / lengths outside [1, max_pos] */
#define ALBERT_ERR_CUDA     7  /* a CUDA runtime call failed                        */
#define ALBERT_ERR_TIMEOUT  8  /* device: a bounded wait inside a kernel expired    */
#define ALBERT_ERR_ALLOC    9  /* device memory allocation failed in albert_create  */

/* ---- precision of the whole path ---- */
#define ALBERT_BF16 0  /* bf16 weights and activations, fp32 accumulation and norms */
#define ALBERT_FP32 1  /* fp32 everywhere (SIMT kernels; small workloads)          */
#define ALBERT_FP8  2  /* the four layer GEMMs (Q|K|V, out-proj, FFN up and down)
                          on E4M3 operands with per-row scales (activations per
                          token, weights per output channel), everything else as
                          ALBERT_BF16; see albert_test_quant_e4m3               */

/* Architecture and capacity.  The kernels support exactly: emb 128, hidden 768,
 * heads 12 (64 wide), ffn 2048, max_pos <= 512, out_dim 512 or 0 (0 = return the
 * [.., 768] hidden states).  n_exec >= 0 is free.  n_groups: distinct layer weight
 * sets, 1 <= n_groups <= max(n_exec, 1); execution i uses set
 * floor(i * n_groups / n_exec), i.e. consecutive blocks of executions share a set
 * ("ALBERT: How Kokoro's Phoneme Encoder Works", section "2. Cross-layer
 * parameter sharing"; 1 = one fully shared layer, Kokoro's case).  max_tokens
 * is the workspace capacity in rows: albert_forward needs B*T <= max_tokens,
 * albert_forward_varlen needs total tokens <= max_tokens. */
typedef struct {
    int vocab;       /* 178 for Kokoro                                  */
    int emb;         /* E = 128                                         */
    int hidden;      /* H = 768                                         */
    int heads;       /* 12                                              */
    int ffn;         /* 2048                                            */
    int n_exec;      /* executions of the shared layer, 12 for Kokoro   */
    int n_groups;    /* distinct layer weight sets (1 = fully shared)   */
    int max_pos;     /* rows of the position table, <= 512              */
    int n_types;     /* rows of the token-type table (type 0 is used)   */
    int out_dim;     /* 512, or 0 for no final projection               */
    int dtype;       /* ALBERT_BF16 or ALBERT_FP32                      */
    int max_tokens;  /* workspace capacity in rows (>= 1)               */
    int pack;        /* albert_forward: 1 = pack valid tokens by length
                        (the GEMMs run on sum(L_b) rows), 0 = run on all B*T
                        padded rows                                     */
    int out_layout;  /* albert_forward output: 0 = [B, T, D] token-major;
                        1 = [B, D, T], each sequence's projection transposed
                        ("ALBERT: How Kokoro's Phoneme Encoder Works", section
                        "Inside One Real ALBERT Layer": Kokoro projects to
                        [T, 512] and transposes it).  Padding positions are
                        0 in both.  albert_forward_varlen needs 0.      */
    float ln_eps;    /* LayerNorm epsilon, 1e-12 for Kokoro             */
} albert_config;

/* Parameters: DEVICE pointers to fp32 tensors in PyTorch layouts ([out, in] for
 * linears).  albert_create copies them (converting to bf16 for ALBERT_BF16), so
 * the caller may free them afterwards.  w_out/b_out may be NULL if out_dim == 0.
 * With n_groups > 1 every layer parameter (wq .. ln2_b) holds n_groups copies
 * back to back, set g at offset g * (its size); the embedding tables, w_in/b_in
 * and w_out/b_out are single. */
typedef struct {
    const float *word;      /* [vocab, emb]     */
    const float *pos;       /* [max_pos, emb]   */
    const float *type;      /* [n_types, emb]   */
    const float *emb_ln_g;  /* [emb]            */
    const float *emb_ln_b;  /* [emb]            */
    const float *w_in;      /* [hidden, emb]    */
    const float *b_in;      /* [hidden]         */
    const float *wq, *bq;   /* [hidden, hidden], [hidden] */
    const float *wk, *bk;
    const float *wv, *bv;
    const float *wo, *bo;
    const float *ln1_g, *ln1_b;  /* [hidden]    */
    const float *w1, *b1;   /* [ffn, hidden], [ffn]       */
    const float *w2, *b2;   /* [hidden, ffn], [hidden]    */
    const float *ln2_g, *ln2_b;
    const float *w_out, *b_out;  /* [out_dim, hidden], [out_dim] */
} albert_weights;

typedef struct albert_handle albert_handle;

/* Validate cfg, copy/pack the weights, allocate the workspace for max_tokens
 * rows and build the TMA descriptors.  Synchronous.  On success *out receives
 * the handle; on failure *out is NULL and nothing stays allocated. */
int albert_create(const albert_weights *w, const albert_config *cfg, albert_handle **out);

/* Padded batch.  ids: [B, T] int64 (device); mask: [B, T] uint8 (device),
 * 1 = token, each row a non-empty prefix of ones; out: [B, T, D] (device),
 * D = out_dim or hidden, bf16 for ALBERT_BF16 and fp32 for ALBERT_FP32.
 * Rows at padding slots are written as zeros.  Ids at padding slots are not
 * read for the result and may hold anything.  Asynchronous on `stream`.
 * Host errors: NULL pointers, B < 1, T < 1, T > max_pos, B*T > max_tokens. */
int albert_forward(albert_handle *h, const int64_t *ids, const uint8_t *mask, int B, int T,
                   void *out, void *stream);

/* Packed variable-length batch.  ids: [N_tok] int64 (device), the sequences
 * back to back; cu_seqlens: [nseq+1] int32 (device), cu_seqlens[0] = 0,
 * sequence s = rows cu_seqlens[s] .. cu_seqlens[s+1]-1, each length in
 * [1, max_pos] and N_tok = cu_seqlens[nseq] <= max_tokens (checked on the
 * device); out: [N_tok, D] (device).  max_len bounds every length (host check
 * max_len <= max_pos; the device checks each length against it).
 * Asynchronous on `stream`. */
int albert_forward_varlen(albert_handle *h, const int64_t *ids, const int32_t *cu_seqlens,
                          int nseq, int max_len, void *out, void *stream);

/* The encoder from its post-embedding-LayerNorm rows instead of ids: emb is
 * [N_tok, 128] fp32 (device, 16-byte aligned), the rows of the packed
 * sequences as albert_forward_varlen lays out ids; everything after the
 * embedding's LayerNorm (the 128 -> 768 projection on) runs as in
 * albert_forward_varlen, and out is [N_tok, D].  This is the input the pages
 * evaluate a compiled encoder on ("Kokoro-82M-encoder-hailo10h", section "How
 * to deploy on Hailo-10H": the encoder takes the [1, 128, 128] LayerNorm output
 * computed on the CPU; section "Eval results": 16 random N(0,1) inputs of that
 * shape).
 * Errors as albert_forward_varlen; out_layout must be 0. */
int albert_forward_embedded(albert_handle *h, const float *emb, const int32_t *cu_seqlens, int nseq, int max_len,
                            void *out, void *stream);

/* Convenience path with HOST buffers: copies ids/mask (pinned or pageable) to
 * the handle's device staging area, runs albert_forward, copies the result
 * back to out_host and synchronizes `stream`.  Returns the device status. */
int albert_forward_host(albert_handle *h, const int64_t *ids_host, const uint8_t *mask_host,
                        int B, int T, void *out_host, void *stream);

/* Pipelined path with HOST buffers for a sequence of batches (throughput
 * serving).  Each call enqueues one batch on `stream`: copies of ids/mask to one
 * of two device staging slots, the forward, and the copy of its output back to
 * out_host on a stream the handle owns, so that a batch's output copy overlaps
 * the next batch's forward.  The call does not wait for its own batch; it first
 * waits for the batch issued two calls earlier (same slot) to reach the host and
 * returns that batch's status (ALBERT_OK when there was none), or a host-side
 * error.  Host buffers of a batch must stay valid, and out_host unread, until it
 * has been waited for (pinned host memory for the copies to overlap).  The first
 * call allocates the second staging slot (max_tokens rows).  Do not mix with
 * albert_forward_host on the same handle while batches are in flight. */
int albert_forward_host_async(albert_handle *h, const int64_t *ids_host, const uint8_t *mask_host,
                              int B, int T, void *out_host, void *stream);

/* The same pipelined path for a PACKED batch (as albert_forward_varlen): ids_host
 * [cu_seqlens_host[nseq]] int64, cu_seqlens_host [nseq + 1] int32 on the host,
 * out_host [cu_seqlens_host[nseq], out_dim] -- only the valid rows travel to the
 * device and back.  The copy sizes are read from cu_seqlens_host: cu[0] != 0 or a
 * total outside 1..max_tokens returns ALBERT_ERR_SHAPE before any work; the rest
 * of the lengths are checked on the device as in albert_forward_varlen.  Shares
 * the staging slots, ordering and waiting rules of albert_forward_host_async
 * (the two may be mixed on one handle). */
int albert_forward_varlen_host_async(albert_handle *h, const int64_t *ids_host, const int32_t *cu_seqlens_host,
                                     int nseq, int max_len, void *out_host, void *stream);

/* Wait for every batch of albert_forward_host_async / albert_forward_varlen_host_async
 * still in flight; returns the first non-OK status among them (ALBERT_OK if none). */
int albert_forward_host_wait(albert_handle *h);

/* Synchronize `stream` and return the status recorded by the last forward on
 * this handle (ALBERT_OK, ALBERT_ERR_ID, _MASK, _SEQLENS, _SHAPE or _TIMEOUT). */
int albert_get_status(albert_handle *h, void *stream);

/* Free everything the handle owns.  NULL is ignored. */
void albert_destroy(albert_handle *h);

/* ---- bounded waits and their failure path ----
 * Every wait inside the bf16 kernels (on a TMA copy, a tensor-core product or
 * another warp's hand-off) is bounded in wall time.  When a wait runs out, the
 * kernel records ALBERT_ERR_TIMEOUT in the status word, lets its in-flight
 * copies and products finish, frees its tensor memory and returns; every later
 * kernel of the forward then skips its work, so `out` is left as it was and
 * the context stays usable.  (A wait that runs out inside the kernel that
 * writes `out` stops that kernel's remaining work; rows it had already
 * written stay written.)  (The pages' checked-kernel contract: a failed
 * check stops downstream work and reports an integer status -- "How Kokoro TTS
 * Works and Where CKE Stands", sections on checked kernels.)
 *
 * albert_set_wait_limit: the limit, in nanoseconds, of the waits of every
 * kernel of later forwards on this handle; 0 restores the default (2 s).
 * ns < 0 returns ALBERT_ERR_CONFIG.  A limit shorter than a kernel's normal
 * waits makes healthy forwards fail with ALBERT_ERR_TIMEOUT. */
int albert_set_wait_limit(albert_handle *h, long long ns);

/* Failure injection for tests of the path above: on later forwards, the
 * launches of the kernel classes set in class_mask (bit i = class i of
 * albert_profile_name; only the GEMM classes, the small-batch kernel and the
 * embedding + input projection kernel are accepted) run with their TMA
 * producer withholding every load, so their first wait on an operand tile can
 * never complete and runs out after the wait limit.  Nothing faults: the
 * forward reports ALBERT_ERR_TIMEOUT through albert_get_status with `out`
 * untouched.  0 turns it off.  Returns ALBERT_ERR_CONFIG for other classes, or
 * for a non-zero mask on an ALBERT_FP32 handle (its kernels have no waits). */
int albert_test_stall(albert_handle *h, int class_mask);

/* Number of kernel launches one forward of this handle enqueues for a batch
 * of max_tokens rows through the per-layer kernels (padded_api: 1 for
 * albert_forward, 0 for albert_forward_varlen). */
int albert_launches_per_forward(const albert_handle *h, int padded_api);

/* Kernel launches the last forward on this handle enqueued (-1 for NULL). */
int albert_last_forward_launches(const albert_handle *h);

/* Small batches.  When a forward holds at most 128 token rows (B*T <= 128 for
 * albert_forward, nseq*max_len <= 128 for albert_forward_varlen) and the handle
 * is bf16 with one weight set (n_groups == 1) and n_exec >= 1, everything after
 * the embedding runs in ONE persistent kernel: a cooperative grid that walks
 * the layer's steps as phases separated by grid barriers (Q|K|V, attention,
 * out-projection, FFN up, FFN down, each over all SMs of the grid, with the
 * intermediate tiles in L2), instead of ~64 per-layer launches ("ALBERT: How Kokoro's
 * Phoneme Encoder Works", section "Inside One Real ALBERT Layer", steps 2-6,
 * and "2. Cross-layer parameter sharing").  Same results within the stated
 * tolerances; deterministic.  enable: 1 (default) uses it when it applies,
 * 0 always runs the per-layer kernels.  Other values: ALBERT_ERR_CONFIG. */
int albert_set_small_batch_kernel(albert_handle *h, int enable);

/* ---- per-kernel timing (optional) ----
 * albert_profile_enable(h, class_mask): for every kernel class whose bit is set
 * in class_mask (-1 = all, 0 = off), each forward records a CUDA event before
 * and after each launch of that class on the forward's stream.  albert_profile_read synchronizes the
 * last recorded stream and adds, per kernel class, the launch count and the
 * summed milliseconds since the last reset.  Classes are numbered
 * 0..albert_profile_classes()-1 and named by albert_profile_name(). */
int albert_profile_enable(albert_handle *h, int class_mask);
/* retain = 1: a read keeps the recorded event pairs armed instead of recycling
 * them.  For a forward captured in a CUDA graph with profiling enabled: every
 * replay re-records the same events, and a read after each replay adds that
 * replay's times.  retain = 0 (default) disarms them. */
int albert_profile_retain(albert_handle *h, int retain);
/* Time only launch k of each enabled class with k % stride == offset, k counted
 * per class from this call (default stride 1: every launch).  Fewer event
 * records between launches keep more of the launch chaining intact. */
int albert_profile_stride(albert_handle *h, int stride, int offset);
int albert_profile_reset(albert_handle *h);
int albert_profile_classes(void);
const char *albert_profile_name(int cls);
int albert_profile_read(albert_handle *h, int *launches, double *ms);

/* ---- length regulation (the step after the encoder) ----
 * "How Kokoro TTS Works and Where CKE Stands", section "The time axis is where a
 * circuit becomes difficult": per token, the sigmoid duration channels are summed,
 * divided by the speed, rounded and clamped to at least one frame; A = sum d[t]
 * is the number of aligned frames; token features are repeated by the duration
 * vector ("Qwen3-TTS and Kokoro: Two Routes from Text to Speech", section "Path
 * one: Kokoro decides how long each sound lasts": durations 2, 1, 3 ->
 * p1 p1 p2 p3 p3 p3).
 *
 * For a packed batch of nseq sequences (token rows in cu_seqlens order, n_tok =
 * cu_seqlens[nseq]), all device pointers, asynchronous on `stream`:
 *   logits      [n_tok, C] fp32: duration channels (pre-sigmoid);
 *   feats       [n_tok, D] bf16: token features (the encoder output), 16-byte aligned;
 *   durations   [n_tok] int32 out: d[t] = max(1, rint(sum_c sigmoid(z[t,c]) / speed)),
 *               taken in fp64, rint = round half to even;
 *   frame_start [n_tok] int32 out: first frame of token t (frames of all sequences
 *               back to back: token t owns frames frame_start[t] .. + d[t] - 1);
 *   cu_frames   [nseq+1] int32 out: sequence b owns frames cu_frames[b] ..
 *               cu_frames[b+1]-1, so A_b = cu_frames[b+1] - cu_frames[b];
 *   frames      [max_frames, D] bf16 out: frame rows, 16-byte aligned;
 *   scratch     device workspace of albert_length_regulate_scratch_bytes(n_tok)
 *               bytes, 8-byte aligned (owned by the caller; one call at a time);
 *   status      [1] int32 out: ALBERT_OK, ALBERT_ERR_SEQLENS (cu_seqlens not
 *               monotone from 0 to n_tok) or ALBERT_ERR_SHAPE (sum of durations
 *               above max_frames; frames untouched).
 * Host-side errors (returned at once): NULL pointers, C < 1, D not a positive
 * multiple of 8, nseq or n_tok < 1 (ALBERT_ERR_SHAPE), speed not finite and
 * positive or an unaligned feats/frames/scratch (ALBERT_ERR_CONFIG).  Allocates
 * nothing.
 * This step is not part of the pages' encoder; it is the workload their text
 * names next on Kokoro's path. */
int albert_length_regulate(const float *logits, int C, float speed, const void *feats, int D,
                           const int32_t *cu_seqlens, int nseq, int n_tok, int32_t *durations,
                           int32_t *frame_start, int32_t *cu_frames, void *frames, int max_frames,
                           void *scratch, int32_t *status, void *stream);

/* Bytes of device scratch albert_length_regulate needs for n_tok tokens. */
size_t albert_length_regulate_scratch_bytes(int n_tok);

/* ---- single-kernel entry points (parity tests of one kernel) ----
 * These run one kernel of the path in isolation, synchronously, and return its
 * status.  They allocate and free temporary device memory. */

/* Y = epilogue(A W^T + bias) with the tcgen05 GEMM.  A: [M, K] bf16, W: [N, K]
 * bf16, bias: [N] fp32 (device).  epi: 0 = bias -> bf16 Y[M, N];
 * 1 = tanh-GELU(+bias) -> bf16; 2 = LN(A W^T + bias + R; g, b, eps) -> bf16,
 * with R: [M, N] bf16 and N == 768; 3 = bias -> bf16 rows scattered to
 * row_dst[r] (row_dst[r] < 0 skips the row).  K % 64 == 0, N % 256 == 0;
 * bias and ln_g 16-byte aligned (else ALBERT_ERR_CONFIG).  Adding
 * ALBERT_GEMM_SINGLE_CTA, ALBERT_GEMM_CTA_PAIR or ALBERT_GEMM_NARROW to epi
 * forces that kernel variant (one CTA per 128x256 tile, a two-CTA cluster per
 * 256x256 tile, or one CTA per 128x128 tile); by default the choice is
 * albert_forward's: one CTA for M <= 128, the 128x128 tile when the pair tiles
 * would leave clusters idle and every 128x128 tile runs at once, else the pair.
 * More than one of the three: ALBERT_ERR_CONFIG. */
#define ALBERT_GEMM_SINGLE_CTA 16
#define ALBERT_GEMM_CTA_PAIR 32
#define ALBERT_GEMM_NARROW 128
/* Adding ALBERT_GEMM_E4M3 runs the E4M3 variant: A and W are first quantized
 * per row as albert_test_quant_e4m3 does (into temporaries), then multiplied
 * on tcgen05 (kind::f8f6f4) with the epilogue starting from
 * acc * a_scale[row] * w_scale[col].  Needs K % 256 == 0 and K <= 2048. */
#define ALBERT_GEMM_E4M3 64
int albert_test_gemm(const void *A, const void *W, const float *bias, const void *R,
                     const float *ln_g, const float *ln_b, float eps, const int32_t *row_dst,
                     void *Y, int M, int N, int K, int epi, void *stream);

/* Row quantization of the FP8 variant (the reading of "Kokoro-82M-encoder-
 * hailo10h", section "Eval results", that a quantized encoder is compared with
 * its full-precision outputs; the scheme is this library's): for each row of
 * x [rows, K] bf16 (device), amax = max |x|, scale[row] = amax / 448 and
 * q = E4M3(fp32(x * (448 / amax))) with round to nearest even and saturation
 * (fp32 divisions and product); a row of zeros gives scale 0 and q 0.
 * q: [rows, K] bytes (E4M3 codes), scale: [rows] fp32, device.  K % 256 == 0,
 * 256 <= K <= 2048 (else ALBERT_ERR_SHAPE).  Synchronous. */
int albert_test_quant_e4m3(const void *x, int rows, int K, void *q, float *scale, void *stream);

/* Masked bidirectional attention on a packed [N_tok, 3*768] bf16 QKV buffer
 * (Q | K | V, head h = columns 64h..64h+63 of each); cu_seqlens as in
 * albert_forward_varlen; ctx: [N_tok, 768] bf16.  dtype ALBERT_BF16 runs the
 * kernel the forward pass uses for this max_len (tcgen05 with one item per
 * (group, head) for max_len <= 128, a group being one sequence or two of at
 * most 64 tokens each (albert_test_attention_groups);
 * tcgen05 with one item per (sequence, 128-query block, head) and all of its
 * scores in tensor memory for 128 < max_len <= 512); 2 forces the mma.sync
 * kernel; ALBERT_FP32 runs the fp32 kernel on fp32 buffers. */
int albert_test_attention(const void *qkv, const int32_t *cu_seqlens, int nseq, int max_len,
                          void *ctx, int dtype, void *stream);

/* The attention groups the forward pass forms for a packed batch (device
 * cu_seqlens as in albert_forward_varlen): the sequences of at most 64 tokens
 * are paired in batch order (1st with 2nd, 3rd with 4th, ...), each pair sharing
 * one item as its two 64-row halves; longer sequences and an unpaired last short
 * one have an item each.  groups_out: host, room for nseq int32 quadruples
 * {start row, length, partner start row, partner length (0: none)}: the pairs
 * first, then the longer sequences in batch order, then the unpaired short one;
 * *n_out: the number written.
 * Synchronous.  Invalid cu_seqlens: ALBERT_ERR_SEQLENS. */
int albert_test_attention_groups(const int32_t *cu_seqlens, int nseq, int max_len, int32_t *groups_out,
                                 int *n_out, void *stream);

/* ---- residual + LayerNorm GEMM without any device allocation ----
 * The pages have no counterpart of this entry point; it exists for callers
 * that must not allocate device memory while running -- a real-time audio
 * thread that cannot absorb cudaMalloc's device-wide synchronization and
 * latency, or a runtime that lays out all device memory before its first
 * request.  It computes Y = LN(A W^T + bias + R; ln_g, ln_b, eps) with the
 * same two kernels as albert_test_gemm with epi = 2 (the GEMM whose epilogue
 * forms the pre-norm row, then the row normalization), but their scratch
 * (z * ln_g as bf16, per-row partial statistics, a row-count word and the
 * status word) lives in file-scope __device__ arrays of about 3.1 MiB inside
 * the library instead of memory the call allocates; it calls no
 * cudaMalloc/cudaFree.
 *   A: [M, K] bf16, W: [768, K] bf16, bias/ln_g/ln_b: [768] fp32,
 *   R: [M, 768] bf16, Y: [M, 768] bf16, all device pointers the caller owns.
 *   Limits: 1 <= M <= 2048 (the rows the arrays hold), K % 64 == 0;
 *   anything else returns ALBERT_ERR_SHAPE before any work is enqueued;
 *   bias and ln_g must be 16-byte aligned (else ALBERT_ERR_CONFIG).
 * The arrays are reserved on every device where the library's module holding
 * them is loaded and stay until the process exits.  Every call looks up their
 * device addresses (cudaGetSymbolAddress) with the caller's device current.
 * The CUDA runtime loads a library's modules lazily: the first call on a
 * device loads the modules behind it (the arrays and the two kernels), which
 * reserves their memory and synchronizes the device once.  The no-allocation
 * guarantee therefore holds from the second call on: make one warm-up call on
 * each device at set-up time, before any stream capture and before the thread
 * that must not allocate starts calling.  Every call shares the same arrays
 * (the status word is reset by each call; the intermediates are rewritten
 * before they are read, so nothing else needs clearing), so calls that overlap
 * on the GPU -- on different streams or from different threads -- race and
 * must be serialized by the caller.  Synchronous: the call synchronizes its
 * stream before returning the kernel's status, so holding a host-side lock
 * around each call is enough to serialize them. */
int albert_gemm_residual_ln_noalloc(const void *A, const void *W, const float *bias, const void *R,
                                    const float *ln_g, const float *ln_b, float eps, void *Y, int M,
                                    int K, void *stream);

#ifdef __cplusplus
}
#endif
#endif /* ALBERT_B200_H */
