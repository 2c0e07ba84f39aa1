// albert_api.cu -- the C ABI (include/albert.h): weights, workspace, TMA
// descriptors and the launch schedule of one forward pass.
//
// Schedule of one forward ("ALBERT: How Kokoro's Phoneme Encoder Works",
// section "Inside One Real ALBERT Layer" and the paragraph after it):
//   prep (mask / lengths -> packed row offsets) -> embed+LN -> GEMM 128->768
//   -> n_exec x [ GEMM Q|K|V -> attention -> GEMM Wo + residual + LN
//                 -> GEMM W1 + GELU -> GEMM W2 + residual + LN ]
//   -> GEMM 768->512 scattered to [B, T, 512] -> zero padding rows.
// The shared layer's weights exist once in device memory and every execution
// reads the same copy, which stays resident in L2 across executions.
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <new>
#include <vector>

#include "albert.h"
#include "kernels.h"

using namespace albert;

namespace {

enum ProfClass {
    kProfPrep = 0, kProfEmbed, kProfGemmIn, kProfGemmQKV, kProfAttention, kProfGemmWoLN,
    kProfGemmW1Gelu, kProfGemmW2LN, kProfGemmOut, kProfOutput, kProfLayerNorm, kProfSmall, kProfQuant,
    kProfEmbedProj, kProfClasses
};
const char *kProfNames[kProfClasses] = {
    "prep", "embed_ln", "gemm_in_proj", "gemm_qkv", "attention", "gemm_out_proj_ln",
    "gemm_ffn_up_gelu", "gemm_ffn_down_ln", "gemm_final_proj", "output_rows", "layer_norm_f32",
    "small_batch_forward", "quant_e4m3", "embed_proj"};

constexpr int kEventPool = 16384;

}  // namespace

struct albert_handle {
    albert_config cfg{};
    int device = 0, num_sms = 0;
    int rows_cap = 0;   // workspace rows (multiple of 128)
    int seq_cap = 0;    // sequences
    std::vector<void *> allocs;

    // parameters shared by every execution
    float *word = nullptr, *pos = nullptr, *type = nullptr, *emb_g = nullptr, *emb_b = nullptr;
    float *b_in = nullptr, *b_out = nullptr;
    void *w_in = nullptr, *w_out = nullptr;
    void *wblock = nullptr;
    size_t wblock_bytes = 0;
    // one layer weight set per group; execution l uses group group_of(cfg, l)
    struct Group {
        float *bqkv = nullptr, *bo = nullptr, *ln1_g = nullptr, *ln1_b = nullptr;
        float *b1 = nullptr, *b2 = nullptr, *ln2_g = nullptr, *ln2_b = nullptr;
        void *wqkv = nullptr, *wo = nullptr, *w1 = nullptr, *w2 = nullptr;
        CUtensorMap tm_wqkv, tm_wo, tm_w1, tm_w2;
        float *s_1 = nullptr, *c_1 = nullptr, *bias_21 = nullptr;  // bf16: this group's LN1 folded
        // ALBERT_FP8: E4M3 copies of the four layer matrices with per-row scales
        uint8_t *q_wqkv = nullptr, *q_wo = nullptr, *q_w1 = nullptr, *q_w2 = nullptr;
        float *s_wqkv = nullptr, *s_wo = nullptr, *s_w1 = nullptr, *s_w2 = nullptr;
        CUtensorMap tq_wqkv, tq_wo, tq_w1, tq_w2;
    };
    std::vector<Group> grp;
    // bf16, execution l >= 1: its group's Q|K|V and out-projection with the LN2
    // of execution l-1 (possibly another group) folded in
    struct Exec {
        float *s_qkv = nullptr, *c_qkv = nullptr, *bias_o2 = nullptr;
    };
    std::vector<Exec> ex;

    // workspace
    // bf16: X = input projection output, X1 = z1 * gamma1, Z = z2 * gamma2 (z1, z2:
    // the pre-norm rows of the two LayerNorms, normalized by their consumers);
    // fp32: X, X1 = LayerNorm outputs, Z = pre-norm rows.
    void *E = nullptr, *X = nullptr, *QKV = nullptr, *C = nullptr, *X1 = nullptr, *H = nullptr, *Z = nullptr;
    float2 *st1 = nullptr, *st2 = nullptr;  // partial (mean, M2) of z1 / z2, [rows][6]
    // folded LayerNorm constants (s = W gamma, c = W beta + b, biases plus the beta
    // of a rebuilt residual): per group and per execution above, the final ones here
    float *fold = nullptr;
    float *s_out = nullptr, *c_out = nullptr;
    int *seq_start = nullptr, *seq_len = nullptr, *row_dst = nullptr, *n_rows = nullptr, *status = nullptr;
    int4 *att_groups = nullptr;  // attention items of sequences <= 128 tokens (one or two sequences each)
    int *n_att_groups = nullptr;

    // out_layout 1: token-major staging of the output, transposed per sequence into `out`
    void *tout = nullptr;

    // ALBERT_FP8: the A operand of the current layer GEMM as E4M3 codes with row
    // scales (one buffer reused by every GEMM), seen as [rows, 768] and [rows, 2048]
    uint8_t *qA = nullptr;
    float *sA = nullptr;
    CUtensorMap tq_A768, tq_A2048;

    // host-buffer staging
    int64_t *st_ids = nullptr;
    uint8_t *st_mask = nullptr;
    void *st_out = nullptr;

    // pipelined host path: two staging slots (slot 0 is the one above), a copy
    // stream for the outputs, per-slot events and pinned per-batch status words
    struct Slot {
        int64_t *ids = nullptr;
        uint8_t *mask = nullptr;
        int32_t *cu = nullptr;           // cu_seqlens of a packed batch
        void *out = nullptr;
        cudaEvent_t d2h_done = nullptr;  // output copied to the host
        cudaEvent_t fwd_done = nullptr;  // forward (and its status copy) complete
        bool in_flight = false;
    } slot[2];
    cudaStream_t copy_stream = nullptr;
    int *status_host = nullptr;          // pinned, [2]
    long long async_issued = 0;

    // TMA descriptors (bf16)
    CUtensorMap tm_E, tm_X, tm_C, tm_X1, tm_H, tm_Z, tm_QKV, tm_QKV64;
    CUtensorMap tm_win, tm_wout;
    CUtensorMap t32_X, t32_QKV, t32_X1, t32_H, t32_Z;  // 32x32-box maps: epilogue stores / residual loads

    // small batches (at most 128 token rows): the whole forward after the
    // embedding in one persistent kernel; its own statistics, FFN partial sums,
    // barrier counter and {64, 64}-box tensor maps
    bool small_ok = false;       // the handle's configuration allows it
    bool small_enabled = true;   // albert_set_small_batch_kernel
    float2 *sst1 = nullptr, *sst2 = nullptr;
    int *sbar = nullptr;
    CUtensorMap sm_E, sm_X, sm_C, sm_X1, sm_Z, sm_H, sm_win, sm_wqkv, sm_wo, sm_w1, sm_w2, sm_wout;
    int last_launches = 0;       // kernel launches of the last forward

    // bounded waits inside the kernels: limit (0 = the kernels' default, 2 s) and,
    // for failure-path tests, kernel classes whose GEMM producer withholds its loads
    unsigned long long wait_ns = 0;
    unsigned stall_mask = 0;

    // per-kernel timing
    unsigned prof_mask = 0;  // classes whose launches are timed
    bool prof_retain = false;  // keep recorded pairs armed after a read (graph replays)
    int prof_stride = 1, prof_offset = 0;  // time launch k of a class iff k % stride == offset
    int prof_count[kProfClasses] = {};      // launches of each class since the stride was set
    bool prof_open = false;                 // begin() recorded a start event for this launch
    std::vector<cudaEvent_t> ev;
    std::vector<int> ev_cls;
    int ev_used = 0;
    int prof_launches[kProfClasses] = {};
    double prof_ms[kProfClasses] = {};
};

namespace {

#define TRY(x)                                                     \
    do {                                                           \
        cudaError_t e_ = (x);                                      \
        if (e_ != cudaSuccess) {                                   \
            if (getenv("ALBERT_DEBUG"))                            \
                fprintf(stderr, "albert: %s failed: %s (%s:%d)\n", #x, \
                        cudaGetErrorString(e_), __FILE__, __LINE__); \
            return ALBERT_ERR_CUDA;                                \
        }                                                          \
    } while (0)

int dev_alloc(albert_handle *h, void **p, size_t bytes) {
    if (bytes == 0) bytes = 16;
    if (cudaMalloc(p, bytes) != cudaSuccess) {
        *p = nullptr;
        return ALBERT_ERR_ALLOC;
    }
    h->allocs.push_back(*p);
    return ALBERT_OK;
}

size_t elem_bytes(const albert_handle *h) { return h->cfg.dtype == ALBERT_FP32 ? 4 : 2; }
int out_width(const albert_handle *h) { return h->cfg.out_dim > 0 ? h->cfg.out_dim : kHidden; }

// Weight group of execution l: ALBERT's grouped sharing splits the executions
// into n_groups consecutive runs of equal length (floor(l * n_groups / n_exec)).
int group_of(const albert_config &c, int l) {
    return c.n_exec > 0 ? (int)((long long)l * c.n_groups / c.n_exec) : 0;
}

int check_config(const albert_config *c) {
    if (c->emb != kEmb || c->hidden != kHidden || c->heads != kHeads || c->ffn != kFfn) return ALBERT_ERR_CONFIG;
    if (c->n_exec < 0 || c->n_groups < 1 || c->n_groups > (c->n_exec > 0 ? c->n_exec : 1)) return ALBERT_ERR_CONFIG;
    if (c->max_pos < 1 || c->max_pos > kMaxPos || c->vocab < 1 || c->n_types < 1) return ALBERT_ERR_CONFIG;
    if (c->out_dim != 0 && c->out_dim != 512) return ALBERT_ERR_CONFIG;
    if (c->dtype != ALBERT_BF16 && c->dtype != ALBERT_FP32 && c->dtype != ALBERT_FP8) return ALBERT_ERR_CONFIG;
    if (c->max_tokens < 1 || c->max_tokens > (1 << 24)) return ALBERT_ERR_CONFIG;
    if (c->pack != 0 && c->pack != 1) return ALBERT_ERR_CONFIG;
    if (c->out_layout != 0 && c->out_layout != 1) return ALBERT_ERR_CONFIG;
    if (!(c->ln_eps >= 0.f)) return ALBERT_ERR_CONFIG;
    return ALBERT_OK;
}

// ---- per-kernel timing ----
int prof_harvest(albert_handle *h) {
    if (h->ev_used == 0) return ALBERT_OK;
    TRY(cudaEventSynchronize(h->ev[h->ev_used - 1]));
    for (int i = 0; i + 1 < h->ev_used; i += 2) {
        float ms = 0.f;
        TRY(cudaEventElapsedTime(&ms, h->ev[i], h->ev[i + 1]));
        h->prof_ms[h->ev_cls[i]] += ms;
        h->prof_launches[h->ev_cls[i]] += 1;
    }
    if (!h->prof_retain) h->ev_used = 0;
    return ALBERT_OK;
}

struct Launch {
    albert_handle *h;
    cudaStream_t s;
    int cls = -1;
    // Inside stream capture a plain event record only orders captured streams;
    // an external record becomes a graph node that records the event on replay.
    cudaError_t record(cudaEvent_t e) {
        cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
        cudaError_t err = cudaStreamIsCapturing(s, &cs);
        if (err != cudaSuccess) return err;
        return cudaEventRecordWithFlags(e, s, cs == cudaStreamCaptureStatusActive ? cudaEventRecordExternal
                                                                                    : cudaEventRecordDefault);
    }
    int begin(int c) {
        cls = c;
        h->prof_open = false;
        if (!(h->prof_mask >> c & 1u)) return ALBERT_OK;
        if (h->prof_count[c]++ % h->prof_stride != h->prof_offset) return ALBERT_OK;
        h->prof_open = true;
        if (h->ev_used + 2 > kEventPool) {
            if (h->prof_retain) return ALBERT_ERR_CONFIG;  // armed pairs cannot be recycled
            int rc = prof_harvest(h);
            if (rc) return rc;
        }
        h->ev_cls[h->ev_used] = c;
        TRY(record(h->ev[h->ev_used++]));
        return ALBERT_OK;
    }
    int end(cudaError_t launched) {
        if (launched == cudaSuccess) ++h->last_launches;
        if (launched != cudaSuccess) {
            if (getenv("ALBERT_DEBUG"))
                fprintf(stderr, "albert: launch of %s failed: %s\n", kProfNames[cls], cudaGetErrorString(launched));
            return ALBERT_ERR_CUDA;
        }
        if (!h->prof_open) return ALBERT_OK;
        h->ev_cls[h->ev_used] = cls;
        TRY(record(h->ev[h->ev_used++]));
        return ALBERT_OK;
    }
};

#define LAUNCH(L, cls, call)               \
    do {                                   \
        int rc_ = (L).begin(cls);          \
        if (rc_) return rc_;               \
        rc_ = (L).end(call);               \
        if (rc_) return rc_;               \
    } while (0)

GemmArgs gemm_args(albert_handle *h, int N, int K, const float *bias, void *out, int ld_out) {
    GemmArgs a{};
    a.N = N;
    a.K = K;
    a.rows_cap = h->rows_cap;
    a.n_rows = h->n_rows;
    a.bias = bias;
    a.out = static_cast<bf16 *>(out);
    a.ld_out = ld_out;
    a.row_dst = h->row_dst;
    a.status = h->status;
    a.eps = h->cfg.ln_eps;
    a.trigger = 1;  // inside a forward the next launch is one of ours with PDL
    a.wait_ns = h->wait_ns;
    return a;
}

int gemm_bf16(Launch &L, int cls, int epi, const CUtensorMap &A, const CUtensorMap &B, const CUtensorMap &Out,
              const CUtensorMap &Res, GemmArgs a) {
    const int grid = gemm_grid(epi, a.rows_cap, a.N, L.h->num_sms);
    a.withhold_loads = (L.h->stall_mask >> cls) & 1u;
    if (epi == kEpiResStats && a.N != gemm::LN_N) return ALBERT_ERR_CONFIG;
    if (!gemm_vectors_aligned(a)) return ALBERT_ERR_CONFIG;
    LAUNCH(L, cls, launch_gemm(epi, A, B, Out, Res, a, grid, L.h->num_sms, L.s));
    return ALBERT_OK;
}

GemmF32Args f32_args(albert_handle *h, const void *A, const void *W, const float *bias, void *out,
                     int ld_out, int N, int K) {
    GemmF32Args a{};
    a.A = static_cast<const float *>(A);
    a.W = static_cast<const float *>(W);
    a.bias = bias;
    a.out = static_cast<float *>(out);
    a.ld_out = ld_out;
    a.N = N;
    a.K = K;
    a.rows_cap = h->rows_cap;
    a.n_rows = h->n_rows;
    a.row_dst = h->row_dst;
    a.status = h->status;
    return a;
}

// Everything after the prep kernel; `padded_api` selects zero-filled padding rows.
int run_layers(albert_handle *h, Launch &L, const int64_t *ids, int ids_padded, int nseq, int T,
               int max_len, void *out, int padded_api, const float *emb_in = nullptr) {
    const albert_config &c = h->cfg;
    const int out_rows = padded_api ? nseq * T : c.max_tokens;
    // out_layout 1: the final stage writes token-major rows to the staging buffer,
    // which the last kernel transposes per sequence into the caller's output
    void *const user_out = out;
    if (padded_api && c.out_layout == 1) out = h->tout;
    const bool bf = c.dtype != ALBERT_FP32;  // bf16 activations (ALBERT_BF16 and ALBERT_FP8)
    const bool f8 = c.dtype == ALBERT_FP8;
    EmbedArgs ea{};
    ea.ids = ids;
    ea.ids_padded = ids_padded;
    ea.T = T;
    ea.seq_start = h->seq_start;
    ea.seq_len = h->seq_len;
    ea.nseq = nseq;
    ea.n_rows = h->n_rows;
    ea.rows_cap = h->rows_cap;
    ea.word = h->word;
    ea.pos = h->pos;
    ea.type = h->type;
    ea.g = h->emb_g;
    ea.b = h->emb_b;
    ea.eps = c.ln_eps;
    ea.vocab = c.vocab;
    ea.E = h->E;
    ea.out_f32 = bf ? 0 : 1;
    ea.row_dst = h->row_dst;
    ea.dst_padded = padded_api;
    ea.status = h->status;
    ea.trigger = bf ? 1 : 0;  // bf16: a kernel of ours (PDL) follows; fp32: a plain launch
    ea.emb_in = emb_in;

    const int D = out_width(h);
    // small batches: everything after the embedding in one kernel
    const long long row_bound = padded_api ? (long long)nseq * T : (long long)nseq * max_len;
    const bool small = bf && h->small_ok && h->small_enabled && row_bound <= kSmallMaxRows && max_len <= kAttnTcMaxLen;
    if (bf && !small) {
        // larger bf16 batches: the embedding and the input projection in one kernel
        LAUNCH(L, kProfEmbedProj, launch_embed_proj(h->tm_win, ea, h->b_in, static_cast<bf16 *>(h->X), h->num_sms,
                                                    L.s, h->wait_ns, (h->stall_mask >> kProfEmbedProj) & 1u));
    } else {
        LAUNCH(L, kProfEmbed, launch_embed(ea, L.s));
    }
    if (small) {
        const auto &W = h->grp[0];
        const auto &E1 = h->ex[c.n_exec > 1 ? 1 : 0];
        SmallFwdArgs s{};
        s.tmE = h->sm_E; s.tmX = h->sm_X; s.tmC = h->sm_C; s.tmX1 = h->sm_X1; s.tmZ = h->sm_Z; s.tmH = h->sm_H;
        s.tmQKV = h->tm_QKV; s.tmQKV64 = h->tm_QKV64;
        s.tmWin = h->sm_win; s.tmWqkv = h->sm_wqkv; s.tmWo = h->sm_wo; s.tmW1 = h->sm_w1; s.tmW2 = h->sm_w2;
        s.tmWout = c.out_dim > 0 ? h->sm_wout : h->sm_wo;  // (unused without a final projection)
        s.X = static_cast<bf16 *>(h->X); s.QKV = static_cast<bf16 *>(h->QKV); s.C = static_cast<bf16 *>(h->C);
        s.X1 = static_cast<bf16 *>(h->X1); s.Z = static_cast<bf16 *>(h->Z); s.H = static_cast<bf16 *>(h->H);
        s.st1 = h->sst1; s.st2 = h->sst2;
        s.b_in = h->b_in;
        s.bqkv0 = W.bqkv; s.bqkv = E1.c_qkv; s.s_qkv = E1.s_qkv;
        s.bo0 = W.bo; s.bo = E1.bias_o2;
        s.ln1_g = W.ln1_g; s.s_1 = W.s_1; s.c_1 = W.c_1; s.bias_21 = W.bias_21;
        s.ln2_g = W.ln2_g; s.ln2_b = W.ln2_b; s.s_out = h->s_out; s.c_out = h->c_out;
        s.out = static_cast<bf16 *>(out); s.out_dim = c.out_dim; s.row_dst = h->row_dst; s.out_rows = out_rows;
        s.seq_start = h->seq_start; s.seq_len = h->seq_len; s.nseq = nseq;
        s.n_rows = h->n_rows; s.status = h->status; s.bar = h->sbar;
        s.n_exec = c.n_exec; s.eps = c.ln_eps; s.wait_ns = h->wait_ns;
        s.withhold_loads = (h->stall_mask >> kProfSmall) & 1u;
        LAUNCH(L, kProfSmall, launch_forward_small(s, small_forward_grid(h->num_sms), L.s));
        if (padded_api && c.out_layout == 1)
            LAUNCH(L, kProfOutput, launch_transpose_out(h->tout, user_out, nseq, T, D, (int)elem_bytes(h), h->seq_len,
                                                        h->status, L.s));
        else if (padded_api)
            LAUNCH(L, kProfOutput, launch_zero_pad(out, nseq, T, D, (int)elem_bytes(h), h->seq_len, h->status, L.s));
        return ALBERT_OK;
    }
    if (bf) {
        int rc;
        for (int l = 0; l < c.n_exec; ++l) {
            const auto &W = h->grp[group_of(c, l)];                  // this execution's weights
            const auto &Wp = h->grp[group_of(c, l > 0 ? l - 1 : 0)];  // the previous execution's (its LN2)
            // ALBERT_FP8: a layer GEMM's A operand is first quantized per row (E4M3 codes
            // and scales in qA / sA); the GEMM reads the codes and the weights' codes.
            // The quantizer does not let the GEMM start early: resident GEMM CTAs
            // would hold the registers its warps need.
            auto e4m3_operand = [&](const void *A, int K, const float *ws, GemmArgs &ga) -> int {
                LAUNCH(L, kProfQuant, launch_quant_rows_e4m3(static_cast<const bf16 *>(A), K, h->rows_cap, h->n_rows,
                                                             h->qA, h->sA, h->status, L.s, true, false));
                ga.e4m3 = 1;
                ga.a_scale = h->sA;
                ga.w_scale = ws;
                return ALBERT_OK;
            };
            // Q|K|V from the layer input: X for the first execution, else LN2(z2) folded
            {
                GemmArgs a = gemm_args(h, kQKV, kHidden, l == 0 ? W.bqkv : h->ex[l].c_qkv, nullptr, 0);
                if (l > 0) {
                    a.fold_s = h->ex[l].s_qkv;
                    a.in_stats = h->st2;
                }
                const int epi = l == 0 ? kEpiBias : kEpiLnIn;
                if (f8) {
                    if ((rc = e4m3_operand(l == 0 ? h->X : h->Z, kHidden, W.s_wqkv, a))) return rc;
                    rc = gemm_bf16(L, kProfGemmQKV, epi, h->tq_A768, W.tq_wqkv, h->t32_QKV, h->t32_QKV, a);
                } else {
                    rc = gemm_bf16(L, kProfGemmQKV, epi, l == 0 ? h->tm_X : h->tm_Z, W.tm_wqkv, h->t32_QKV, h->t32_QKV, a);
                }
            }
            if (rc) return rc;
            if (max_len <= kAttnTcMaxLen) {
                LAUNCH(L, kProfAttention, launch_attention_tc(h->tm_QKV, h->tm_QKV64, static_cast<bf16 *>(h->C),
                                                             h->att_groups, h->n_att_groups, nseq, h->status,
                                                             h->num_sms, L.s, true, h->wait_ns));
            } else if (max_len <= kAttnTcLongMaxLen) {
                LAUNCH(L, kProfAttention, launch_attention_tc_long(h->tm_QKV, h->tm_QKV64, static_cast<bf16 *>(h->C), h->seq_start,
                                                                  h->seq_len, nseq, h->status, h->num_sms, L.s, true,
                                                                  h->wait_ns));
            } else {
                LAUNCH(L, kProfAttention, launch_attention_bf16(static_cast<bf16 *>(h->QKV), static_cast<bf16 *>(h->C),
                                                               h->seq_start, h->seq_len, nseq, max_len, h->status, L.s,
                                                               true));
            }
            // z1 = C Wo^T + bo + layer input -> X1 = z1 * gamma1, st1
            GemmArgs a = gemm_args(h, kHidden, kHidden, l == 0 ? W.bo : h->ex[l].bias_o2, nullptr, 0);
            a.res_stats = l == 0 ? nullptr : h->st2;
            a.res_g = Wp.ln2_g;
            a.out_g = W.ln1_g;
            a.out_stats = h->st1;
            if (f8 && (rc = e4m3_operand(h->C, kHidden, W.s_wo, a))) return rc;
            if ((rc = gemm_bf16(L, kProfGemmWoLN, kEpiResStats, f8 ? h->tq_A768 : h->tm_C, f8 ? W.tq_wo : W.tm_wo,
                                h->t32_X1, l == 0 ? h->t32_X : h->t32_Z, a)))
                return rc;
            // H = GELU(LN1(z1) W1^T + b1)
            a = gemm_args(h, kFfn, kHidden, W.c_1, nullptr, 0);
            a.fold_s = W.s_1;
            a.in_stats = h->st1;
            if (f8 && (rc = e4m3_operand(h->X1, kHidden, W.s_w1, a))) return rc;
            if ((rc = gemm_bf16(L, kProfGemmW1Gelu, kEpiLnInGelu, f8 ? h->tq_A768 : h->tm_X1, f8 ? W.tq_w1 : W.tm_w1,
                                h->t32_H, h->t32_H, a)))
                return rc;
            // z2 = H W2^T + b2 + LN1(z1) -> Z = z2 * gamma2, st2
            a = gemm_args(h, kHidden, kFfn, W.bias_21, nullptr, 0);
            a.res_stats = h->st1;
            a.res_g = W.ln1_g;
            a.out_g = W.ln2_g;
            a.out_stats = h->st2;
            if (f8 && (rc = e4m3_operand(h->H, kFfn, W.s_w2, a))) return rc;
            if ((rc = gemm_bf16(L, kProfGemmW2LN, kEpiResStats, f8 ? h->tq_A2048 : h->tm_H, f8 ? W.tq_w2 : W.tm_w2,
                                h->t32_Z, h->t32_X1, a)))
                return rc;
        }
        if (c.out_dim > 0) {
            // the final projection is followed by zero_pad only in the padded API
            if (c.n_exec == 0) {
                GemmArgs a = gemm_args(h, c.out_dim, kHidden, h->b_out, out, c.out_dim);
                a.trigger = padded_api;
                rc = gemm_bf16(L, kProfGemmOut, kEpiScatter, h->tm_X, h->tm_wout, h->t32_X, h->t32_X, a);
            } else {
                GemmArgs a = gemm_args(h, c.out_dim, kHidden, h->c_out, out, c.out_dim);
                a.trigger = padded_api;
                a.fold_s = h->s_out;
                a.in_stats = h->st2;
                rc = gemm_bf16(L, kProfGemmOut, kEpiLnInScatter, h->tm_Z, h->tm_wout, h->t32_X, h->t32_X, a);
            }
            if (rc) return rc;
        } else if (c.n_exec == 0) {
            LAUNCH(L, kProfOutput, launch_scatter_rows(h->X, out, kHidden, 2, h->rows_cap, h->n_rows, h->row_dst, h->status, L.s));
        } else {
            const auto &Wl = h->grp[group_of(c, c.n_exec - 1)];
            LAUNCH(L, kProfOutput, launch_ln_rows(static_cast<bf16 *>(h->Z), h->st2, Wl.ln2_g, Wl.ln2_b, c.ln_eps,
                                                  static_cast<bf16 *>(out), h->row_dst, out_rows, h->rows_cap, h->n_rows,
                                                  h->status, L.s));
        }
    } else {
        LAUNCH(L, kProfGemmIn, launch_gemm_f32(kF32Bias, f32_args(h, h->E, h->w_in, h->b_in, h->X, kHidden, kHidden, kEmb), L.s));
        for (int l = 0; l < c.n_exec; ++l) {
            const auto &W = h->grp[group_of(c, l)];
            LAUNCH(L, kProfGemmQKV, launch_gemm_f32(kF32Bias, f32_args(h, h->X, W.wqkv, W.bqkv, h->QKV, kQKV, kQKV, kHidden), L.s));
            LAUNCH(L, kProfAttention, launch_attention_f32(static_cast<float *>(h->QKV), static_cast<float *>(h->C), h->seq_start,
                                                          h->seq_len, nseq, max_len, h->status, L.s));
            GemmF32Args a = f32_args(h, h->C, W.wo, W.bo, h->Z, kHidden, kHidden, kHidden);
            a.resid = static_cast<float *>(h->X);
            LAUNCH(L, kProfGemmWoLN, launch_gemm_f32(kF32Resid, a, L.s));
            LAUNCH(L, kProfLayerNorm, launch_layer_norm_f32(static_cast<float *>(h->Z), static_cast<float *>(h->X1), W.ln1_g, W.ln1_b,
                                                           c.ln_eps, h->rows_cap, h->n_rows, h->status, L.s));
            LAUNCH(L, kProfGemmW1Gelu, launch_gemm_f32(kF32Gelu, f32_args(h, h->X1, W.w1, W.b1, h->H, kFfn, kFfn, kHidden), L.s));
            a = f32_args(h, h->H, W.w2, W.b2, h->Z, kHidden, kHidden, kFfn);
            a.resid = static_cast<float *>(h->X1);
            LAUNCH(L, kProfGemmW2LN, launch_gemm_f32(kF32Resid, a, L.s));
            LAUNCH(L, kProfLayerNorm, launch_layer_norm_f32(static_cast<float *>(h->Z), static_cast<float *>(h->X), W.ln2_g, W.ln2_b,
                                                           c.ln_eps, h->rows_cap, h->n_rows, h->status, L.s));
        }
        if (c.out_dim > 0) {
            LAUNCH(L, kProfGemmOut, launch_gemm_f32(kF32Scatter, f32_args(h, h->X, h->w_out, h->b_out, out, c.out_dim, c.out_dim, kHidden), L.s));
        } else {
            LAUNCH(L, kProfOutput, launch_scatter_rows(h->X, out, kHidden, 4, h->rows_cap, h->n_rows, h->row_dst, h->status, L.s));
        }
    }
    if (padded_api && c.out_layout == 1)
        LAUNCH(L, kProfOutput, launch_transpose_out(h->tout, user_out, nseq, T, D, (int)elem_bytes(h), h->seq_len,
                                                    h->status, L.s));
    else if (padded_api)
        LAUNCH(L, kProfOutput, launch_zero_pad(out, nseq, T, D, (int)elem_bytes(h), h->seq_len, h->status, L.s));
    return ALBERT_OK;
}

int copy_param(float *dst, const float *src, size_t n, cudaStream_t s) {
    if (!src) return ALBERT_ERR_NULL;
    TRY(cudaMemcpyAsync(dst, src, n * sizeof(float), cudaMemcpyDeviceToDevice, s));
    return ALBERT_OK;
}

int copy_matrix(albert_handle *h, void *dst, const float *src, size_t n, cudaStream_t s) {
    if (!src) return ALBERT_ERR_NULL;
    if (h->cfg.dtype != ALBERT_FP32) {
        TRY(launch_f32_to_bf16(src, static_cast<bf16 *>(dst), n, s));
    } else {
        TRY(cudaMemcpyAsync(dst, src, n * sizeof(float), cudaMemcpyDeviceToDevice, s));
    }
    return ALBERT_OK;
}

int create_impl(albert_handle *h, const albert_weights *w) {
    const albert_config &c = h->cfg;
    TRY(cudaGetDevice(&h->device));
    TRY(cudaDeviceGetAttribute(&h->num_sms, cudaDevAttrMultiProcessorCount, h->device));
    h->rows_cap = (c.max_tokens + 127) / 128 * 128;
    h->seq_cap = c.max_tokens;
    const size_t R = h->rows_cap;
    const bool bf = c.dtype != ALBERT_FP32;  // bf16 activations (ALBERT_BF16 and ALBERT_FP8)
    const bool f8 = c.dtype == ALBERT_FP8;
    const size_t eb = elem_bytes(h);
    int rc;
    cudaStream_t s = nullptr;
    TRY(cudaStreamCreateWithFlags(&s, cudaStreamNonBlocking));
    struct StreamGuard { cudaStream_t s; ~StreamGuard() { cudaStreamDestroy(s); } } guard{s};

    // ---- small fp32 parameters: one block (shared ones, then per group) ----
    const size_t V = c.vocab, P = c.max_pos, NT = c.n_types, O = c.out_dim, G = c.n_groups;
    auto sl = [](size_t n) { return (n + 63) / 64 * 64; };
    const size_t n_group_small = sl(kQKV) + sl(kHidden) + 2 * sl(kHidden) + sl(kFfn) + sl(kHidden) + 2 * sl(kHidden);
    const size_t n_small = sl(V * kEmb) + sl(P * kEmb) + sl(NT * kEmb) + 2 * sl(kEmb) + sl(kHidden) + sl(O) +
                           G * n_group_small;
    float *small = nullptr;
    if ((rc = dev_alloc(h, (void **)&small, n_small * sizeof(float)))) return rc;
    float *q = small;
    // slices start on 256-byte boundaries (kernels read several of them as float4)
    auto take = [&](size_t n) { float *r = q; q += (n + 63) / 64 * 64; return r; };
    h->word = take(V * kEmb); h->pos = take(P * kEmb); h->type = take(NT * kEmb);
    h->emb_g = take(kEmb); h->emb_b = take(kEmb); h->b_in = take(kHidden); h->b_out = take(O);
    if ((rc = copy_param(h->word, w->word, V * kEmb, s))) return rc;
    if ((rc = copy_param(h->pos, w->pos, P * kEmb, s))) return rc;
    if ((rc = copy_param(h->type, w->type, NT * kEmb, s))) return rc;
    if ((rc = copy_param(h->emb_g, w->emb_ln_g, kEmb, s))) return rc;
    if ((rc = copy_param(h->emb_b, w->emb_ln_b, kEmb, s))) return rc;
    if ((rc = copy_param(h->b_in, w->b_in, kHidden, s))) return rc;
    if (O && (rc = copy_param(h->b_out, w->b_out, O, s))) return rc;
    h->grp.assign(G, albert_handle::Group{});
    for (size_t g = 0; g < G; ++g) {
        auto &gp = h->grp[g];
        gp.bqkv = take(kQKV); gp.bo = take(kHidden); gp.ln1_g = take(kHidden); gp.ln1_b = take(kHidden);
        gp.b1 = take(kFfn); gp.b2 = take(kHidden); gp.ln2_g = take(kHidden); gp.ln2_b = take(kHidden);
        // group g's copy of each per-layer tensor follows group g-1's
        if ((rc = copy_param(gp.bqkv, w->bq + g * kHidden, kHidden, s))) return rc;
        if ((rc = copy_param(gp.bqkv + kHidden, w->bk + g * kHidden, kHidden, s))) return rc;
        if ((rc = copy_param(gp.bqkv + 2 * kHidden, w->bv + g * kHidden, kHidden, s))) return rc;
        if ((rc = copy_param(gp.bo, w->bo + g * kHidden, kHidden, s))) return rc;
        if ((rc = copy_param(gp.ln1_g, w->ln1_g + g * kHidden, kHidden, s))) return rc;
        if ((rc = copy_param(gp.ln1_b, w->ln1_b + g * kHidden, kHidden, s))) return rc;
        if ((rc = copy_param(gp.b1, w->b1 + g * kFfn, kFfn, s))) return rc;
        if ((rc = copy_param(gp.b2, w->b2 + g * kHidden, kHidden, s))) return rc;
        if ((rc = copy_param(gp.ln2_g, w->ln2_g + g * kHidden, kHidden, s))) return rc;
        if ((rc = copy_param(gp.ln2_b, w->ln2_b + g * kHidden, kHidden, s))) return rc;
    }

    // ---- matrices: one contiguous block (bf16 or fp32), 256-byte aligned pieces ----
    const size_t n_win = (size_t)kHidden * kEmb, n_qkv = (size_t)kQKV * kHidden, n_wo = (size_t)kHidden * kHidden;
    const size_t n_w1 = (size_t)kFfn * kHidden, n_w2 = (size_t)kHidden * kFfn, n_out = O * kHidden;
    auto al = [](size_t b) { return (b + 255) / 256 * 256; };
    const size_t group_bytes = al(n_qkv * eb) + al(n_wo * eb) + al(n_w1 * eb) + al(n_w2 * eb);
    const size_t off_groups = al(n_win * eb), off_out = off_groups + G * group_bytes;
    h->wblock_bytes = off_out + al(n_out * eb);
    if ((rc = dev_alloc(h, &h->wblock, h->wblock_bytes))) return rc;
    uint8_t *wb = static_cast<uint8_t *>(h->wblock);
    h->w_in = wb;
    h->w_out = wb + off_out;
    if ((rc = copy_matrix(h, h->w_in, w->w_in, n_win, s))) return rc;
    if (O && (rc = copy_matrix(h, h->w_out, w->w_out, n_out, s))) return rc;
    for (size_t g = 0; g < G; ++g) {
        auto &gp = h->grp[g];
        uint8_t *gb = wb + off_groups + g * group_bytes;
        gp.wqkv = gb;
        gp.wo = gb + al(n_qkv * eb);
        gp.w1 = static_cast<uint8_t *>(gp.wo) + al(n_wo * eb);
        gp.w2 = static_cast<uint8_t *>(gp.w1) + al(n_w1 * eb);
        if ((rc = copy_matrix(h, gp.wqkv, w->wq + g * n_wo, n_wo, s))) return rc;
        if ((rc = copy_matrix(h, static_cast<uint8_t *>(gp.wqkv) + n_wo * eb, w->wk + g * n_wo, n_wo, s))) return rc;
        if ((rc = copy_matrix(h, static_cast<uint8_t *>(gp.wqkv) + 2 * n_wo * eb, w->wv + g * n_wo, n_wo, s))) return rc;
        if ((rc = copy_matrix(h, gp.wo, w->wo + g * n_wo, n_wo, s))) return rc;
        if ((rc = copy_matrix(h, gp.w1, w->w1 + g * n_w1, n_w1, s))) return rc;
        if ((rc = copy_matrix(h, gp.w2, w->w2 + g * n_w2, n_w2, s))) return rc;
    }

    // ---- workspace ----
    if ((rc = dev_alloc(h, &h->E, R * kEmb * eb))) return rc;
    if ((rc = dev_alloc(h, &h->X, R * kHidden * eb))) return rc;
    if ((rc = dev_alloc(h, &h->QKV, R * kQKV * eb))) return rc;
    if ((rc = dev_alloc(h, &h->C, R * kHidden * eb))) return rc;
    if ((rc = dev_alloc(h, &h->X1, R * kHidden * eb))) return rc;
    if ((rc = dev_alloc(h, &h->H, R * kFfn * eb))) return rc;
    if ((rc = dev_alloc(h, &h->Z, R * kHidden * eb))) return rc;
    if (bf) {
        const size_t nst = R * gemm::LN_PARTS;
        if ((rc = dev_alloc(h, (void **)&h->st1, nst * sizeof(float2)))) return rc;
        if ((rc = dev_alloc(h, (void **)&h->st2, nst * sizeof(float2)))) return rc;
        TRY(cudaMemsetAsync(h->st1, 0, nst * sizeof(float2), s));
        TRY(cudaMemsetAsync(h->st2, 0, nst * sizeof(float2), s));
        // every vector starts on a 256-byte boundary: the epilogues read them as float4
        auto seg = [](size_t n) { return (n + 63) / 64 * 64; };
        const int NX = c.n_exec;
        const size_t nf = G * (seg(kFfn) * 2 + seg(kHidden)) + (size_t)NX * (2 * seg(kQKV) + seg(kHidden)) + 2 * seg(O);
        if ((rc = dev_alloc(h, (void **)&h->fold, nf * sizeof(float)))) return rc;
        float *f = h->fold;
        if (f8) {
            // E4M3 copies of the layer matrices (quantized from their bf16 copies) and the
            // A-operand buffer; the folded LayerNorm constants of these GEMMs are taken
            // from the E4M3 weights, so that the mean correction matches the product
            for (auto &gp : h->grp) {
                struct { uint8_t **q; float **sc; const void *w; int N, K; } mats[4] = {
                    {&gp.q_wqkv, &gp.s_wqkv, gp.wqkv, kQKV, kHidden}, {&gp.q_wo, &gp.s_wo, gp.wo, kHidden, kHidden},
                    {&gp.q_w1, &gp.s_w1, gp.w1, kFfn, kHidden}, {&gp.q_w2, &gp.s_w2, gp.w2, kHidden, kFfn}};
                for (auto &m : mats) {
                    if ((rc = dev_alloc(h, (void **)m.q, (size_t)m.N * m.K))) return rc;
                    if ((rc = dev_alloc(h, (void **)m.sc, (size_t)m.N * sizeof(float)))) return rc;
                    TRY(launch_quant_rows_e4m3(static_cast<const bf16 *>(m.w), m.K, m.N, nullptr, *m.q, *m.sc, nullptr,
                                               s, false, false));
                }
            }
            if ((rc = dev_alloc(h, (void **)&h->qA, R * kFfn))) return rc;
            if ((rc = dev_alloc(h, (void **)&h->sA, R * sizeof(float)))) return rc;
            TRY(cudaMemsetAsync(h->qA, 0, R * kFfn, s));
            TRY(cudaMemsetAsync(h->sA, 0, R * sizeof(float), s));
        }
        for (auto &gp : h->grp) {
            gp.s_1 = f; f += seg(kFfn); gp.c_1 = f; f += seg(kFfn); gp.bias_21 = f; f += seg(kHidden);
            if (f8)
                TRY(launch_fold_ln_e4m3(gp.q_w1, gp.s_w1, kFfn, kHidden, gp.ln1_g, gp.ln1_b, gp.b1, gp.s_1, gp.c_1, s));
            else
                TRY(launch_fold_ln(static_cast<const bf16 *>(gp.w1), kFfn, kHidden, gp.ln1_g, gp.ln1_b, gp.b1, gp.s_1,
                                   gp.c_1, s));
            TRY(launch_vec_add(gp.b2, gp.ln1_b, gp.bias_21, kHidden, s));
        }
        h->ex.assign(NX, albert_handle::Exec{});
        for (int l = 1; l < NX; ++l) {
            auto &e = h->ex[l];
            const auto &cur = h->grp[group_of(c, l)], &prev = h->grp[group_of(c, l - 1)];
            e.s_qkv = f; f += seg(kQKV); e.c_qkv = f; f += seg(kQKV); e.bias_o2 = f; f += seg(kHidden);
            if (f8)
                TRY(launch_fold_ln_e4m3(cur.q_wqkv, cur.s_wqkv, kQKV, kHidden, prev.ln2_g, prev.ln2_b, cur.bqkv,
                                        e.s_qkv, e.c_qkv, s));
            else
                TRY(launch_fold_ln(static_cast<const bf16 *>(cur.wqkv), kQKV, kHidden, prev.ln2_g, prev.ln2_b, cur.bqkv,
                                   e.s_qkv, e.c_qkv, s));
            TRY(launch_vec_add(cur.bo, prev.ln2_b, e.bias_o2, kHidden, s));
        }
        h->s_out = f; f += seg(O); h->c_out = f;
        if (O && NX > 0) {
            const auto &last = h->grp[group_of(c, NX - 1)];
            TRY(launch_fold_ln(static_cast<const bf16 *>(h->w_out), (int)O, kHidden, last.ln2_g, last.ln2_b, h->b_out,
                               h->s_out, h->c_out, s));
        }
    }
    if ((rc = dev_alloc(h, (void **)&h->seq_start, (h->seq_cap + 1) * sizeof(int)))) return rc;
    if ((rc = dev_alloc(h, (void **)&h->seq_len, (h->seq_cap + 1) * sizeof(int)))) return rc;
    if ((rc = dev_alloc(h, (void **)&h->row_dst, R * sizeof(int)))) return rc;
    if ((rc = dev_alloc(h, (void **)&h->n_rows, 4 * sizeof(int)))) return rc;
    h->status = h->n_rows + 1;
    h->n_att_groups = h->n_rows + 2;
    if ((rc = dev_alloc(h, (void **)&h->att_groups, (h->seq_cap + 1) * sizeof(int4)))) return rc;
    if ((rc = dev_alloc(h, (void **)&h->st_ids, (size_t)c.max_tokens * sizeof(int64_t)))) return rc;
    if ((rc = dev_alloc(h, (void **)&h->st_mask, (size_t)c.max_tokens))) return rc;
    if ((rc = dev_alloc(h, &h->st_out, (size_t)c.max_tokens * out_width(h) * eb))) return rc;
    if (c.out_layout == 1 && (rc = dev_alloc(h, &h->tout, (size_t)c.max_tokens * out_width(h) * eb))) return rc;
    // Deterministic contents for rows a forward never writes.
    for (void *p : {h->E, h->X, h->QKV, h->C, h->X1, h->H, h->Z}) {
        size_t bytes = (p == h->E ? kEmb : p == h->QKV ? kQKV : p == h->H ? kFfn : kHidden) * R * eb;
        TRY(cudaMemsetAsync(p, 0, bytes, s));
    }
    TRY(cudaMemsetAsync(h->n_rows, 0, 4 * sizeof(int), s));

    // ---- TMA descriptors ----
    if (bf) {
        if (make_tmap_bf16(&h->tm_E, h->E, R, kEmb, gemm::BM) || make_tmap_bf16(&h->tm_X, h->X, R, kHidden, gemm::BM) ||
            make_tmap_bf16(&h->tm_C, h->C, R, kHidden, gemm::BM) || make_tmap_bf16(&h->tm_X1, h->X1, R, kHidden, gemm::BM) ||
            make_tmap_bf16(&h->tm_H, h->H, R, kFfn, gemm::BM) || make_tmap_bf16(&h->tm_Z, h->Z, R, kHidden, gemm::BM) ||
            make_tmap_bf16(&h->tm_QKV, h->QKV, R, kQKV, 128) || make_tmap_bf16(&h->tm_QKV64, h->QKV, R, kQKV, 64) ||
            make_tmap_bf16(&h->tm_win, h->w_in, kHidden, kEmb, gemm::B_BOX) ||
            (O && make_tmap_bf16(&h->tm_wout, h->w_out, O, kHidden, gemm::B_BOX)) ||
            make_tmap_bf16_tile32(&h->t32_X, h->X, R, kHidden) || make_tmap_bf16_tile32(&h->t32_QKV, h->QKV, R, kQKV) ||
            make_tmap_bf16_tile32(&h->t32_X1, h->X1, R, kHidden) || make_tmap_bf16_tile32(&h->t32_H, h->H, R, kFfn) ||
            make_tmap_bf16_tile32(&h->t32_Z, h->Z, R, kHidden))
            return ALBERT_ERR_CUDA;
        for (auto &gp : h->grp)
            if (make_tmap_bf16(&gp.tm_wqkv, gp.wqkv, kQKV, kHidden, gemm::B_BOX) ||
                make_tmap_bf16(&gp.tm_wo, gp.wo, kHidden, kHidden, gemm::B_BOX) ||
                make_tmap_bf16(&gp.tm_w1, gp.w1, kFfn, kHidden, gemm::B_BOX) ||
                make_tmap_bf16(&gp.tm_w2, gp.w2, kHidden, kFfn, gemm::B_BOX))
                return ALBERT_ERR_CUDA;
        if (f8) {
            if (make_tmap_e4m3(&h->tq_A768, h->qA, R, kHidden, gemm::BM) ||
                make_tmap_e4m3(&h->tq_A2048, h->qA, R, kFfn, gemm::BM))
                return ALBERT_ERR_CUDA;
            for (auto &gp : h->grp)
                if (make_tmap_e4m3(&gp.tq_wqkv, gp.q_wqkv, kQKV, kHidden, gemm::B_BOX) ||
                    make_tmap_e4m3(&gp.tq_wo, gp.q_wo, kHidden, kHidden, gemm::B_BOX) ||
                    make_tmap_e4m3(&gp.tq_w1, gp.q_w1, kFfn, kHidden, gemm::B_BOX) ||
                    make_tmap_e4m3(&gp.tq_w2, gp.q_w2, kHidden, kFfn, gemm::B_BOX))
                    return ALBERT_ERR_CUDA;
        }
        // the small-batch kernel: bf16, one weight set, at least one execution
        if (!f8 && c.n_groups == 1 && c.n_exec >= 1) {
            const auto &gp = h->grp[0];
            if ((rc = dev_alloc(h, (void **)&h->sst1, kSmallMaxRows * kSmallParts * sizeof(float2)))) return rc;
            if ((rc = dev_alloc(h, (void **)&h->sst2, kSmallMaxRows * kSmallParts * sizeof(float2)))) return rc;
            if ((rc = dev_alloc(h, (void **)&h->sbar, sizeof(int)))) return rc;
            if (make_tmap_bf16(&h->sm_E, h->E, R, kEmb, 64) || make_tmap_bf16(&h->sm_X, h->X, R, kHidden, 64) ||
                make_tmap_bf16(&h->sm_C, h->C, R, kHidden, 64) || make_tmap_bf16(&h->sm_X1, h->X1, R, kHidden, 64) ||
                make_tmap_bf16(&h->sm_Z, h->Z, R, kHidden, 64) || make_tmap_bf16(&h->sm_H, h->H, R, kFfn, 64) ||
                make_tmap_bf16(&h->sm_win, h->w_in, kHidden, kEmb, 64) ||
                make_tmap_bf16(&h->sm_wqkv, gp.wqkv, kQKV, kHidden, 64) ||
                make_tmap_bf16(&h->sm_wo, gp.wo, kHidden, kHidden, 32) ||
                make_tmap_bf16(&h->sm_w1, gp.w1, kFfn, kHidden, 64) ||
                make_tmap_bf16(&h->sm_w2, gp.w2, kHidden, kFfn, 32) ||
                (O && make_tmap_bf16(&h->sm_wout, h->w_out, O, kHidden, 64)))
                return ALBERT_ERR_CUDA;
            h->small_ok = true;
        }
    }
    TRY(cudaStreamSynchronize(s));
    return ALBERT_OK;
}

void free_all(albert_handle *h) {
    for (cudaEvent_t e : h->ev) cudaEventDestroy(e);
    h->ev.clear();
    for (auto &sl : h->slot) {
        if (sl.d2h_done) cudaEventDestroy(sl.d2h_done);
        if (sl.fwd_done) cudaEventDestroy(sl.fwd_done);
        sl.d2h_done = sl.fwd_done = nullptr;
    }
    if (h->copy_stream) cudaStreamDestroy(h->copy_stream);
    h->copy_stream = nullptr;
    if (h->status_host) cudaFreeHost(h->status_host);
    h->status_host = nullptr;
    for (void *p : h->allocs) cudaFree(p);
    h->allocs.clear();
}

int forward_padded(albert_handle *h, const int64_t *ids, const uint8_t *mask, int B, int T, void *out,
                   cudaStream_t s) {
    h->last_launches = 0;
    Launch L{h, s};
    LAUNCH(L, kProfPrep, launch_prep_padded(mask, B, T, h->cfg.pack, h->cfg.max_tokens, h->seq_start, h->seq_len,
                                            h->n_rows, h->status, h->att_groups, h->n_att_groups, s, true));
    return run_layers(h, L, ids, 1, B, T, T, out, 1);
}

}  // namespace

extern "C" {

int albert_create(const albert_weights *w, const albert_config *cfg, albert_handle **out) {
    if (!out) return ALBERT_ERR_NULL;
    *out = nullptr;
    if (!w || !cfg) return ALBERT_ERR_NULL;
    int rc = check_config(cfg);
    if (rc) return rc;
    albert_handle *h = new (std::nothrow) albert_handle();
    if (!h) return ALBERT_ERR_ALLOC;
    h->cfg = *cfg;
    rc = create_impl(h, w);
    if (rc) {
        free_all(h);
        delete h;
        return rc;
    }
    *out = h;
    return ALBERT_OK;
}

int albert_forward(albert_handle *h, const int64_t *ids, const uint8_t *mask, int B, int T, void *out,
                   void *stream) {
    if (!h || !ids || !mask || !out) return ALBERT_ERR_NULL;
    if (B < 1 || T < 1 || T > h->cfg.max_pos || (long long)B * T > h->cfg.max_tokens) return ALBERT_ERR_SHAPE;
    return forward_padded(h, ids, mask, B, T, out, static_cast<cudaStream_t>(stream));
}

int albert_forward_varlen(albert_handle *h, const int64_t *ids, const int32_t *cu_seqlens, int nseq,
                          int max_len, void *out, void *stream) {
    if (!h || !ids || !cu_seqlens || !out) return ALBERT_ERR_NULL;
    if (nseq < 1 || nseq > h->seq_cap || max_len < 1 || max_len > h->cfg.max_pos) return ALBERT_ERR_SHAPE;
    if (h->cfg.out_layout != 0) return ALBERT_ERR_CONFIG;  // packed rows have no per-sequence [D, T] form
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    h->last_launches = 0;
    Launch L{h, s};
    LAUNCH(L, kProfPrep, launch_prep_varlen(cu_seqlens, nseq, max_len, h->cfg.max_tokens, h->seq_start, h->seq_len,
                                            h->n_rows, h->status, h->att_groups, h->n_att_groups, s, true));
    return run_layers(h, L, ids, 0, nseq, 0, max_len, out, 0);
}

int albert_forward_embedded(albert_handle *h, const float *emb, const int32_t *cu_seqlens, int nseq, int max_len,
                            void *out, void *stream) {
    if (!h || !emb || !cu_seqlens || !out) return ALBERT_ERR_NULL;
    if (nseq < 1 || nseq > h->seq_cap || max_len < 1 || max_len > h->cfg.max_pos) return ALBERT_ERR_SHAPE;
    if (h->cfg.out_layout != 0) return ALBERT_ERR_CONFIG;
    if (reinterpret_cast<uintptr_t>(emb) & 15) return ALBERT_ERR_CONFIG;  // rows are read as float4
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    h->last_launches = 0;
    Launch L{h, s};
    LAUNCH(L, kProfPrep, launch_prep_varlen(cu_seqlens, nseq, max_len, h->cfg.max_tokens, h->seq_start, h->seq_len,
                                            h->n_rows, h->status, h->att_groups, h->n_att_groups, s, true));
    return run_layers(h, L, nullptr, 0, nseq, 0, max_len, out, 0, emb);
}

int albert_forward_host(albert_handle *h, const int64_t *ids_host, const uint8_t *mask_host, int B, int T,
                        void *out_host, void *stream) {
    if (!h || !ids_host || !mask_host || !out_host) return ALBERT_ERR_NULL;
    if (B < 1 || T < 1 || T > h->cfg.max_pos || (long long)B * T > h->cfg.max_tokens) return ALBERT_ERR_SHAPE;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const size_t n = (size_t)B * T;
    TRY(cudaMemcpyAsync(h->st_ids, ids_host, n * sizeof(int64_t), cudaMemcpyHostToDevice, s));
    TRY(cudaMemcpyAsync(h->st_mask, mask_host, n, cudaMemcpyHostToDevice, s));
    int rc = forward_padded(h, h->st_ids, h->st_mask, B, T, h->st_out, s);
    if (rc) return rc;
    TRY(cudaMemcpyAsync(out_host, h->st_out, n * out_width(h) * elem_bytes(h), cudaMemcpyDeviceToHost, s));
    return albert_get_status(h, stream);
}

// Resources of the pipelined host path, made on first use.
static int async_setup(albert_handle *h) {
    if (h->copy_stream) return ALBERT_OK;
    const size_t n = (size_t)h->cfg.max_tokens;
    int rc;
    h->slot[0].ids = h->st_ids;
    h->slot[0].mask = h->st_mask;
    h->slot[0].out = h->st_out;
    if ((rc = dev_alloc(h, (void **)&h->slot[1].ids, n * sizeof(int64_t)))) return rc;
    if ((rc = dev_alloc(h, (void **)&h->slot[1].mask, n))) return rc;
    if ((rc = dev_alloc(h, &h->slot[1].out, n * out_width(h) * elem_bytes(h)))) return rc;
    for (auto &sl : h->slot) {
        if ((rc = dev_alloc(h, (void **)&sl.cu, ((size_t)h->seq_cap + 1) * sizeof(int32_t)))) return rc;
        TRY(cudaEventCreateWithFlags(&sl.d2h_done, cudaEventDisableTiming));
        TRY(cudaEventCreateWithFlags(&sl.fwd_done, cudaEventDisableTiming));
    }
    TRY(cudaHostAlloc(reinterpret_cast<void **>(&h->status_host), 2 * sizeof(int), cudaHostAllocDefault));
    TRY(cudaStreamCreateWithFlags(&h->copy_stream, cudaStreamNonBlocking));
    return ALBERT_OK;
}

// Wait for the batch in a slot to be complete on the host side; its status.
static int async_reap(albert_handle *h, int b) {
    auto &sl = h->slot[b];
    if (!sl.in_flight) return ALBERT_OK;
    TRY(cudaEventSynchronize(sl.d2h_done));
    sl.in_flight = false;
    return h->status_host[b];
}

int albert_forward_host_async(albert_handle *h, const int64_t *ids_host, const uint8_t *mask_host, int B, int T,
                              void *out_host, void *stream) {
    if (!h || !ids_host || !mask_host || !out_host) return ALBERT_ERR_NULL;
    if (B < 1 || T < 1 || T > h->cfg.max_pos || (long long)B * T > h->cfg.max_tokens) return ALBERT_ERR_SHAPE;
    int rc = async_setup(h);
    if (rc) return rc;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const int b = (int)(h->async_issued & 1);
    // the batch two calls back used this slot: its output must have reached the host
    const int prev = async_reap(h, b);
    auto &sl = h->slot[b];
    const size_t n = (size_t)B * T;
    TRY(cudaMemcpyAsync(sl.ids, ids_host, n * sizeof(int64_t), cudaMemcpyHostToDevice, s));
    TRY(cudaMemcpyAsync(sl.mask, mask_host, n, cudaMemcpyHostToDevice, s));
    if ((rc = forward_padded(h, sl.ids, sl.mask, B, T, sl.out, s))) return rc;
    // this batch's status, before the next forward's prep kernel resets the word
    TRY(cudaMemcpyAsync(h->status_host + b, h->status, sizeof(int), cudaMemcpyDeviceToHost, s));
    TRY(cudaEventRecord(sl.fwd_done, s));
    TRY(cudaStreamWaitEvent(h->copy_stream, sl.fwd_done, 0));
    TRY(cudaMemcpyAsync(out_host, sl.out, n * out_width(h) * elem_bytes(h), cudaMemcpyDeviceToHost, h->copy_stream));
    TRY(cudaEventRecord(sl.d2h_done, h->copy_stream));
    sl.in_flight = true;
    ++h->async_issued;
    return prev;
}

int albert_forward_varlen_host_async(albert_handle *h, const int64_t *ids_host, const int32_t *cu_seqlens_host,
                                     int nseq, int max_len, void *out_host, void *stream) {
    if (!h || !ids_host || !cu_seqlens_host || !out_host) return ALBERT_ERR_NULL;
    if (nseq < 1 || nseq > h->seq_cap || max_len < 1 || max_len > h->cfg.max_pos) return ALBERT_ERR_SHAPE;
    if (h->cfg.out_layout != 0) return ALBERT_ERR_CONFIG;
    // the copy sizes come from the host's cu_seqlens; the device checks the rest
    const long long n_tok = cu_seqlens_host[nseq];
    if (cu_seqlens_host[0] != 0 || n_tok < 1 || n_tok > h->cfg.max_tokens) return ALBERT_ERR_SHAPE;
    int rc = async_setup(h);
    if (rc) return rc;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const int b = (int)(h->async_issued & 1);
    const int prev = async_reap(h, b);
    auto &sl = h->slot[b];
    TRY(cudaMemcpyAsync(sl.ids, ids_host, (size_t)n_tok * sizeof(int64_t), cudaMemcpyHostToDevice, s));
    TRY(cudaMemcpyAsync(sl.cu, cu_seqlens_host, ((size_t)nseq + 1) * sizeof(int32_t), cudaMemcpyHostToDevice, s));
    if ((rc = albert_forward_varlen(h, sl.ids, sl.cu, nseq, max_len, sl.out, s))) return rc;
    TRY(cudaMemcpyAsync(h->status_host + b, h->status, sizeof(int), cudaMemcpyDeviceToHost, s));
    TRY(cudaEventRecord(sl.fwd_done, s));
    TRY(cudaStreamWaitEvent(h->copy_stream, sl.fwd_done, 0));
    TRY(cudaMemcpyAsync(out_host, sl.out, (size_t)n_tok * out_width(h) * elem_bytes(h), cudaMemcpyDeviceToHost,
                        h->copy_stream));
    TRY(cudaEventRecord(sl.d2h_done, h->copy_stream));
    sl.in_flight = true;
    ++h->async_issued;
    return prev;
}

int albert_forward_host_wait(albert_handle *h) {
    if (!h) return ALBERT_ERR_NULL;
    if (!h->copy_stream) return ALBERT_OK;
    const int b0 = (int)(h->async_issued & 1);  // the older batch first
    int first = ALBERT_OK;
    for (int i = 0; i < 2; ++i) {
        const int st = async_reap(h, b0 ^ i);
        if (first == ALBERT_OK) first = st;
    }
    return first;
}

int albert_get_status(albert_handle *h, void *stream) {
    if (!h) return ALBERT_ERR_NULL;
    TRY(cudaStreamSynchronize(static_cast<cudaStream_t>(stream)));
    int st = 0;
    TRY(cudaMemcpy(&st, h->status, sizeof(int), cudaMemcpyDeviceToHost));
    return st;
}

void albert_destroy(albert_handle *h) {
    if (!h) return;
    cudaDeviceSynchronize();
    free_all(h);
    delete h;
}

int albert_launches_per_forward(const albert_handle *h, int padded_api) {
    if (!h) return -1;
    const int per_layer = h->cfg.dtype == ALBERT_BF16 ? 5 : h->cfg.dtype == ALBERT_FP8 ? 9 : 7;
    return 1 /*prep*/ + 1 /*embed*/ + 1 /*in proj*/ + per_layer * h->cfg.n_exec + 1 /*final or scatter*/ +
           (padded_api ? 1 : 0);
}

int albert_profile_enable(albert_handle *h, int class_mask) {
    if (!h) return ALBERT_ERR_NULL;
    if (class_mask && h->ev.empty()) {
        h->ev.resize(kEventPool);
        h->ev_cls.assign(kEventPool, 0);
        for (auto &e : h->ev) TRY(cudaEventCreate(&e));
    }
    h->prof_mask = (unsigned)class_mask & ((1u << kProfClasses) - 1u);
    return ALBERT_OK;
}

int albert_profile_reset(albert_handle *h) {
    if (!h) return ALBERT_ERR_NULL;
    int rc = prof_harvest(h);
    for (int i = 0; i < kProfClasses; ++i) { h->prof_launches[i] = 0; h->prof_ms[i] = 0.0; }
    return rc;
}

int albert_profile_stride(albert_handle *h, int stride, int offset) {
    if (!h) return ALBERT_ERR_NULL;
    if (stride < 1 || offset < 0 || offset >= stride) return ALBERT_ERR_CONFIG;
    h->prof_stride = stride;
    h->prof_offset = offset;
    for (int &n : h->prof_count) n = 0;
    return ALBERT_OK;
}

int albert_profile_retain(albert_handle *h, int on) {
    if (!h) return ALBERT_ERR_NULL;
    h->prof_retain = on != 0;
    if (!h->prof_retain) h->ev_used = 0;
    return ALBERT_OK;
}

int albert_set_small_batch_kernel(albert_handle *h, int enable) {
    if (!h) return ALBERT_ERR_NULL;
    if (enable != 0 && enable != 1) return ALBERT_ERR_CONFIG;
    h->small_enabled = enable == 1;
    return ALBERT_OK;
}

int albert_last_forward_launches(const albert_handle *h) { return h ? h->last_launches : -1; }

int albert_set_wait_limit(albert_handle *h, long long ns) {
    if (!h) return ALBERT_ERR_NULL;
    if (ns < 0) return ALBERT_ERR_CONFIG;
    h->wait_ns = (unsigned long long)ns;
    return ALBERT_OK;
}

int albert_test_stall(albert_handle *h, int class_mask) {
    if (!h) return ALBERT_ERR_NULL;
    const unsigned gemm_classes = (1u << kProfGemmIn) | (1u << kProfGemmQKV) | (1u << kProfGemmWoLN) |
                                  (1u << kProfGemmW1Gelu) | (1u << kProfGemmW2LN) | (1u << kProfGemmOut) |
                                  (1u << kProfSmall) | (1u << kProfEmbedProj);
    if ((unsigned)class_mask & ~gemm_classes) return ALBERT_ERR_CONFIG;
    if (class_mask && h->cfg.dtype == ALBERT_FP32) return ALBERT_ERR_CONFIG;  // the fp32 kernels never wait
    h->stall_mask = (unsigned)class_mask;
    return ALBERT_OK;
}

int albert_profile_classes(void) { return kProfClasses; }

const char *albert_profile_name(int cls) { return (cls >= 0 && cls < kProfClasses) ? kProfNames[cls] : ""; }

int albert_profile_read(albert_handle *h, int *launches, double *ms) {
    if (!h || !launches || !ms) return ALBERT_ERR_NULL;
    int rc = prof_harvest(h);
    for (int i = 0; i < kProfClasses; ++i) { launches[i] = h->prof_launches[i]; ms[i] = h->prof_ms[i]; }
    return rc;
}

// ------------------------------------------------------ single-kernel entries --
int albert_test_gemm(const void *A, const void *W, const float *bias, const void *R, const float *ln_g,
                     const float *ln_b, float eps, const int32_t *row_dst, void *Y, int M, int N, int K,
                     int epi, void *stream) {
    if (!A || !W || !bias || !Y) return ALBERT_ERR_NULL;
    const bool e4m3 = (epi & ALBERT_GEMM_E4M3) != 0;
    if (M < 1 || N < gemm::BN || N % gemm::BN || K < gemm::BK || K % gemm::BK) return ALBERT_ERR_SHAPE;
    if (e4m3 && (K % 256 || K > 2048 || N % 8)) return ALBERT_ERR_SHAPE;  // the row quantizer's limits
    const int forced = (epi & ALBERT_GEMM_SINGLE_CTA ? 1 : 0) + (epi & ALBERT_GEMM_CTA_PAIR ? 1 : 0) +
                       (epi & ALBERT_GEMM_NARROW ? 1 : 0);
    if (forced > 1) return ALBERT_ERR_CONFIG;
    const int variant = (epi & ALBERT_GEMM_SINGLE_CTA) ? kGemmSingle : (epi & ALBERT_GEMM_CTA_PAIR) ? kGemmPair
                        : (epi & ALBERT_GEMM_NARROW) ? kGemmNarrow : kGemmAuto;
    epi &= ~(ALBERT_GEMM_SINGLE_CTA | ALBERT_GEMM_CTA_PAIR | ALBERT_GEMM_NARROW | ALBERT_GEMM_E4M3);
    if (epi < 0 || epi > 3) return ALBERT_ERR_CONFIG;
    if (epi == 2 && (!R || !ln_g || !ln_b || N != gemm::LN_N)) return ALBERT_ERR_CONFIG;
    if (epi == 3 && !row_dst) return ALBERT_ERR_NULL;
    if ((reinterpret_cast<uintptr_t>(bias) | reinterpret_cast<uintptr_t>(ln_g)) & 15) return ALBERT_ERR_CONFIG;
    const int kepi = epi == 0 ? kEpiBias : epi == 1 ? kEpiGelu : epi == 2 ? kEpiResStats : kEpiScatter;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    int dev = 0, sms = 0;
    TRY(cudaGetDevice(&dev));
    TRY(cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev));
    const int rows_cap = (M + gemm::BM - 1) / gemm::BM * gemm::BM;
    const int grid = gemm_grid(kepi, rows_cap, N, sms, variant);
    // epi 2 writes z * gamma and row statistics to temporaries, then normalizes them into Y
    int *ints = nullptr;
    void *zg = nullptr;
    float2 *stats = nullptr;
    TRY(cudaMalloc(&ints, 2 * sizeof(int)));
    if (epi == 2 && (cudaMalloc(&zg, (size_t)rows_cap * N * 2) != cudaSuccess ||
                     cudaMalloc(&stats, (size_t)rows_cap * gemm::LN_PARTS * sizeof(float2)) != cudaSuccess)) {
        cudaFree(ints);
        cudaFree(zg);
        return ALBERT_ERR_ALLOC;
    }
    // E4M3: both operands quantized per row into temporaries first
    uint8_t *qa = nullptr, *qw = nullptr;
    float *sa = nullptr, *sw = nullptr;
    if (e4m3) {
        if (cudaMalloc(&qa, (size_t)rows_cap * K) != cudaSuccess || cudaMalloc(&qw, (size_t)N * K) != cudaSuccess ||
            cudaMalloc(&sa, (size_t)rows_cap * sizeof(float)) != cudaSuccess ||
            cudaMalloc(&sw, (size_t)N * sizeof(float)) != cudaSuccess) {
            cudaFree(ints); cudaFree(zg); cudaFree(stats); cudaFree(qa); cudaFree(qw); cudaFree(sa);
            return ALBERT_ERR_ALLOC;
        }
    }
    CUtensorMap ta, tb, to, tr;
    int bad = e4m3 ? (make_tmap_e4m3(&ta, qa, M, K, gemm::BM) || make_tmap_e4m3(&tb, qw, N, K, gemm::B_BOX))
                   : (make_tmap_bf16(&ta, A, M, K, gemm::BM) || make_tmap_bf16(&tb, W, N, K, gemm::B_BOX));
    if (epi == 2) bad = bad || make_tmap_bf16_tile32(&to, zg, rows_cap, N) || make_tmap_bf16_tile32(&tr, R, M, N);
    else if (epi != 3) bad = bad || make_tmap_bf16_tile32(&to, Y, M, N);
    if (epi == 3) to = ta;
    if (epi != 2) tr = to;
    cudaError_t e = bad ? cudaErrorInvalidValue : cudaSuccess;
    const int host_ints[2] = {M, 0};
    if (e == cudaSuccess) e = cudaMemcpyAsync(ints, host_ints, sizeof(host_ints), cudaMemcpyHostToDevice, s);
    GemmArgs a{};
    a.N = N; a.K = K; a.rows_cap = rows_cap; a.n_rows = ints; a.bias = bias; a.eps = eps;
    a.out_g = ln_g; a.out_stats = stats; a.out = static_cast<bf16 *>(Y); a.ld_out = N;
    a.row_dst = row_dst; a.status = ints + 1;
    a.e4m3 = e4m3 ? 1 : 0; a.a_scale = sa; a.w_scale = sw;
    if (e == cudaSuccess && e4m3) {
        e = cudaMemsetAsync(sa, 0, (size_t)rows_cap * sizeof(float), s);
        if (e == cudaSuccess)
            e = launch_quant_rows_e4m3(static_cast<const bf16 *>(A), K, M, nullptr, qa, sa, nullptr, s, false, false);
        if (e == cudaSuccess)
            e = launch_quant_rows_e4m3(static_cast<const bf16 *>(W), K, N, nullptr, qw, sw, nullptr, s, false, false);
    }
    // follows a copy in the stream: a plain launch
    if (e == cudaSuccess) e = launch_gemm(kepi, ta, tb, to, tr, a, grid, sms, s, variant, false);
    if (e == cudaSuccess && epi == 2)
        e = launch_ln_rows(static_cast<const bf16 *>(zg), stats, ln_g, ln_b, eps, static_cast<bf16 *>(Y), nullptr, M,
                           rows_cap, ints, ints + 1, s);
    int st = 0;
    if (e == cudaSuccess) e = cudaMemcpyAsync(&st, ints + 1, sizeof(int), cudaMemcpyDeviceToHost, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    cudaFree(ints);
    if (zg) cudaFree(zg);
    if (stats) cudaFree(stats);
    if (qa) cudaFree(qa);
    if (qw) cudaFree(qw);
    if (sa) cudaFree(sa);
    if (sw) cudaFree(sw);
    return e == cudaSuccess ? st : ALBERT_ERR_CUDA;
}

int albert_test_quant_e4m3(const void *x, int rows, int K, void *q, float *scale, void *stream) {
    if (!x || !q || !scale) return ALBERT_ERR_NULL;
    if (rows < 1 || K < 256 || K > 2048 || K % 256) return ALBERT_ERR_SHAPE;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    TRY(launch_quant_rows_e4m3(static_cast<const bf16 *>(x), K, rows, nullptr, static_cast<uint8_t *>(q), scale,
                               nullptr, s, false, false));
    TRY(cudaStreamSynchronize(s));
    return ALBERT_OK;
}

int albert_test_attention(const void *qkv, const int32_t *cu_seqlens, int nseq, int max_len, void *ctx, int dtype,
                          void *stream) {
    if (!qkv || !cu_seqlens || !ctx) return ALBERT_ERR_NULL;
    if (nseq < 1 || max_len < 1 || max_len > kMaxPos) return ALBERT_ERR_SHAPE;
    if (dtype < 0 || dtype > 2) return ALBERT_ERR_CONFIG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    int dev = 0, sms = 0;
    TRY(cudaGetDevice(&dev));
    TRY(cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev));
    int n_tok = 0;
    TRY(cudaMemcpy(&n_tok, cu_seqlens + nseq, sizeof(int), cudaMemcpyDeviceToHost));
    if (n_tok < 1) return ALBERT_ERR_SHAPE;
    int *ints = nullptr;
    TRY(cudaMalloc(&ints, (6 * (size_t)nseq + 12) * sizeof(int)));
    int4 *groups = reinterpret_cast<int4 *>(ints);  // [nseq], first: 16-byte aligned
    int *seq_start = ints + 4 * (size_t)nseq, *seq_len = seq_start + nseq + 1, *n_rows = seq_len + nseq + 1;
    int *status = n_rows + 1, *n_groups = n_rows + 2;
    cudaError_t e = launch_prep_varlen(cu_seqlens, nseq, max_len, 1 << 30, seq_start, seq_len, n_rows, status, groups,
                                       n_groups, s, false);
    if (e == cudaSuccess) {
        if (dtype == ALBERT_FP32) {
            e = launch_attention_f32(static_cast<const float *>(qkv), static_cast<float *>(ctx), seq_start, seq_len, nseq,
                                     max_len, status, s);
        } else if (dtype == ALBERT_BF16 && max_len <= kAttnTcLongMaxLen) {
            CUtensorMap tm, tm64;
            if (make_tmap_bf16(&tm, qkv, (uint64_t)n_tok, kQKV, 128) || make_tmap_bf16(&tm64, qkv, (uint64_t)n_tok, kQKV, 64))
                e = cudaErrorInvalidValue;
            else if (max_len <= kAttnTcMaxLen)
                e = launch_attention_tc(tm, tm64, static_cast<bf16 *>(ctx), groups, n_groups, nseq, status, sms, s,
                                        false);
            else
                e = launch_attention_tc_long(tm, tm64, static_cast<bf16 *>(ctx), seq_start, seq_len, nseq, status, sms, s,
                                             false);
        } else {
            e = launch_attention_bf16(static_cast<const bf16 *>(qkv), static_cast<bf16 *>(ctx), seq_start, seq_len, nseq,
                                      max_len, status, s, false);
        }
    }
    int st = 0;
    if (e == cudaSuccess) e = cudaMemcpyAsync(&st, status, sizeof(int), cudaMemcpyDeviceToHost, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    cudaFree(ints);
    return e == cudaSuccess ? st : ALBERT_ERR_CUDA;
}

int albert_test_attention_groups(const int32_t *cu_seqlens, int nseq, int max_len, int32_t *groups_out, int *n_out,
                                 void *stream) {
    if (!cu_seqlens || !groups_out || !n_out) return ALBERT_ERR_NULL;
    if (nseq < 1 || max_len < 1 || max_len > kMaxPos) return ALBERT_ERR_SHAPE;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    int *ints = nullptr;
    TRY(cudaMalloc(&ints, (6 * (size_t)nseq + 12) * sizeof(int)));
    int4 *groups = reinterpret_cast<int4 *>(ints);  // [nseq], first: 16-byte aligned
    int *seq_start = ints + 4 * (size_t)nseq, *seq_len = seq_start + nseq + 1, *n_rows = seq_len + nseq + 1;
    int *status = n_rows + 1, *n_groups = n_rows + 2;
    int host[2] = {0, 0};
    cudaError_t e = launch_prep_varlen(cu_seqlens, nseq, max_len, 1 << 30, seq_start, seq_len, n_rows, status, groups,
                                       n_groups, s, false);
    if (e == cudaSuccess) e = cudaMemcpyAsync(host, status, 2 * sizeof(int), cudaMemcpyDeviceToHost, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    const int ng = host[1];
    if (e == cudaSuccess && host[0] == 0 && ng >= 0 && ng <= nseq)
        e = cudaMemcpy(groups_out, groups, (size_t)ng * sizeof(int4), cudaMemcpyDeviceToHost);
    cudaFree(ints);
    if (e != cudaSuccess) return ALBERT_ERR_CUDA;
    if (host[0] != 0) return host[0];
    if (ng < 0 || ng > nseq) return ALBERT_ERR_CUDA;
    *n_out = ng;
    return ALBERT_OK;
}

}  // extern "C"
