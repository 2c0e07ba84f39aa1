/*
 * TEST INFRASTRUCTURE -- plain fp64 CPU oracle of Kokoro's ALBERT phoneme encoder.
 *
 * Only the test suite, the package smoke check and the benchmark's CPU-baseline
 * leg may load this library.  It shares no code, header, table or helper with the
 * CUDA path; the two meet only through the seeded input generators.
 *
 * What it computes, and where each step is defined:
 *   "ALBERT: How Kokoro's Phoneme Encoder Works, and Where CKE Has Reached It"
 *     (shivasnotes), section "Inside One Real ALBERT Layer", steps 1-6 and the
 *     paragraph after them (shared layer run 12 times, final [T,512] projection);
 *     section "1. Factorized embedding" (table sizes);
 *     section "How CKE Represents It" (LayerNorm epsilon 1e-12, tanh-form GELU,
 *     additive mask semantics, 12 heads of 64, 128->768 projection).
 *   "How Kokoro TTS Works and Where CKE Stands", section "What ALBERT does here"
 *     (softmax(Q K^T / sqrt(d) + mask) V).
 *   "Qwen3-TTS and Kokoro", section "A. A projection is a dot product with an
 *     optional bias" (y_j = b_j + sum_i x_i W_{j,i}, fp64 sum in ascending index
 *     order) and section "D. Attention is two matrix products with a softmax
 *     between" (max-subtracted softmax; here without the causal restriction,
 *     since the encoder is bidirectional).
 *   "Kokoro-82M-encoder-hailo10h" model card, section "How to recompile from
 *     scratch" step 3 (the GELU is the tanh approximation with a cubic term).
 *
 * Readings where the pages are silent (each is also listed in the design notes):
 *   - LayerNorm is the textbook one: biased variance, eps inside the square root,
 *     per-channel gamma/beta;
 *   - post-LN: LN(x + sublayer(x));
 *   - GELU(x) = 0.5 x (1 + tanh(sqrt(2/pi) (x + 0.044715 x^3)));
 *   - the key-padding mask adds -infinity, i.e. masked keys get weight exactly 0;
 *   - head h = columns 64h..64h+63 of Q, K, V and of the context;
 *   - positions are the slot index 0..T-1 (right padding), token type 0;
 *   - all linears are biased.
 *
 * Activations stay in fp64 throughout; every dot product is summed in fp64 in
 * ascending index order.  OpenMP only splits independent output elements across
 * threads, so results do not depend on the thread count.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

typedef struct {
    int vocab, emb, hidden, heads, ffn, n_exec, max_pos, n_types, out_dim;
    double ln_eps;
} orc_cfg;

/* Parameters in [out, in] layout, fp64. */
typedef struct {
    const double *word, *pos, *type, *emb_ln_g, *emb_ln_b;
    const double *w_in, *b_in;
    const double *wq, *bq, *wk, *bk, *wv, *bv;
    const double *wo, *bo, *ln1_g, *ln1_b;
    const double *w1, *b1, *w2, *b2, *ln2_g, *ln2_b;
    const double *w_out, *b_out;
} orc_weights;

int orc_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

void orc_set_threads(int n) {
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}

/* Linear layer, "Qwen3-TTS and Kokoro" section A:
 *   y[t][j] = b[j] + sum_{i=0..in-1} x[t][i] * W[j][i],  i ascending, fp64.
 * b may be NULL (no bias). */
void orc_linear(const double *x, int rows, int in, const double *W, const double *b,
                int out, double *y) {
    long n = (long)rows * out;
#pragma omp parallel for schedule(static)
    for (long idx = 0; idx < n; ++idx) {
        int t = (int)(idx / out), j = (int)(idx % out);
        const double *xr = x + (long)t * in, *wr = W + (long)j * in;
        double s = b ? b[j] : 0.0;
        for (int i = 0; i < in; ++i) s += xr[i] * wr[i];
        y[idx] = s;
    }
}

/* LayerNorm over the last axis of length n (textbook form):
 *   mu = (1/n) sum x,  var = (1/n) sum (x - mu)^2,
 *   y = (x - mu) / sqrt(var + eps) * g + b. */
void orc_layer_norm(const double *x, int rows, int n, const double *g, const double *b,
                    double eps, double *y) {
#pragma omp parallel for schedule(static)
    for (int t = 0; t < rows; ++t) {
        const double *xr = x + (long)t * n;
        double *yr = y + (long)t * n;
        double mu = 0.0;
        for (int i = 0; i < n; ++i) mu += xr[i];
        mu /= n;
        double var = 0.0;
        for (int i = 0; i < n; ++i) var += (xr[i] - mu) * (xr[i] - mu);
        var /= n;
        double inv = 1.0 / sqrt(var + eps);
        for (int i = 0; i < n; ++i) yr[i] = (xr[i] - mu) * inv * g[i] + b[i];
    }
}

/* tanh-approximation GELU (Hendrycks & Gimpel), the variant with a cubic term. */
double orc_gelu_tanh(double x) {
    const double c = sqrt(2.0 / M_PI);
    return 0.5 * x * (1.0 + tanh(c * (x + 0.044715 * x * x * x)));
}

void orc_gelu_rows(const double *x, long n, double *y) {
#pragma omp parallel for schedule(static)
    for (long i = 0; i < n; ++i) y[i] = orc_gelu_tanh(x[i]);
}

/* Bidirectional multi-head attention with a key-padding mask, per head h:
 *   s[t][u] = q_h[t] . k_h[u] / sqrt(dh)  for keys u with key_mask[u] != 0,
 *   p[t][u] = exp(s[t][u] - max_u s[t][u]) / sum_u exp(s[t][u] - max_u s[t][u]),
 *   ctx_h[t] = sum_u p[t][u] v_h[u];
 * masked keys (key_mask[u] == 0) carry weight exactly 0 (additive -infinity).
 * q, k, v, ctx are [T, heads*dh] with row stride ld_in / ld_out; head h is the
 * column slice h*dh .. h*dh+dh-1.  Every query row (valid or not) attends to the
 * valid keys.  Returns -1 if no key is valid. */
int orc_attention(const double *q, const double *k, const double *v, int ld_in,
                  const uint8_t *key_mask, int T, int heads, int dh,
                  double *ctx, int ld_out) {
    int any = 0;
    for (int u = 0; u < T; ++u) any |= key_mask[u] != 0;
    if (!any) return -1;
    const double scale = 1.0 / sqrt((double)dh);
#pragma omp parallel
    {
        double *s = (double *)malloc(sizeof(double) * (size_t)T);
#pragma omp for schedule(static) collapse(2)
        for (int h = 0; h < heads; ++h) {
            for (int t = 0; t < T; ++t) {
                const double *qt = q + (long)t * ld_in + h * dh;
                double m = -INFINITY;
                for (int u = 0; u < T; ++u) {
                    if (!key_mask[u]) continue;
                    const double *ku = k + (long)u * ld_in + h * dh;
                    double d = 0.0;
                    for (int i = 0; i < dh; ++i) d += qt[i] * ku[i];
                    s[u] = d * scale;
                    if (s[u] > m) m = s[u];
                }
                double den = 0.0;
                for (int u = 0; u < T; ++u) {
                    if (!key_mask[u]) continue;
                    s[u] = exp(s[u] - m);
                    den += s[u];
                }
                double *ct = ctx + (long)t * ld_out + h * dh;
                for (int i = 0; i < dh; ++i) {
                    double acc = 0.0;
                    for (int u = 0; u < T; ++u) {
                        if (!key_mask[u]) continue;
                        acc += (s[u] / den) * v[(long)u * ld_in + h * dh + i];
                    }
                    ct[i] = acc;
                }
            }
        }
        free(s);
    }
    return 0;
}

/* Three-table embedding + LayerNorm at width E (page 1, step 1):
 *   e[t] = word[ids[t]] + pos[t] + type[0];  out[t] = LN_E(e[t]).
 * Returns -1 on an id outside [0, vocab) at a slot whose mask is set. */
int orc_embed(const orc_cfg *c, const orc_weights *w, const int64_t *ids,
              const uint8_t *mask, int T, double *out) {
    const int E = c->emb;
    if (T > c->max_pos) return -1;
    double *e = (double *)malloc(sizeof(double) * (size_t)T * E);
    for (int t = 0; t < T; ++t) {
        int64_t id = ids[t];
        if (id < 0 || id >= c->vocab) {
            if (mask[t]) { free(e); return -1; }
            id = 0; /* padding slot: any id; its row never reaches a valid output */
        }
        for (int i = 0; i < E; ++i)
            e[(long)t * E + i] = w->word[id * E + i] + w->pos[(long)t * E + i] + w->type[i];
    }
    orc_layer_norm(e, T, E, w->emb_ln_g, w->emb_ln_b, c->ln_eps, out);
    free(e);
    return 0;
}

/* One execution of the shared layer (page 1, steps 3-6), post-LN:
 *   q,k,v = x Wq^T + bq, ...;  c = MHA(q, k, v; mask);
 *   x1 = LN(x + c Wo^T + bo; ln1);
 *   x  = LN(x1 + GELU(x1 W1^T + b1) W2^T + b2; ln2).
 * x is [T, H] and is updated in place. */
int orc_layer(const orc_cfg *c, const orc_weights *w, double *x, const uint8_t *mask, int T) {
    const int H = c->hidden, F = c->ffn, NH = c->heads, DH = c->hidden / c->heads;
    size_t TH = (size_t)T * H;
    double *q = (double *)malloc(sizeof(double) * TH);
    double *k = (double *)malloc(sizeof(double) * TH);
    double *v = (double *)malloc(sizeof(double) * TH);
    double *ctx = (double *)malloc(sizeof(double) * TH);
    double *tmp = (double *)malloc(sizeof(double) * TH);
    double *x1 = (double *)malloc(sizeof(double) * TH);
    double *g = (double *)malloc(sizeof(double) * (size_t)T * F);
    int rc = 0;

    orc_linear(x, T, H, w->wq, w->bq, H, q);
    orc_linear(x, T, H, w->wk, w->bk, H, k);
    orc_linear(x, T, H, w->wv, w->bv, H, v);
    rc = orc_attention(q, k, v, H, mask, T, NH, DH, ctx, H);
    if (rc == 0) {
        orc_linear(ctx, T, H, w->wo, w->bo, H, tmp);
        for (size_t i = 0; i < TH; ++i) tmp[i] += x[i];                 /* residual */
        orc_layer_norm(tmp, T, H, w->ln1_g, w->ln1_b, c->ln_eps, x1);
        orc_linear(x1, T, H, w->w1, w->b1, F, g);
        orc_gelu_rows(g, (long)T * F, g);
        orc_linear(g, T, F, w->w2, w->b2, H, tmp);
        for (size_t i = 0; i < TH; ++i) tmp[i] += x1[i];                /* residual */
        orc_layer_norm(tmp, T, H, w->ln2_g, w->ln2_b, c->ln_eps, x);
    }
    free(q); free(k); free(v); free(ctx); free(tmp); free(x1); free(g);
    return rc;
}

/* Whole encoder for one sequence of T slots with key-padding mask:
 *   E = LN(embed);  x = E W_in^T + b_in;  repeat n_exec times x = layer(x);
 *   out = x W_out^T + b_out  if out_dim > 0, else out = x.
 * out is [T, out_dim or hidden]; rows at masked slots are computed but are not
 * part of the result. */
int orc_encode(const orc_cfg *c, const orc_weights *w, const int64_t *ids,
               const uint8_t *mask, int T, double *out) {
    const int E = c->emb, H = c->hidden;
    double *e = (double *)malloc(sizeof(double) * (size_t)T * E);
    double *x = (double *)malloc(sizeof(double) * (size_t)T * H);
    int rc = orc_embed(c, w, ids, mask, T, e);
    if (rc == 0) {
        orc_linear(e, T, E, w->w_in, w->b_in, H, x);
        for (int l = 0; l < c->n_exec && rc == 0; ++l) rc = orc_layer(c, w, x, mask, T);
        if (rc == 0) {
            if (c->out_dim > 0)
                orc_linear(x, T, H, w->w_out, w->b_out, c->out_dim, out);
            else
                memcpy(out, x, sizeof(double) * (size_t)T * H);
        }
    }
    free(e); free(x);
    return rc;
}

/* A batch of B independent sequences of T slots each (ids, mask: [B, T]). */
int orc_encode_batch(const orc_cfg *c, const orc_weights *w, const int64_t *ids,
                     const uint8_t *mask, int B, int T, double *out) {
    const int D = c->out_dim > 0 ? c->out_dim : c->hidden;
    for (int b = 0; b < B; ++b) {
        int rc = orc_encode(c, w, ids + (long)b * T, mask + (long)b * T, T,
                            out + (long)b * T * D);
        if (rc) return rc;
    }
    return 0;
}
