/*
 * Plain CPU oracle for the Orthrus dual-view decode step.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the
 * benchmark's CPU-baseline leg load this library.  The CUDA product path
 * shares no code with it.
 *
 * Source: "Orthrus: Memory-Efficient Parallel Token Generation via Dual-View
 * Diffusion" as described by the paper-notes page (zhangshuibai.github.io,
 * spec-rl note 17): §2.1 (dual-view layer: per-layer extra W_Q/W_K/W_V, shared
 * LM head, frozen backbone), §2.2-2.3 (one shared AR-only KV cache, transient
 * diffusion K/V), §3.2 (diffusion-view mask: committed prefix before the
 * anchor plus bidirectional attention inside the block), §4.1 (the cycle:
 * parallel projection, AR verification, consensus and cache truncation),
 * §4.2 (greedy consensus), §4.3 (rejection sampling at T>0).  The
 * hotdry.top engineering page ("推理机制") restates the same cycle.  The
 * training-side pieces follow §3.1-3.3 of the paper-notes page (packed
 * sequences of anchor blocks, the dual-pass block mask, forward KL against
 * the frozen AR view) and the hotdry.top page's training section
 * ("训练策略：双通块掩码与前向 KL 蒸馏").  Tree verification follows the
 * paper-notes page's §7.5 (DDTree: a best-first tree of the top prefixes of
 * one diffusion forward's marginals, verified by one tree-attention pass)
 * and §9.6 (the same proposed for Orthrus's K marginals); greedy only.
 *
 * Arithmetic is fp64 throughout.  Weights arrive as fp32 arrays holding the
 * exact model values (bf16 values are exactly representable in fp32).  Every
 * output element is computed by one loop in ascending index order, so a row
 * of a block gives bit-for-bit the value that the same row gives alone.
 *
 * Readings where the pages are silent (each restated in the design notes):
 *   - pre-norm decoder, RMSNorm eps 1e-6, no biases, no QK-norm, SwiGLU FFN
 *     down(silu(gate a) * up a), rotate-half RoPE with inv_freq_i =
 *     theta^(-2i/hd), attention scale 1/sqrt(hd), GQA head h -> kv head
 *     h / (n_q / n_kv);
 *   - the cache holds x_<t; the anchor's K/V come from the block;
 *   - block row k (0-based) sits at position t+k and predicts position t+k+1;
 *   - the verify input is [x_t, y_1 .. y_{K-1}], no bonus token, n in [1, K];
 *   - ties in argmax go to the lowest index;
 *   - sampling at T>0 is Gumbel-max over Philox4x32-10 uniforms keyed by
 *     (seed, step, row, id, purpose); acceptance is u < p/q; the residual is
 *     max(0, p - q) renormalised, falling back to argmax p if it has no mass.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define OC_OK 0
#define OC_ERR_ARG 1
#define OC_ERR_NOMEM 2
#define OC_ERR_CAPACITY 3

enum { OC_PURPOSE_DRAFT = 1, OC_PURPOSE_ACCEPT = 2, OC_PURPOSE_RESIDUAL = 3, OC_PURPOSE_AR = 4 };

typedef struct {
    int n_layers, hidden, n_q_heads, n_kv_heads, head_dim, ffn, vocab, mask_id;
    double rope_theta, rms_eps;
} oc_cfg;

typedef struct {
    const float *attn_norm, *wq, *wk, *wv, *wq_diff, *wk_diff, *wv_diff;
    const float *wo, *ffn_norm, *w_gate, *w_up, *w_down;
} oc_layer;

typedef struct {
    const float *embed, *final_norm, *lm_head;
    const oc_layer *layers;
} oc_model;

/* ------------------------------------------------------------------------ */
/* Building blocks of the frozen backbone (paper notes §2.1: everything but   */
/* W_Q/W_K/W_V is the unchanged pre-trained layer).                           */
/* ------------------------------------------------------------------------ */

/* y = x / sqrt(mean(x^2) + eps) * gain */
void oc_rmsnorm(const double *x, const float *gain, int n, double eps, double *y)
{
    double ss = 0.0;
    for (int i = 0; i < n; ++i) ss += x[i] * x[i];
    double inv = 1.0 / sqrt(ss / n + eps);
    for (int i = 0; i < n; ++i) y[i] = x[i] * inv * (double)gain[i];
}

/* y[r][o] = sum_i x[r][i] * W[o][i]   (W row-major [out][in]) */
void oc_linear(const double *x, int R, int in, const float *W, int out, double *y)
{
    #pragma omp parallel for schedule(static) collapse(2) if ((long)R * out * in > 2000000)
    for (int r = 0; r < R; ++r)
        for (int o = 0; o < out; ++o) {
            const double *xr = x + (size_t)r * in;
            const float *w = W + (size_t)o * in;
            double s = 0.0;
            for (int i = 0; i < in; ++i) s += xr[i] * (double)w[i];
            y[(size_t)r * out + o] = s;
        }
}

/* Rotate-half rotary embedding of n_heads vectors of length hd at `pos`:
 * pairs (i, i + hd/2) rotate by pos * theta^(-2i/hd). */
void oc_rope(double *x, int n_heads, int hd, int pos, double theta)
{
    int half = hd / 2;
    for (int i = 0; i < half; ++i) {
        double inv_freq = pow(theta, -2.0 * i / hd);
        double ang = (double)pos * inv_freq;
        double c = cos(ang), s = sin(ang);
        for (int h = 0; h < n_heads; ++h) {
            double *v = x + (size_t)h * hd;
            double a = v[i], b = v[i + half];
            v[i] = a * c - b * s;
            v[i + half] = b * c + a * s;
        }
    }
}

double oc_silu(double g) { return g / (1.0 + exp(-g)); }

/*
 * Dual-view attention for a block of R query rows at positions t .. t+R-1.
 *   q      [R][n_q][hd]
 *   kc, vc [>= t][n_kv][hd]  committed cache rows 0 .. t-1
 *   kb, vb [R][n_kv][hd]     the block's own K/V
 *   mode 0 (AR verify / prefill, paper notes §4.1 step 2): row r sees cache
 *          rows [0, t) and block rows 0 .. r (causal);
 *   mode 1 (diffusion draft, paper notes §3.2): row r sees cache rows [0, t)
 *          and every block row (bidirectional inside the block).
 *   o      [R][n_q][hd]
 */
void oc_attention(const double *q, int R, int n_q, int n_kv, int hd,
                  const double *kc, const double *vc, int t,
                  const double *kb, const double *vb, int mode, double *o)
{
    int g = n_q / n_kv;
    double scale = 1.0 / sqrt((double)hd);
    #pragma omp parallel for schedule(static) collapse(2) if ((long)R * n_q * (t + R) * hd > 1000000)
    for (int r = 0; r < R; ++r)
        for (int h = 0; h < n_q; ++h) {
            int kvh = h / g;
            int nblk = (mode == 0) ? r + 1 : R;
            int nkeys = t + nblk;
            const double *qv = q + ((size_t)r * n_q + h) * hd;
            double *s = (double *)malloc(sizeof(double) * (size_t)(nkeys > 0 ? nkeys : 1));
            double m = -INFINITY;
            for (int j = 0; j < nkeys; ++j) {
                const double *kv = (j < t) ? kc + ((size_t)j * n_kv + kvh) * hd
                                           : kb + ((size_t)(j - t) * n_kv + kvh) * hd;
                double d = 0.0;
                for (int i = 0; i < hd; ++i) d += qv[i] * kv[i];
                s[j] = d * scale;
                if (s[j] > m) m = s[j];
            }
            double l = 0.0;
            for (int j = 0; j < nkeys; ++j) { s[j] = exp(s[j] - m); l += s[j]; }
            double *ov = o + ((size_t)r * n_q + h) * hd;
            for (int i = 0; i < hd; ++i) ov[i] = 0.0;
            for (int j = 0; j < nkeys; ++j) {
                const double *vv = (j < t) ? vc + ((size_t)j * n_kv + kvh) * hd
                                           : vb + ((size_t)(j - t) * n_kv + kvh) * hd;
                double p = s[j] / l;
                for (int i = 0; i < hd; ++i) ov[i] += p * vv[i];
            }
            free(s);
        }
}

/*
 * Tree-masked attention for the verification of a draft tree (the DDTree
 * comparison of the paper-notes page, §7.5, and its suggestion in §9.6: one
 * diffusion forward's marginals expanded best-first into a tree that one AR
 * forward verifies with a tree mask).  Block row r is a tree node; parent[r]
 * is its parent row (parent[0] = -1: the root, the anchor; 0 <= parent[r] <
 * r otherwise).  Row r sees cache rows [0, t) and the block rows on its own
 * root path (its ancestors and itself), in row order.  A chain (parent[r] =
 * r - 1) is mode 0 of oc_attention key for key.
 */
void oc_attention_tree(const double *q, int R, int n_q, int n_kv, int hd,
                       const double *kc, const double *vc, int t,
                       const double *kb, const double *vb, const int32_t *parent, double *o)
{
    int g = n_q / n_kv;
    double scale = 1.0 / sqrt((double)hd);
    #pragma omp parallel for schedule(static) collapse(2) if ((long)R * n_q * (t + R) * hd > 1000000)
    for (int r = 0; r < R; ++r)
        for (int h = 0; h < n_q; ++h) {
            int kvh = h / g;
            char *on_path = (char *)calloc((size_t)R, 1);
            for (int a = r; a >= 0; a = parent[a]) on_path[a] = 1;
            const double *qv = q + ((size_t)r * n_q + h) * hd;
            double *s = (double *)malloc(sizeof(double) * (size_t)(t + R));
            double m = -INFINITY;
            for (int j = 0; j < t + R; ++j) {
                if (j >= t && !on_path[j - t]) continue;
                const double *kv = (j < t) ? kc + ((size_t)j * n_kv + kvh) * hd
                                           : kb + ((size_t)(j - t) * n_kv + kvh) * hd;
                double d = 0.0;
                for (int i = 0; i < hd; ++i) d += qv[i] * kv[i];
                s[j] = d * scale;
                if (s[j] > m) m = s[j];
            }
            double l = 0.0;
            for (int j = 0; j < t + R; ++j) {
                if (j >= t && !on_path[j - t]) continue;
                s[j] = exp(s[j] - m);
                l += s[j];
            }
            double *ov = o + ((size_t)r * n_q + h) * hd;
            for (int i = 0; i < hd; ++i) ov[i] = 0.0;
            for (int j = 0; j < t + R; ++j) {
                if (j >= t && !on_path[j - t]) continue;
                const double *vv = (j < t) ? vc + ((size_t)j * n_kv + kvh) * hd
                                           : vb + ((size_t)(j - t) * n_kv + kvh) * hd;
                double p = s[j] / l;
                for (int i = 0; i < hd; ++i) ov[i] += p * vv[i];
            }
            free(s);
            free(on_path);
        }
}

/* ------------------------------------------------------------------------ */
/* One forward of either view over a block of R rows.                         */
/* ------------------------------------------------------------------------ */

/*
 * view 0 = AR (frozen W_Q/W_K/W_V), view 1 = diffusion (W^diff); all other
 * weights are shared (paper notes §2.1).
 * mode 0: the block's K/V are written into the cache at positions t .. t+R-1
 *         (the AR path is the only writer of the cache, §2.2) and rows attend
 *         causally;
 * mode 1: the block's K/V stay in a transient buffer that is freed on return
 *         (they never enter the cache, §2.1/§2.3) and rows attend to the
 *         whole block.
 * kc, vc: [n_layers][cap][n_kv][hd]; rows [0, t) are the committed prefix.
 * logits [R][vocab] and final_hidden [R][hidden] (after the final norm) may
 * be NULL.
 */
static int forward_rows(const oc_cfg *c, const oc_model *w, int view, int mode,
                        const int32_t *tokens, const int32_t *parent, int R, int t,
                        double *kc, double *vc, int cap,
                        double *logits, double *final_hidden);

int oc_forward(const oc_cfg *c, const oc_model *w, int view, int mode,
               const int32_t *tokens, int R, int t,
               double *kc, double *vc, int cap,
               double *logits, double *final_hidden)
{
    return forward_rows(c, w, view, mode, tokens, NULL, R, t, kc, vc, cap, logits, final_hidden);
}

/*
 * AR forward of a draft tree (paper notes §7.5 / §9.6, tree verification):
 * row r is a node with token tokens[r] and parent parent[r] (see
 * oc_attention_tree), at position t + depth(r) (depth(0) = 0, depth(r) =
 * depth(parent[r]) + 1); the rows' K/V are written into cache slots t ..
 * t+R-1 in row order and every row attends to the cache and its own root
 * path.  A node's logits are those of a plain causal forward of its root
 * path.
 */
int oc_forward_tree(const oc_cfg *c, const oc_model *w, const int32_t *tokens, const int32_t *parent, int R,
                    int t, double *kc, double *vc, int cap, double *logits)
{
    if (!parent || R <= 0 || parent[0] != -1) return OC_ERR_ARG;
    for (int r = 1; r < R; ++r)
        if (parent[r] < 0 || parent[r] >= r) return OC_ERR_ARG;
    return forward_rows(c, w, 0, 0, tokens, parent, R, t, kc, vc, cap, logits, NULL);
}

static int forward_rows(const oc_cfg *c, const oc_model *w, int view, int mode,
                        const int32_t *tokens, const int32_t *parent, int R, int t,
                        double *kc, double *vc, int cap,
                        double *logits, double *final_hidden)
{
    if (!c || !w || !tokens || R <= 0 || t < 0 || (view != 0 && view != 1) || (mode != 0 && mode != 1))
        return OC_ERR_ARG;
    if (t + R > cap && mode == 0) return OC_ERR_CAPACITY;
    if (t > cap) return OC_ERR_CAPACITY;
    const int d = c->hidden, nq = c->n_q_heads, nkv = c->n_kv_heads, hd = c->head_dim;
    const int F = c->ffn, V = c->vocab;
    for (int r = 0; r < R; ++r)
        if (tokens[r] < 0 || tokens[r] >= V) return OC_ERR_ARG;

    size_t qn = (size_t)nq * hd, kn = (size_t)nkv * hd;
    double *h = calloc((size_t)R * d, sizeof(double));
    double *a = calloc((size_t)R * d, sizeof(double));
    double *q = calloc((size_t)R * qn, sizeof(double));
    double *k = calloc((size_t)R * kn, sizeof(double));
    double *v = calloc((size_t)R * kn, sizeof(double));
    double *o = calloc((size_t)R * qn, sizeof(double));
    double *y = calloc((size_t)R * d, sizeof(double));
    double *gt = calloc((size_t)R * F, sizeof(double));
    double *up = calloc((size_t)R * F, sizeof(double));
    int *pos = calloc((size_t)R, sizeof(int));
    int rc = OC_OK;
    if (!h || !a || !q || !k || !v || !o || !y || !gt || !up || !pos) { rc = OC_ERR_NOMEM; goto done; }
    for (int r = 0; r < R; ++r)   /* a chain sits at t + r; a tree node one past its parent */
        pos[r] = !parent ? t + r : (r == 0 ? t : pos[parent[r]] + 1);

    for (int r = 0; r < R; ++r)
        for (int i = 0; i < d; ++i) h[(size_t)r * d + i] = (double)w->embed[(size_t)tokens[r] * d + i];

    for (int l = 0; l < c->n_layers; ++l) {
        const oc_layer *L = &w->layers[l];
        double *kcl = kc + (size_t)l * cap * kn, *vcl = vc + (size_t)l * cap * kn;
        for (int r = 0; r < R; ++r) oc_rmsnorm(h + (size_t)r * d, L->attn_norm, d, c->rms_eps, a + (size_t)r * d);
        oc_linear(a, R, d, view ? L->wq_diff : L->wq, nq * hd, q);
        oc_linear(a, R, d, view ? L->wk_diff : L->wk, nkv * hd, k);
        oc_linear(a, R, d, view ? L->wv_diff : L->wv, nkv * hd, v);
        for (int r = 0; r < R; ++r) {
            oc_rope(q + r * qn, nq, hd, pos[r], c->rope_theta);
            oc_rope(k + r * kn, nkv, hd, pos[r], c->rope_theta);
        }
        if (mode == 0) {
            memcpy(kcl + (size_t)t * kn, k, sizeof(double) * R * kn);
            memcpy(vcl + (size_t)t * kn, v, sizeof(double) * R * kn);
            if (parent)
                oc_attention_tree(q, R, nq, nkv, hd, kcl, vcl, t, kcl + (size_t)t * kn, vcl + (size_t)t * kn, parent, o);
            else
                oc_attention(q, R, nq, nkv, hd, kcl, vcl, t, kcl + (size_t)t * kn, vcl + (size_t)t * kn, 0, o);
        } else {
            oc_attention(q, R, nq, nkv, hd, kcl, vcl, t, k, v, 1, o);
        }
        oc_linear(o, R, nq * hd, L->wo, d, y);
        for (size_t i = 0; i < (size_t)R * d; ++i) h[i] += y[i];
        for (int r = 0; r < R; ++r) oc_rmsnorm(h + (size_t)r * d, L->ffn_norm, d, c->rms_eps, a + (size_t)r * d);
        oc_linear(a, R, d, L->w_gate, F, gt);
        oc_linear(a, R, d, L->w_up, F, up);
        for (size_t i = 0; i < (size_t)R * F; ++i) gt[i] = oc_silu(gt[i]) * up[i];
        oc_linear(gt, R, F, L->w_down, d, y);
        for (size_t i = 0; i < (size_t)R * d; ++i) h[i] += y[i];
    }
    for (int r = 0; r < R; ++r) oc_rmsnorm(h + (size_t)r * d, w->final_norm, d, c->rms_eps, a + (size_t)r * d);
    if (final_hidden) memcpy(final_hidden, a, sizeof(double) * R * d);
    if (logits) oc_linear(a, R, d, w->lm_head, V, logits);
done:
    free(h); free(a); free(q); free(k); free(v); free(o); free(y); free(gt); free(up); free(pos);
    return rc;
}

/* AR causal forward over prompt[0 .. P-2]; returns the committed length
 * P-1 (paper notes §2.2: the AR view pre-fills the shared cache). */
int oc_prefill(const oc_cfg *c, const oc_model *w, const int32_t *prompt, int P,
               double *kc, double *vc, int cap)
{
    if (P < 1) return -OC_ERR_ARG;
    if (P == 1) return 0;
    int rc = oc_forward(c, w, 0, 0, prompt, P - 1, 0, kc, vc, cap, NULL, NULL);
    return rc ? -rc : P - 1;
}

/* ------------------------------------------------------------------------ */
/* Randomness: Philox4x32-10 (Salmon, Moraes, Dror, Shaw, SC'11), written    */
/* from the published round function.                                         */
/* ------------------------------------------------------------------------ */

void oc_philox4x32_10(const uint32_t ctr_in[4], const uint32_t key_in[2], uint32_t out[4])
{
    uint32_t x0 = ctr_in[0], x1 = ctr_in[1], x2 = ctr_in[2], x3 = ctr_in[3];
    uint32_t k0 = key_in[0], k1 = key_in[1];
    for (int round = 0; round < 10; ++round) {
        uint64_t p0 = (uint64_t)0xD2511F53u * x0;
        uint64_t p1 = (uint64_t)0xCD9E8D57u * x2;
        uint32_t y0 = (uint32_t)(p1 >> 32) ^ x1 ^ k0;
        uint32_t y1 = (uint32_t)p1;
        uint32_t y2 = (uint32_t)(p0 >> 32) ^ x3 ^ k1;
        uint32_t y3 = (uint32_t)p0;
        x0 = y0; x1 = y1; x2 = y2; x3 = y3;
        k0 += 0x9E3779B9u;
        k1 += 0xBB67AE85u;
    }
    out[0] = x0; out[1] = x1; out[2] = x2; out[3] = x3;
}

/* Uniform in (0, 1): counter (id, row, step, purpose), key (seed lo, hi),
 * first output word, top 24 bits, centred in its cell. */
double oc_uniform(uint64_t seed, uint32_t step, uint32_t row, uint32_t id, uint32_t purpose)
{
    uint32_t ctr[4] = { id, row, step, purpose };
    uint32_t key[2] = { (uint32_t)seed, (uint32_t)(seed >> 32) };
    uint32_t out[4];
    oc_philox4x32_10(ctr, key, out);
    return ((double)(out[0] >> 8) + 0.5) * (1.0 / 16777216.0);
}

double oc_gumbel(uint64_t seed, uint32_t step, uint32_t row, uint32_t id, uint32_t purpose)
{
    return -log(-log(oc_uniform(seed, step, row, id, purpose)));
}

/* The Gumbel noise of ids 0 .. n-1 of one (step, row, purpose): g[i] =
 * oc_gumbel(seed, step, row, i, purpose). */
void oc_gumbel_vec(uint64_t seed, uint32_t step, uint32_t row, uint32_t purpose, int n, double *g)
{
    for (int i = 0; i < n; ++i) g[i] = oc_gumbel(seed, step, row, (uint32_t)i, purpose);
}

/* Lowest index of the maximum; *margin (if given) = best - second best. */
int oc_argmax(const double *x, int n, double *margin)
{
    int best = 0;
    double b = x[0], second = -INFINITY;
    for (int i = 1; i < n; ++i) {
        if (x[i] > b) { second = b; b = x[i]; best = i; }
        else if (x[i] > second) second = x[i];
    }
    if (margin) *margin = b - second;
    return best;
}

/* p = softmax(z / T) */
void oc_softmax_t(const double *z, int n, double T, double *p)
{
    double m = -INFINITY;
    for (int i = 0; i < n; ++i) if (z[i] / T > m) m = z[i] / T;
    double s = 0.0;
    for (int i = 0; i < n; ++i) { p[i] = exp(z[i] / T - m); s += p[i]; }
    for (int i = 0; i < n; ++i) p[i] /= s;
}

/* Gumbel-max draw from softmax(z/T) (one uniform per id). */
int oc_sample_logits(const double *z, int n, double T, uint64_t seed, uint32_t step,
                     uint32_t row, uint32_t purpose, double *margin)
{
    int best = 0;
    double b = -INFINITY, second = -INFINITY;
    for (int i = 0; i < n; ++i) {
        double s = z[i] / T + oc_gumbel(seed, step, row, (uint32_t)i, purpose);
        if (s > b) { second = b; b = s; best = i; }
        else if (s > second) second = s;
    }
    if (margin) *margin = b - second;
    return best;
}

/* ------------------------------------------------------------------------ */
/* Consensus (paper notes §4.1 step 3, §4.2, §4.3).                           */
/* ------------------------------------------------------------------------ */

/* Greedy: accept y_k while it equals the AR argmax g_k; at the first
 * mismatch j emit g_j.  Emitted tokens go to `emit`; returns n in [1, K]. */
int oc_consensus_greedy(const int32_t *draft, const int32_t *g, int K, int32_t *emit)
{
    for (int k = 0; k < K; ++k) {
        emit[k] = g[k];
        if (draft[k] != g[k]) return k + 1;
    }
    return K;
}

/* Leviathan/Chen acceptance probability of a draft with target mass p and
 * draft mass q. */
double oc_accept_prob(double p, double q)
{
    if (q <= 0.0) return 1.0;
    double a = p / q;
    return a < 1.0 ? a : 1.0;
}

/* Residual distribution norm(max(0, p - q)).  Returns 0 and fills r when it
 * has mass; returns 1 (r untouched) when p <= q everywhere. */
int oc_residual(const double *p, const double *q, int n, double *r)
{
    double s = 0.0;
    for (int i = 0; i < n; ++i) { double d = p[i] - q[i]; s += d > 0.0 ? d : 0.0; }
    if (!(s > 0.0)) return 1;
    for (int i = 0; i < n; ++i) { double d = p[i] - q[i]; r[i] = (d > 0.0 ? d : 0.0) / s; }
    return 0;
}

/* ------------------------------------------------------------------------ */
/* The three stages of one cycle.                                             */
/* ------------------------------------------------------------------------ */

/* Parallel projection (§4.1 step 1): block [anchor, mask x (K-1)] at
 * positions t .. t+K-1 through the diffusion view.  With n_iter > 1 the
 * diffusion view runs again n_iter - 1 times, each time on the block
 * [anchor, y_1 .. y_{K-1}] of the previous pass's drafts (the iterative-
 * denoising variant the paper-notes page compares against in §5.4.2; the
 * page gives no procedure, this is its plainest reading).  Pass s draws its
 * Gumbel noise with purpose DRAFT | s << 8, so pass 0 is the single-step
 * draft.  Writes the K drafts of the last pass; at T>0 also q_probs [K][V] =
 * softmax(w/T) of the last pass when given.  logits [K][V] may be NULL. */
int oc_draft_iter(const oc_cfg *c, const oc_model *w, double *kc, double *vc, int cap, int t,
                  int32_t anchor, int K, int n_iter, double T, uint64_t seed, uint32_t step,
                  int32_t *draft, double *q_probs, double *logits, double *min_margin)
{
    if (n_iter < 1) return OC_ERR_ARG;
    int V = c->vocab;
    int32_t *blk = malloc(sizeof(int32_t) * K);
    double *z = malloc(sizeof(double) * (size_t)K * V);
    if (!blk || !z) { free(blk); free(z); return OC_ERR_NOMEM; }
    int rc = OC_OK;
    for (int s = 0; s < n_iter && rc == OC_OK; ++s) {
        blk[0] = anchor;
        for (int k = 1; k < K; ++k) blk[k] = s == 0 ? c->mask_id : draft[k - 1];
        rc = oc_forward(c, w, 1, 1, blk, K, t, kc, vc, cap, z, NULL);
        if (rc != OC_OK) break;
        const int last = s == n_iter - 1;
        for (int k = 0; k < K; ++k) {
            const double *zk = z + (size_t)k * V;
            double mg;
            if (T > 0.0) {
                draft[k] = oc_sample_logits(zk, V, T, seed, step, (uint32_t)k, OC_PURPOSE_DRAFT | ((uint32_t)s << 8), &mg);
                if (last && q_probs) oc_softmax_t(zk, V, T, q_probs + (size_t)k * V);
            } else {
                draft[k] = oc_argmax(zk, V, &mg);
            }
            if (min_margin && mg < *min_margin) *min_margin = mg;
        }
        if (last && logits) memcpy(logits, z, sizeof(double) * (size_t)K * V);
    }
    free(blk); free(z);
    return rc;
}

int oc_draft(const oc_cfg *c, const oc_model *w, double *kc, double *vc, int cap, int t,
             int32_t anchor, int K, double T, uint64_t seed, uint32_t step,
             int32_t *draft, double *q_probs, double *logits, double *min_margin)
{
    return oc_draft_iter(c, w, kc, vc, cap, t, anchor, K, 1, T, seed, step, draft, q_probs, logits, min_margin);
}

/* AR verification (§4.1 step 2): block [anchor, y_1 .. y_{K-1}] through the
 * AR view, K/V written at t .. t+K-1.  Writes g [K] (argmax per row) and, at
 * T>0, p_probs [K][V] = softmax(z/T).  logits may be NULL. */
int oc_verify(const oc_cfg *c, const oc_model *w, double *kc, double *vc, int cap, int t,
              int32_t anchor, const int32_t *draft, int K, double T,
              int32_t *g, double *p_probs, double *logits, double *min_margin)
{
    int V = c->vocab;
    int32_t *blk = malloc(sizeof(int32_t) * K);
    double *z = malloc(sizeof(double) * (size_t)K * V);
    if (!blk || !z) { free(blk); free(z); return OC_ERR_NOMEM; }
    blk[0] = anchor;
    for (int k = 1; k < K; ++k) blk[k] = draft[k - 1];
    int rc = oc_forward(c, w, 0, 0, blk, K, t, kc, vc, cap, z, NULL);
    if (rc == OC_OK) {
        for (int k = 0; k < K; ++k) {
            double mg;
            g[k] = oc_argmax(z + (size_t)k * V, V, &mg);
            if (T > 0.0 && p_probs) oc_softmax_t(z + (size_t)k * V, V, T, p_probs + (size_t)k * V);
            if (min_margin && T <= 0.0 && mg < *min_margin) *min_margin = mg;
        }
        if (logits) memcpy(logits, z, sizeof(double) * (size_t)K * V);
    }
    free(blk); free(z);
    return rc;
}

/* Consensus at T>0 (§4.3): accept y_k with probability min(1, p_k/q_k) using
 * u_k; at the first rejection j draw the correction from norm(max(0, p_j -
 * q_j)).  Returns n and fills emit. */
int oc_consensus_sample(const double *p, const double *q, const int32_t *draft, const int32_t *g,
                        int K, int V, uint64_t seed, uint32_t step, int32_t *emit,
                        double *min_margin)
{
    double *r = malloc(sizeof(double) * V);
    double *lr = malloc(sizeof(double) * V);
    int n = K;
    for (int k = 0; k < K; ++k) {
        const double *pk = p + (size_t)k * V, *qk = q + (size_t)k * V;
        double a = oc_accept_prob(pk[draft[k]], qk[draft[k]]);
        double u = oc_uniform(seed, step, (uint32_t)k, 0, OC_PURPOSE_ACCEPT);
        if (min_margin && fabs(u - a) < *min_margin) *min_margin = fabs(u - a);
        if (u < a) { emit[k] = draft[k]; continue; }
        if (oc_residual(pk, qk, V, r) == 0) {
            for (int i = 0; i < V; ++i) lr[i] = r[i] > 0.0 ? log(r[i]) : -INFINITY;
            double mg;
            emit[k] = oc_sample_logits(lr, V, 1.0, seed, step, (uint32_t)k, OC_PURPOSE_RESIDUAL, &mg);
            if (min_margin && mg < *min_margin) *min_margin = mg;
        } else {
            emit[k] = g[k];
        }
        n = k + 1;
        break;
    }
    free(r); free(lr);
    return n;
}

/*
 * Whole decode from a prompt.  method 0 = plain AR (one AR forward per
 * token), method 1 = Orthrus (draft, verify, consensus, commit per cycle).
 * Stops once N tokens are out; out[N].  n_per_cycle (may be NULL) receives
 * the tokens emitted by each cycle and *n_cycles their count.  *min_margin
 * (may be NULL) receives the smallest argmax / acceptance decision margin
 * seen, so callers can tell a decision that fp32 rounding could flip, and
 * cycle_margin[c] (may be NULL; N entries) the smallest margin among the
 * decisions of cycle c alone (draft argmaxes or samples, verify argmaxes at
 * T = 0, acceptance tests and the residual draw at T > 0).
 * kc_out / vc_out (may be NULL) receive the final committed cache
 * [n_layers][cap][n_kv][hd], cap = P + N + K, rows beyond the committed length
 * zeroed.  *t_out (may be NULL) receives the final committed length.
 */
int oc_generate_iter(const oc_cfg *c, const oc_model *w, const int32_t *prompt, int P, int K, int N,
                     double T, uint64_t seed, int method, int n_iter, int32_t *out, int32_t *n_per_cycle,
                     int *n_cycles, double *min_margin, double *kc_out, double *vc_out, int *t_out,
                     double *cycle_margin)
{
    if (!c || !w || !prompt || P < 1 || N < 1 || K < 1 || (method != 0 && method != 1) || n_iter < 1)
        return OC_ERR_ARG;
    const int V = c->vocab;
    const int cap = P + N + K;
    const size_t kn = (size_t)c->n_kv_heads * c->head_dim;
    const size_t csz = (size_t)c->n_layers * cap * kn;
    double *kc = calloc(csz, sizeof(double)), *vc = calloc(csz, sizeof(double));
    int32_t *draft = malloc(sizeof(int32_t) * K), *g = malloc(sizeof(int32_t) * K);
    int32_t *emit = malloc(sizeof(int32_t) * K);
    double *p = NULL, *q = NULL, *z = malloc(sizeof(double) * V);
    if (T > 0.0) { p = malloc(sizeof(double) * (size_t)K * V); q = malloc(sizeof(double) * (size_t)K * V); }
    int rc = OC_OK;
    if (!kc || !vc || !draft || !g || !emit || !z || (T > 0.0 && (!p || !q))) { rc = OC_ERR_NOMEM; goto done; }
    if (min_margin) *min_margin = INFINITY;

    int t = oc_prefill(c, w, prompt, P, kc, vc, cap);
    if (t < 0) { rc = -t; goto done; }
    int32_t anchor = prompt[P - 1];
    int produced = 0, cycles = 0;
    while (produced < N) {
        int n;
        double cm = INFINITY;   /* smallest decision margin of this cycle */
        if (method == 0) {
            rc = oc_forward(c, w, 0, 0, &anchor, 1, t, kc, vc, cap, z, NULL);
            if (rc) goto done;
            emit[0] = (T > 0.0) ? oc_sample_logits(z, V, T, seed, (uint32_t)produced, 0, OC_PURPOSE_AR, &cm)
                                : oc_argmax(z, V, &cm);
            n = 1;
        } else {
            rc = oc_draft_iter(c, w, kc, vc, cap, t, anchor, K, n_iter, T, seed, (uint32_t)cycles, draft, q, NULL,
                               &cm);
            if (rc) goto done;
            rc = oc_verify(c, w, kc, vc, cap, t, anchor, draft, K, T, g, p, NULL, &cm);
            if (rc) goto done;
            n = (T > 0.0) ? oc_consensus_sample(p, q, draft, g, K, V, seed, (uint32_t)cycles, emit, &cm)
                          : oc_consensus_greedy(draft, g, K, emit);
        }
        if (min_margin && cm < *min_margin) *min_margin = cm;
        if (cycle_margin) cycle_margin[cycles] = cm;
        /* commit (§4.1 step 3): keep cache rows t .. t+n-1 (already written by
         * the AR forward for the accepted inputs), discard the rest. */
        t += n;
        anchor = emit[n - 1];
        for (int i = 0; i < n && produced < N; ++i) out[produced++] = emit[i];
        if (n_per_cycle) n_per_cycle[cycles] = n;
        ++cycles;
    }
    if (n_cycles) *n_cycles = cycles;
    if (t_out) *t_out = t;
    if (kc_out || vc_out) {
        for (int l = 0; l < c->n_layers; ++l) {
            double *kl = kc + (size_t)l * cap * kn, *vl = vc + (size_t)l * cap * kn;
            memset(kl + (size_t)t * kn, 0, sizeof(double) * (size_t)(cap - t) * kn);
            memset(vl + (size_t)t * kn, 0, sizeof(double) * (size_t)(cap - t) * kn);
        }
        if (kc_out) memcpy(kc_out, kc, sizeof(double) * csz);
        if (vc_out) memcpy(vc_out, vc, sizeof(double) * csz);
    }
done:
    free(kc); free(vc); free(draft); free(g); free(emit); free(p); free(q); free(z);
    return rc;
}

int oc_generate(const oc_cfg *c, const oc_model *w, const int32_t *prompt, int P, int K, int N,
                double T, uint64_t seed, int method, int32_t *out, int32_t *n_per_cycle,
                int *n_cycles, double *min_margin, double *kc_out, double *vc_out, int *t_out)
{
    return oc_generate_iter(c, w, prompt, P, K, N, T, seed, method, 1, out, n_per_cycle, n_cycles, min_margin,
                            kc_out, vc_out, t_out, NULL);
}

/* ------------------------------------------------------------------------ */
/* Exact laws for the losslessness pin (paper notes §4.3, §9.1).              */
/* ------------------------------------------------------------------------ */

static long ipow(int b, int e) { long r = 1; while (e-- > 0) r *= b; return r; }

/* Next-token distribution p_AR(. | seq[0 .. len-1]) at temperature T:
 * prefill seq[0 .. len-2], then one AR row for seq[len-1]. */
static int ar_next(const oc_cfg *c, const oc_model *w, const int32_t *seq, int len, double T, double *p)
{
    int cap = len;
    size_t csz = (size_t)c->n_layers * cap * c->n_kv_heads * c->head_dim;
    double *kc = calloc(csz, sizeof(double)), *vc = calloc(csz, sizeof(double));
    double *z = malloc(sizeof(double) * c->vocab);
    int rc = (!kc || !vc || !z) ? OC_ERR_NOMEM : OC_OK;
    if (rc == OC_OK && len > 1) rc = oc_forward(c, w, 0, 0, seq, len - 1, 0, kc, vc, cap, NULL, NULL);
    if (rc == OC_OK) rc = oc_forward(c, w, 0, 0, seq + len - 1, 1, len - 1, kc, vc, cap, z, NULL);
    if (rc == OC_OK) oc_softmax_t(z, c->vocab, T, p);
    free(kc); free(vc); free(z);
    return rc;
}

/* dist[V^N]: probability of each first-N token string under plain AR
 * sampling at temperature T after the prompt. */
int oc_enumerate_ar(const oc_cfg *c, const oc_model *w, const int32_t *prompt, int P, int N,
                    double T, double *dist)
{
    const int V = c->vocab;
    long total = ipow(V, N);
    int32_t *seq = malloc(sizeof(int32_t) * (P + N));
    double *p = malloc(sizeof(double) * V);
    double *mass = malloc(sizeof(double) * (size_t)total);   /* mass of each prefix, level by level */
    double *next = malloc(sizeof(double) * (size_t)total);
    if (!seq || !p || !mass || !next) { free(seq); free(p); free(mass); free(next); return OC_ERR_NOMEM; }
    memcpy(seq, prompt, sizeof(int32_t) * P);
    mass[0] = 1.0;
    int rc = OC_OK;
    for (int e = 0; e < N && rc == OC_OK; ++e) {
        long cnt = ipow(V, e);
        for (long idx = 0; idx < cnt; ++idx) {
            long rem = idx;
            for (int i = e - 1; i >= 0; --i) { seq[P + i] = (int32_t)(rem % V); rem /= V; }
            rc = ar_next(c, w, seq, P + e, T, p);
            if (rc) break;
            for (int v = 0; v < V; ++v) next[idx * V + v] = mass[idx] * p[v];
        }
        memcpy(mass, next, sizeof(double) * (size_t)cnt * V);
    }
    if (rc == OC_OK) memcpy(dist, mass, sizeof(double) * (size_t)total);
    free(seq); free(p); free(mass); free(next);
    return rc;
}

/*
 * dist[V^N]: exact probability of each first-N token string produced by the
 * Orthrus cycle at temperature T > 0, under ideal randomness: drafts y_k drawn
 * independently from q_k (one diffusion forward), acceptance with
 * oc_accept_prob, correction from oc_residual (or argmax p when it has no
 * mass).  The draft and verify distributions come from oc_draft /
 * oc_verify-equivalent forwards.  planted_error = 1 replaces the residual by
 * p itself (a known mistake that must break losslessness).
 */
int oc_enumerate_orthrus(const oc_cfg *c, const oc_model *w, const int32_t *prompt, int P, int K,
                         int N, double T, int planted_error, double *dist)
{
    const int V = c->vocab;
    const long total = ipow(V, N);
    long ntuple = ipow(V, K);
    int rc = OC_OK;
    /* mass of states by number of emitted tokens e (< N), dense over V^e */
    double **lvl = calloc(N, sizeof(double *));
    int32_t *seq = malloc(sizeof(int32_t) * (P + N + K));
    int32_t *blk = malloc(sizeof(int32_t) * K);
    int32_t *y = malloc(sizeof(int32_t) * K);
    double *qz = malloc(sizeof(double) * (size_t)K * V), *q = malloc(sizeof(double) * (size_t)K * V);
    double *pz = malloc(sizeof(double) * (size_t)K * V), *p = malloc(sizeof(double) * (size_t)K * V);
    double *r = malloc(sizeof(double) * V);
    if (!lvl || !seq || !blk || !y || !qz || !q || !pz || !p || !r) { rc = OC_ERR_NOMEM; goto out; }
    for (int e = 0; e < N; ++e) {
        lvl[e] = calloc((size_t)ipow(V, e), sizeof(double));
        if (!lvl[e]) { rc = OC_ERR_NOMEM; goto out; }
    }
    memset(dist, 0, sizeof(double) * (size_t)total);
    memcpy(seq, prompt, sizeof(int32_t) * P);
    lvl[0][0] = 1.0;
    const int cap = P + N + K;
    const size_t csz = (size_t)c->n_layers * cap * c->n_kv_heads * c->head_dim;
    double *kc = calloc(csz, sizeof(double)), *vc = calloc(csz, sizeof(double));
    if (!kc || !vc) { free(kc); free(vc); rc = OC_ERR_NOMEM; goto out; }

    for (int e = 0; e < N && rc == OC_OK; ++e) {
        long cnt = ipow(V, e);
        for (long idx = 0; idx < cnt && rc == OC_OK; ++idx) {
            double wstate = lvl[e][idx];
            if (wstate == 0.0) continue;
            long rem = idx;
            for (int i = e - 1; i >= 0; --i) { seq[P + i] = (int32_t)(rem % V); rem /= V; }
            int len = P + e;                         /* tokens known so far */
            int t = len - 1;                         /* committed cache length */
            int32_t anchor = seq[len - 1];
            if (t > 0) rc = oc_forward(c, w, 0, 0, seq, t, 0, kc, vc, cap, NULL, NULL);
            if (rc) break;
            blk[0] = anchor;
            for (int k = 1; k < K; ++k) blk[k] = c->mask_id;
            rc = oc_forward(c, w, 1, 1, blk, K, t, kc, vc, cap, qz, NULL);
            if (rc) break;
            for (int k = 0; k < K; ++k) oc_softmax_t(qz + (size_t)k * V, V, T, q + (size_t)k * V);
            long prev_ctx = -1;
            for (long tup = 0; tup < ntuple && rc == OC_OK; ++tup) {
                long rr = tup;
                for (int k = K - 1; k >= 0; --k) { y[k] = (int32_t)(rr % V); rr /= V; }
                double wq = 1.0;
                for (int k = 0; k < K; ++k) wq *= q[(size_t)k * V + y[k]];
                if (wq == 0.0) continue;
                long ctx = tup / V;                  /* verify depends on y_1..y_{K-1} only */
                if (ctx != prev_ctx) {
                    blk[0] = anchor;
                    for (int k = 1; k < K; ++k) blk[k] = y[k - 1];
                    rc = oc_forward(c, w, 0, 0, blk, K, t, kc, vc, cap, pz, NULL);
                    if (rc) break;
                    for (int k = 0; k < K; ++k) oc_softmax_t(pz + (size_t)k * V, V, T, p + (size_t)k * V);
                    prev_ctx = ctx;
                }
                double acc = 1.0;
                int j;
                for (j = 0; j < K; ++j) {
                    const double *pj = p + (size_t)j * V, *qj = q + (size_t)j * V;
                    double a = oc_accept_prob(pj[y[j]], qj[y[j]]);
                    double rej = acc * (1.0 - a);
                    if (rej > 0.0) {
                        int none;
                        if (planted_error) { memcpy(r, pj, sizeof(double) * V); none = 0; }
                        else none = oc_residual(pj, qj, V, r);
                        for (int cc = 0; cc < V; ++cc) {
                            double pr = none ? (cc == oc_argmax(pj, V, NULL) ? 1.0 : 0.0) : r[cc];
                            if (pr == 0.0) continue;
                            /* emitted: y_0..y_{j-1}, cc  (j+1 tokens) */
                            long ne = e + j + 1, nidx = idx;
                            double m = wstate * wq * rej * pr;
                            int lim = ne < N ? (int)ne : N;
                            for (int i = e; i < lim; ++i) nidx = nidx * V + (i - e < j ? y[i - e] : cc);
                            if (ne >= N) dist[nidx] += m; else lvl[ne][nidx] += m;
                        }
                    }
                    acc *= a;
                    if (acc == 0.0) break;
                }
                if (j == K && acc > 0.0) {
                    long ne = e + K, nidx = idx;
                    int lim = ne < N ? (int)ne : N;
                    for (int i = e; i < lim; ++i) nidx = nidx * V + y[i - e];
                    if (ne >= N) dist[nidx] += wstate * wq * acc; else lvl[ne][nidx] += wstate * wq * acc;
                }
            }
        }
    }
    free(kc); free(vc);
out:
    if (lvl) for (int e = 0; e < N; ++e) free(lvl[e]);
    free(lvl); free(seq); free(blk); free(y); free(qz); free(q); free(pz); free(p); free(r);
    return rc;
}

/*
 * As oc_enumerate_orthrus for the two-pass draft (oc_draft_iter, n_iter = 2):
 * first-pass drafts x drawn independently from q1_k (mask block), second-pass
 * drafts y drawn independently from q2_k(. | x) (block [anchor, x_1 ..
 * x_{K-1}]), acceptance with min(1, p_k(y_k) / q2_k(y_k)), correction from
 * norm(max(0, p_j - q2_j)).  The first pass only shapes the proposal, so the
 * law of the emitted string must still be the AR law.  Exponential in K:
 * micro models only.
 */
int oc_enumerate_orthrus_2pass(const oc_cfg *c, const oc_model *w, const int32_t *prompt, int P, int K,
                               int N, double T, int planted_error, double *dist)
{
    const int V = c->vocab;
    const long total = ipow(V, N);
    const long ntuple = ipow(V, K), nctx = ipow(V, K - 1);
    int rc = OC_OK;
    double **lvl = calloc(N, sizeof(double *));
    int32_t *seq = malloc(sizeof(int32_t) * (P + N + K));
    int32_t *blk = malloc(sizeof(int32_t) * K);
    int32_t *x = malloc(sizeof(int32_t) * K), *y = malloc(sizeof(int32_t) * K);
    double *z = malloc(sizeof(double) * (size_t)K * V);
    double *q1 = malloc(sizeof(double) * (size_t)K * V), *q2 = malloc(sizeof(double) * (size_t)K * V);
    double *pc = malloc(sizeof(double) * (size_t)nctx * K * V);   /* verify softmax per draft context */
    double *r = malloc(sizeof(double) * V);
    double *kc = NULL, *vc = NULL;
    if (!lvl || !seq || !blk || !x || !y || !z || !q1 || !q2 || !pc || !r) { rc = OC_ERR_NOMEM; goto out; }
    for (int e = 0; e < N; ++e) {
        lvl[e] = calloc((size_t)ipow(V, e), sizeof(double));
        if (!lvl[e]) { rc = OC_ERR_NOMEM; goto out; }
    }
    memset(dist, 0, sizeof(double) * (size_t)total);
    memcpy(seq, prompt, sizeof(int32_t) * P);
    lvl[0][0] = 1.0;
    const int cap = P + N + K;
    const size_t csz = (size_t)c->n_layers * cap * c->n_kv_heads * c->head_dim;
    kc = calloc(csz, sizeof(double));
    vc = calloc(csz, sizeof(double));
    if (!kc || !vc) { rc = OC_ERR_NOMEM; goto out; }

    for (int e = 0; e < N && rc == OC_OK; ++e) {
        const long cnt = ipow(V, e);
        for (long idx = 0; idx < cnt && rc == OC_OK; ++idx) {
            const double wstate = lvl[e][idx];
            if (wstate == 0.0) continue;
            long rem = idx;
            for (int i = e - 1; i >= 0; --i) { seq[P + i] = (int32_t)(rem % V); rem /= V; }
            const int len = P + e, t = len - 1;
            const int32_t anchor = seq[len - 1];
            if (t > 0) rc = oc_forward(c, w, 0, 0, seq, t, 0, kc, vc, cap, NULL, NULL);
            if (rc) break;
            /* verify distributions for every second-pass context y_1 .. y_{K-1} */
            for (long ctx = 0; ctx < nctx && rc == OC_OK; ++ctx) {
                long rr = ctx;
                blk[0] = anchor;
                for (int k = K - 1; k >= 1; --k) { blk[k] = (int32_t)(rr % V); rr /= V; }
                rc = oc_forward(c, w, 0, 0, blk, K, t, kc, vc, cap, z, NULL);
                for (int k = 0; k < K && rc == OC_OK; ++k)
                    oc_softmax_t(z + (size_t)k * V, V, T, pc + ((size_t)ctx * K + k) * V);
            }
            if (rc) break;
            /* first pass */
            blk[0] = anchor;
            for (int k = 1; k < K; ++k) blk[k] = c->mask_id;
            rc = oc_forward(c, w, 1, 1, blk, K, t, kc, vc, cap, z, NULL);
            if (rc) break;
            for (int k = 0; k < K; ++k) oc_softmax_t(z + (size_t)k * V, V, T, q1 + (size_t)k * V);
            long prev_x = -1;
            for (long tx = 0; tx < ntuple && rc == OC_OK; ++tx) {
                long rr = tx;
                for (int k = K - 1; k >= 0; --k) { x[k] = (int32_t)(rr % V); rr /= V; }
                double wx = 1.0;
                for (int k = 0; k < K; ++k) wx *= q1[(size_t)k * V + x[k]];
                if (wx == 0.0) continue;
                if (tx / V != prev_x) {           /* the second pass sees x_1 .. x_{K-1} only */
                    blk[0] = anchor;
                    for (int k = 1; k < K; ++k) blk[k] = x[k - 1];
                    rc = oc_forward(c, w, 1, 1, blk, K, t, kc, vc, cap, z, NULL);
                    if (rc) break;
                    for (int k = 0; k < K; ++k) oc_softmax_t(z + (size_t)k * V, V, T, q2 + (size_t)k * V);
                    prev_x = tx / V;
                }
                for (long ty = 0; ty < ntuple; ++ty) {
                    long ry = ty;
                    for (int k = K - 1; k >= 0; --k) { y[k] = (int32_t)(ry % V); ry /= V; }
                    double wy = 1.0;
                    for (int k = 0; k < K; ++k) wy *= q2[(size_t)k * V + y[k]];
                    if (wy == 0.0) continue;
                    const double *p = pc + (size_t)(ty / V) * K * V;
                    const double wb = wstate * wx * wy;
                    double acc = 1.0;
                    int j;
                    for (j = 0; j < K; ++j) {
                        const double *pj = p + (size_t)j * V, *qj = q2 + (size_t)j * V;
                        double a = oc_accept_prob(pj[y[j]], qj[y[j]]);
                        double rej = acc * (1.0 - a);
                        if (rej > 0.0) {
                            int none;
                            if (planted_error) { memcpy(r, pj, sizeof(double) * V); none = 0; }
                            else none = oc_residual(pj, qj, V, r);
                            for (int cc = 0; cc < V; ++cc) {
                                double pr = none ? (cc == oc_argmax(pj, V, NULL) ? 1.0 : 0.0) : r[cc];
                                if (pr == 0.0) continue;
                                long ne = e + j + 1, nidx = idx;
                                int lim = ne < N ? (int)ne : N;
                                for (int i = e; i < lim; ++i) nidx = nidx * V + (i - e < j ? y[i - e] : cc);
                                if (ne >= N) dist[nidx] += wb * rej * pr; else lvl[ne][nidx] += wb * rej * pr;
                            }
                        }
                        acc *= a;
                        if (acc == 0.0) break;
                    }
                    if (j == K && acc > 0.0) {
                        long ne = e + K, nidx = idx;
                        int lim = ne < N ? (int)ne : N;
                        for (int i = e; i < lim; ++i) nidx = nidx * V + y[i - e];
                        if (ne >= N) dist[nidx] += wb * acc; else lvl[ne][nidx] += wb * acc;
                    }
                }
            }
        }
    }
out:
    free(kc); free(vc);
    if (lvl) for (int e = 0; e < N; ++e) free(lvl[e]);
    free(lvl); free(seq); free(blk); free(x); free(y); free(z); free(q1); free(q2); free(pc); free(r);
    return rc;
}

/* ------------------------------------------------------------------------ */
/* Training-side pieces (paper notes §3.1-3.3): the dual-pass block mask and  */
/* the forward KL against the frozen AR view.                                 */
/* ------------------------------------------------------------------------ */

/*
 * Block-masked attention of the diffusion pass over one packed training
 * sequence (paper notes §3.1-3.2: a packed sequence of L clean tokens holds
 * n_blocks anchor blocks of K positions; block b starts at anchor position
 * a_b).  The key set is the packed layout itself: the L clean context
 * positions (their AR K/V) followed by every block's K rows (its diffusion
 * K/V).  Query row k of block b may see
 *   - context position p        iff p < a_b  (causal up to, not including,
 *                                             its anchor: the anchor is the
 *                                             block's own row 0),
 *   - row k' of block b'         iff b' == b  (bidirectional inside the
 *                                             block; blocks never see one
 *                                             another).
 *   q            [n_blocks*K][n_q][hd]
 *   kctx, vctx   [L][n_kv][hd]
 *   kblk, vblk   [n_blocks*K][n_kv][hd]
 *   anchors      [n_blocks], 0 <= a_b <= L
 *   o            [n_blocks*K][n_q][hd]
 * The mask is evaluated for every key of the packed layout (L + n_blocks*K
 * of them), so this is a plain masked softmax written out, independent of
 * oc_attention's per-sequence key walk.
 */
void oc_block_mask_attention(const double *q, int n_blocks, int K, int n_q, int n_kv, int hd,
                             const double *kctx, const double *vctx, int L,
                             const double *kblk, const double *vblk, const int32_t *anchors, double *o)
{
    int g = n_q / n_kv;
    long nkeys = (long)L + (long)n_blocks * K;
    double scale = 1.0 / sqrt((double)hd);
    #pragma omp parallel for schedule(static) collapse(2) if ((long)n_blocks * K * n_q * nkeys * hd > 1000000)
    for (int row = 0; row < n_blocks * K; ++row)
        for (int h = 0; h < n_q; ++h) {
            int b = row / K, kvh = h / g;
            const double *qv = q + ((size_t)row * n_q + h) * hd;
            double *s = (double *)malloc(sizeof(double) * (size_t)nkeys);
            char *vis = (char *)malloc((size_t)nkeys);
            double m = -INFINITY;
            for (long j = 0; j < nkeys; ++j) {
                int visible;
                const double *kv;
                if (j < L) {
                    visible = j < anchors[b];
                    kv = kctx + ((size_t)j * n_kv + kvh) * hd;
                } else {
                    long jb = j - L;
                    visible = (int)(jb / K) == b;
                    kv = kblk + ((size_t)jb * n_kv + kvh) * hd;
                }
                vis[j] = (char)visible;
                if (!visible) continue;
                double d = 0.0;
                for (int i = 0; i < hd; ++i) d += qv[i] * kv[i];
                s[j] = d * scale;
                if (s[j] > m) m = s[j];
            }
            double l = 0.0;
            for (long j = 0; j < nkeys; ++j)
                if (vis[j]) { s[j] = exp(s[j] - m); l += s[j]; }
            double *ov = o + ((size_t)row * n_q + h) * hd;
            for (int i = 0; i < hd; ++i) ov[i] = 0.0;
            for (long j = 0; j < nkeys; ++j) {
                if (!vis[j]) continue;
                const double *vv = (j < L) ? vctx + ((size_t)j * n_kv + kvh) * hd
                                           : vblk + ((size_t)(j - L) * n_kv + kvh) * hd;
                double p = s[j] / l;
                for (int i = 0; i < hd; ++i) ov[i] += p * vv[i];
            }
            free(vis);
            free(s);
        }
}

/*
 * Forward KL of the distillation loss (paper notes §3.3): for each row r,
 * z_A = W h_A[r] (frozen AR view) and z_D = W h_D[r] (diffusion view) over
 * the whole vocabulary (the shared LM head W [V][d]; h are the final-normed
 * hidden rows), p = softmax(z) and
 *     KL(p_A || p_D) = sum_v p_A(v) (log p_A(v) - log p_D(v)).
 * Also returns both log-sum-exps.
 */
void oc_kl_rows(const double *hA, const double *hD, int rows, int d, const float *W, int V,
                double *kl, double *lseA, double *lseD)
{
    #pragma omp parallel for schedule(static) if ((long)rows * V * d > 1000000)
    for (int r = 0; r < rows; ++r) {
        double *zA = (double *)malloc(sizeof(double) * (size_t)V);
        double *zD = (double *)malloc(sizeof(double) * (size_t)V);
        double mA = -INFINITY, mD = -INFINITY;
        for (int v = 0; v < V; ++v) {
            const float *w = W + (size_t)v * d;
            double a = 0.0, b = 0.0;
            for (int i = 0; i < d; ++i) {
                a += (double)w[i] * hA[(size_t)r * d + i];
                b += (double)w[i] * hD[(size_t)r * d + i];
            }
            zA[v] = a; zD[v] = b;
            if (a > mA) mA = a;
            if (b > mD) mD = b;
        }
        double sA = 0.0, sD = 0.0;
        for (int v = 0; v < V; ++v) { sA += exp(zA[v] - mA); sD += exp(zD[v] - mD); }
        double la = mA + log(sA), ld = mD + log(sD), acc = 0.0;
        for (int v = 0; v < V; ++v) {
            double lpa = zA[v] - la, lpd = zD[v] - ld;
            acc += exp(lpa) * (lpa - lpd);
        }
        kl[r] = acc;
        if (lseA) lseA[r] = la;
        if (lseD) lseD[r] = ld;
        free(zA);
        free(zD);
    }
}

/* ------------------------------------------------------------------------ */
/* Tree verification (paper notes §7.5 and §9.6: DDTree's best-first tree    */
/* over one diffusion forward's marginals, verified by one tree-masked AR    */
/* forward).  Greedy (T = 0) only: the pages give no sampling rule for it.   */
/* ------------------------------------------------------------------------ */

/* The W largest entries of z [V], best first, ties to the lowest id (W
 * rounds of "largest not yet taken"), and, if lse is not NULL, the
 * log-sum-exp log sum_v exp(z_v) = m + log sum_v exp(z_v - m), m = max z. */
void oc_topw(const double *z, int V, int W, int32_t *ids, double *lse)
{
    for (int r = 0; r < W; ++r) {
        int best = -1;
        for (int v = 0; v < V; ++v) {
            int taken = 0;
            for (int u = 0; u < r; ++u) taken |= ids[u] == v;
            if (!taken && (best < 0 || z[v] > z[best])) best = v;
        }
        ids[r] = best;
    }
    if (lse) {
        double m = -INFINITY, s = 0.0;
        for (int v = 0; v < V; ++v) if (z[v] > m) m = z[v];
        for (int v = 0; v < V; ++v) s += exp(z[v] - m);
        *lse = m + log(s);
    }
}

/* Lexicographic order of rank sequences, a prefix before its extensions. */
static int rankseq_less(const int32_t *a, int la, const int32_t *b, int lb)
{
    for (int i = 0; i < la && i < lb; ++i)
        if (a[i] != b[i]) return a[i] < b[i];
    return la < lb;
}

/*
 * Best-first draft tree.  logp [D][V]: log-probabilities of the token at
 * depth d + 1 (the draft row d's distribution at T = 1).  At every depth
 * the candidates are the W most probable ids of that row (ties: lowest id),
 * ranked 0 .. W-1.  A prefix y_1 .. y_d scores sum_i logp[i-1][y_i]; the
 * tree is the root (the anchor, row 0) plus the N best prefixes of depth
 * 1 .. D, ordered by score and then by their rank sequences (so a prefix
 * always precedes its extensions, and the chosen set is closed under
 * prefixes).  They are found the best-first way: a pool holding, for every
 * chosen node, its best child and its next sibling, from which the best
 * entry is taken N times.  Outputs (N + 1 rows, in selection order, so a
 * parent's row is below its children's): parent (-1 for the root), token
 * (-1 for the root), depth, score.  Returns the number of rows (fewer than
 * N + 1 when fewer prefixes exist), or -OC_ERR_* on bad arguments.
 */
int oc_tree_build(const double *logp, int D, int V, int W, int N, int32_t *parent, int32_t *token,
                  int32_t *depth, double *score)
{
    if (D < 0 || V < 1 || W < 1 || W > V || N < 0 || !parent || !token || !depth || !score) return -OC_ERR_ARG;
    if (D > 0 && !logp) return -OC_ERR_ARG;
    int32_t *cand = malloc(sizeof(int32_t) * (size_t)(D > 0 ? D : 1) * W);   /* [D][W] ranked ids */
    int32_t *rseq = malloc(sizeof(int32_t) * (size_t)(N + 1) * (D > 0 ? D : 1));   /* node rank sequences */
    int pool_cap = 2 * N + 2;
    int32_t *pp = malloc(sizeof(int32_t) * pool_cap), *pr = malloc(sizeof(int32_t) * pool_cap);
    double *ps = malloc(sizeof(double) * pool_cap);
    int32_t *tmp = malloc(sizeof(int32_t) * (size_t)(D > 0 ? D : 1) + sizeof(int32_t));
    int32_t *tmp2 = malloc(sizeof(int32_t) * (size_t)(D > 0 ? D : 1) + sizeof(int32_t));
    if (!cand || !rseq || !pp || !pr || !ps || !tmp || !tmp2) {
        free(cand); free(rseq); free(pp); free(pr); free(ps); free(tmp); free(tmp2);
        return -OC_ERR_NOMEM;
    }
    for (int d = 0; d < D; ++d) oc_topw(logp + (size_t)d * V, V, W, cand + d * W, NULL);
    parent[0] = -1; token[0] = -1; depth[0] = 0; score[0] = 0.0;
    int n = 1, np = 0;
    if (D > 0 && N > 0) { pp[0] = 0; pr[0] = 0; ps[0] = logp[cand[0]]; np = 1; }
    while (n <= N && np > 0) {
        /* the best pool entry: largest score, then smallest rank sequence */
        int bi = 0;
        for (int i = 1; i < np; ++i) {
            if (ps[i] > ps[bi]) { bi = i; continue; }
            if (ps[i] < ps[bi]) continue;
            int li = depth[pp[i]] + 1, lb = depth[pp[bi]] + 1;
            memcpy(tmp, rseq + (size_t)pp[i] * D, sizeof(int32_t) * (li - 1)); tmp[li - 1] = pr[i];
            memcpy(tmp2, rseq + (size_t)pp[bi] * D, sizeof(int32_t) * (lb - 1)); tmp2[lb - 1] = pr[bi];
            if (rankseq_less(tmp, li, tmp2, lb)) bi = i;
        }
        const int par = pp[bi], rk = pr[bi];
        const double sc = ps[bi];
        pp[bi] = pp[np - 1]; pr[bi] = pr[np - 1]; ps[bi] = ps[np - 1]; --np;
        const int d = depth[par] + 1;
        parent[n] = par; depth[n] = d; score[n] = sc; token[n] = cand[(d - 1) * W + rk];
        memcpy(rseq + (size_t)n * D, rseq + (size_t)par * D, sizeof(int32_t) * (d - 1));
        rseq[(size_t)n * D + d - 1] = rk;
        if (rk + 1 < W) {   /* next sibling */
            pp[np] = par; pr[np] = rk + 1; ps[np] = score[par] + logp[(size_t)(d - 1) * V + cand[(d - 1) * W + rk + 1]];
            ++np;
        }
        if (d < D) {   /* best child */
            pp[np] = n; pr[np] = 0; ps[np] = sc + logp[(size_t)d * V + cand[d * W]];
            ++np;
        }
        ++n;
    }
    free(cand); free(rseq); free(pp); free(pr); free(ps); free(tmp); free(tmp2);
    return n;
}

/*
 * Greedy acceptance on a verified tree: from the root, follow the child
 * whose token equals the AR argmax g of the current node while one exists
 * (siblings hold distinct tokens); emit the followed tokens and then g of
 * the last node reached.  path[0 .. m] = the rows of the accepted root path
 * (path[0] = 0); emit[0 .. m] the tokens.  Returns n = m + 1 in [1, depth
 * + 1].  A chain reduces to oc_consensus_greedy.
 */
int oc_tree_accept(const int32_t *parent, const int32_t *token, int R, const int32_t *g, int32_t *emit,
                   int32_t *path)
{
    int cur = 0, m = 0;
    path[0] = 0;
    for (;;) {
        int next = -1;
        for (int c = cur + 1; c < R && next < 0; ++c)
            if (parent[c] == cur && token[c] == g[cur]) next = c;
        if (next < 0) break;
        emit[m++] = token[next];
        path[m] = next;
        cur = next;
    }
    emit[m] = g[cur];
    return m + 1;
}

/* Commit of an accepted tree path: the K/V of path row path[i] (cache slot
 * t + path[i]) move to slot t + i, for i = 1 .. m, in every layer.  path[i]
 * >= i and increasing, so ascending i never overwrites a slot still to be
 * read. */
void oc_tree_commit_kv(double *kc, double *vc, int n_layers, int cap, int kn, int t, const int32_t *path, int m)
{
    for (int l = 0; l < n_layers; ++l) {
        double *kl = kc + (size_t)l * cap * kn, *vl = vc + (size_t)l * cap * kn;
        for (int i = 1; i <= m; ++i) {
            memmove(kl + (size_t)(t + i) * kn, kl + (size_t)(t + path[i]) * kn, sizeof(double) * kn);
            memmove(vl + (size_t)(t + i) * kn, vl + (size_t)(t + path[i]) * kn, sizeof(double) * kn);
        }
    }
}

/*
 * Greedy decoding with tree verification: every cycle one diffusion draft
 * of K rows (oc_draft at T = 0), log-softmax of its rows 0 .. K-2 (the
 * tokens at depths 1 .. K-1), a best-first tree of `nodes` prefixes with W
 * candidates per depth, one tree-masked AR forward of the root plus the
 * nodes, oc_tree_accept and the K/V compaction; the committed length grows
 * by n.  With W = 1 and nodes = K - 1 the tree is the draft chain and every
 * cycle equals oc_generate's.  out / n_per_cycle / cycles / t as there;
 * kc_out, vc_out (may be NULL): the cache, rows >= t zeroed, with capacity
 * P + N + nodes + 1.
 */
int oc_generate_tree(const oc_cfg *c, const oc_model *w, const int32_t *prompt, int P, int K, int W, int nodes,
                     int N, int32_t *out, int32_t *n_per_cycle, int *n_cycles, double *kc_out, double *vc_out,
                     int *t_out)
{
    if (!c || !w || !prompt || P < 1 || N < 1 || K < 1 || W < 1 || W > c->vocab || nodes < 0) return OC_ERR_ARG;
    const int V = c->vocab, D = K - 1;
    const int cap = P + N + nodes + 1;
    const size_t kn = (size_t)c->n_kv_heads * c->head_dim;
    const size_t csz = (size_t)c->n_layers * cap * kn;
    double *kc = calloc(csz, sizeof(double)), *vc = calloc(csz, sizeof(double));
    int32_t *draft = malloc(sizeof(int32_t) * K);
    double *z = malloc(sizeof(double) * (size_t)K * V);
    double *lp = malloc(sizeof(double) * (size_t)(D > 0 ? D : 1) * V);
    int32_t *par = malloc(sizeof(int32_t) * (nodes + 1)), *tok = malloc(sizeof(int32_t) * (nodes + 1));
    int32_t *dep = malloc(sizeof(int32_t) * (nodes + 1)), *g = malloc(sizeof(int32_t) * (nodes + 1));
    int32_t *emit = malloc(sizeof(int32_t) * (nodes + 1)), *path = malloc(sizeof(int32_t) * (nodes + 1));
    double *sc = malloc(sizeof(double) * (nodes + 1));
    double *zt = malloc(sizeof(double) * (size_t)(nodes + 1) * V);
    int rc = OC_OK;
    if (!kc || !vc || !draft || !z || !lp || !par || !tok || !dep || !g || !emit || !path || !sc || !zt) {
        rc = OC_ERR_NOMEM;
        goto done;
    }
    int t = oc_prefill(c, w, prompt, P, kc, vc, cap);
    if (t < 0) { rc = -t; goto done; }
    int32_t anchor = prompt[P - 1];
    int produced = 0, cycles = 0;
    while (produced < N) {
        rc = oc_draft(c, w, kc, vc, cap, t, anchor, K, 0.0, 0, 0, draft, NULL, z, NULL);
        if (rc) goto done;
        for (int d = 0; d < D; ++d) {   /* log-softmax at T = 1 */
            const double *zr = z + (size_t)d * V;
            double m = -INFINITY, s = 0.0;
            for (int v = 0; v < V; ++v) if (zr[v] > m) m = zr[v];
            for (int v = 0; v < V; ++v) s += exp(zr[v] - m);
            for (int v = 0; v < V; ++v) lp[(size_t)d * V + v] = zr[v] - m - log(s);
        }
        const int R = oc_tree_build(lp, D, V, W, nodes, par, tok, dep, sc);
        if (R < 0) { rc = -R; goto done; }
        tok[0] = anchor;
        rc = oc_forward_tree(c, w, tok, par, R, t, kc, vc, cap, zt);
        if (rc) goto done;
        for (int r = 0; r < R; ++r) g[r] = oc_argmax(zt + (size_t)r * V, V, NULL);
        const int n = oc_tree_accept(par, tok, R, g, emit, path);
        oc_tree_commit_kv(kc, vc, c->n_layers, cap, (int)kn, t, path, n - 1);
        t += n;
        anchor = emit[n - 1];
        for (int i = 0; i < n && produced < N; ++i) out[produced++] = emit[i];
        if (n_per_cycle) n_per_cycle[cycles] = n;
        ++cycles;
    }
    if (n_cycles) *n_cycles = cycles;
    if (t_out) *t_out = t;
    if (kc_out || vc_out) {
        for (int l = 0; l < c->n_layers; ++l) {
            memset(kc + ((size_t)l * cap + t) * kn, 0, sizeof(double) * (size_t)(cap - t) * kn);
            memset(vc + ((size_t)l * cap + t) * kn, 0, sizeof(double) * (size_t)(cap - t) * kn);
        }
        if (kc_out) memcpy(kc_out, kc, sizeof(double) * csz);
        if (vc_out) memcpy(vc_out, vc, sizeof(double) * csz);
    }
done:
    free(kc); free(vc); free(draft); free(z); free(lp); free(par); free(tok); free(dep); free(g); free(emit);
    free(path); free(sc); free(zt);
    return rc;
}

/* ------------------------------------------------------------------------ */
/* Adaptive block length (paper notes §7.4 and §9.6: SV's information-gain   */
/* signal deciding how many drafted tokens to verify, suggested for Orthrus; */
/* no rule is given).  Reading: the entropy of each draft row's distribution */
/* is the signal; a cycle verifies the drafted tokens while their rows'      */
/* entropies stay at or below a threshold.  Greedy only.                     */
/* ------------------------------------------------------------------------ */

/* Entropy (nats) of softmax(z) at T = 1: H = LSE - sum_v p_v z_v. */
double oc_entropy(const double *z, int V)
{
    double m = -INFINITY, s = 0.0, e = 0.0;
    for (int v = 0; v < V; ++v) if (z[v] > m) m = z[v];
    for (int v = 0; v < V; ++v) s += exp(z[v] - m);
    const double lse = m + log(s);
    for (int v = 0; v < V; ++v) e += exp(z[v] - lse) * z[v];
    return lse - e;
}

/* The verify length for one cycle: 1 + the number of leading drafted tokens
 * y_1, y_2, ... (y_k comes from draft row k-1) whose rows have entropy <=
 * h_max, at most K.  H [K]: the draft rows' entropies. */
int oc_adaptive_len(const double *H, int K, double h_max)
{
    int k = 1;
    while (k < K && H[k - 1] <= h_max) ++k;
    return k;
}

/*
 * Greedy decoding with an adaptive block length: every cycle drafts K rows
 * (oc_draft, T = 0), takes Kt = oc_adaptive_len(entropies, K, h_max), runs
 * the AR verification of [anchor, y_1 .. y_{Kt-1}] and the greedy consensus
 * over those Kt rows.  Writes out / n_per_cycle / k_per_cycle (the Kt of
 * each cycle) / cycles / t; kc_out, vc_out as oc_generate_iter's (capacity
 * P + N + K).  h_max = +inf is the fixed-K cycle; h_max < 0 verifies the
 * anchor alone (plain AR).
 */
int oc_generate_adaptive(const oc_cfg *c, const oc_model *w, const int32_t *prompt, int P, int K, double h_max,
                         int N, int32_t *out, int32_t *n_per_cycle, int32_t *k_per_cycle, int *n_cycles,
                         double *kc_out, double *vc_out, int *t_out)
{
    if (!c || !w || !prompt || P < 1 || N < 1 || K < 1) return OC_ERR_ARG;
    const int V = c->vocab;
    const int cap = P + N + K;
    const size_t kn = (size_t)c->n_kv_heads * c->head_dim;
    const size_t csz = (size_t)c->n_layers * cap * kn;
    double *kc = calloc(csz, sizeof(double)), *vc = calloc(csz, sizeof(double));
    int32_t *draft = malloc(sizeof(int32_t) * K), *g = malloc(sizeof(int32_t) * K);
    int32_t *emit = malloc(sizeof(int32_t) * K);
    double *z = malloc(sizeof(double) * (size_t)K * V), *H = malloc(sizeof(double) * K);
    int rc = OC_OK;
    if (!kc || !vc || !draft || !g || !emit || !z || !H) { rc = OC_ERR_NOMEM; goto done; }
    int t = oc_prefill(c, w, prompt, P, kc, vc, cap);
    if (t < 0) { rc = -t; goto done; }
    int32_t anchor = prompt[P - 1];
    int produced = 0, cycles = 0;
    while (produced < N) {
        rc = oc_draft(c, w, kc, vc, cap, t, anchor, K, 0.0, 0, 0, draft, NULL, z, NULL);
        if (rc) goto done;
        for (int k = 0; k < K; ++k) H[k] = oc_entropy(z + (size_t)k * V, V);
        const int Kt = oc_adaptive_len(H, K, h_max);
        rc = oc_verify(c, w, kc, vc, cap, t, anchor, draft, Kt, 0.0, g, NULL, NULL, NULL);
        if (rc) goto done;
        const int n = oc_consensus_greedy(draft, g, Kt, emit);
        t += n;
        anchor = emit[n - 1];
        for (int i = 0; i < n && produced < N; ++i) out[produced++] = emit[i];
        if (n_per_cycle) n_per_cycle[cycles] = n;
        if (k_per_cycle) k_per_cycle[cycles] = Kt;
        ++cycles;
    }
    if (n_cycles) *n_cycles = cycles;
    if (t_out) *t_out = t;
    if (kc_out || vc_out) {
        for (int l = 0; l < c->n_layers; ++l) {
            memset(kc + ((size_t)l * cap + t) * kn, 0, sizeof(double) * (size_t)(cap - t) * kn);
            memset(vc + ((size_t)l * cap + t) * kn, 0, sizeof(double) * (size_t)(cap - t) * kn);
        }
        if (kc_out) memcpy(kc_out, kc, sizeof(double) * csz);
        if (vc_out) memcpy(vc_out, vc, sizeof(double) * csz);
    }
done:
    free(kc); free(vc); free(draft); free(g); free(emit); free(z); free(H);
    return rc;
}
