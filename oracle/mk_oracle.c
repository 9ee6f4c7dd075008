/*
 * mk_oracle.c -- plain, slow, single-threaded CPU definition of the decode
 * step.  TEST INFRASTRUCTURE ONLY (see mk_oracle.h for what it follows and
 * who may use it).  Every loop is written in the order of the definition;
 * there is no blocking, fusion or reordering.
 */
#include "mk_oracle.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>

/* ---- bf16 storage format ------------------------------------------------ */

double orc_bf16_to_double(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* Round a double to the nearest bf16 value (8 significant bits, float
 * exponent range, gradual underflow), ties to even, then return its bits. */
uint16_t orc_double_to_bf16(double x)
{
    if (isnan(x)) return 0x7FC0;
    if (isinf(x)) return x > 0 ? 0x7F80 : 0xFF80;
    double ax = fabs(x);
    double r;
    if (ax == 0.0) {
        r = 0.0;
    } else if (ax < ldexp(1.0, -126)) {
        /* subnormal range: fixed quantum 2^-133 */
        r = nearbyint(ax / ldexp(1.0, -133)) * ldexp(1.0, -133);
    } else {
        int e;
        double m = frexp(ax, &e);            /* ax = m * 2^e, m in [0.5,1) */
        double s = nearbyint(ldexp(m, 8));   /* 8 significant bits, RNE   */
        r = ldexp(s, e - 8);
    }
    /* largest finite bf16 is (2 - 2^-7) * 2^127 */
    if (r > ldexp(2.0 - ldexp(1.0, -7), 127)) {
        return x > 0 ? 0x7F80 : 0xFF80;
    }
    float f = (float)r;                       /* exact: r has <= 8 bits */
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    uint16_t b = (uint16_t)(u >> 16);
    if (x < 0) b |= 0x8000;
    return b;
}

/* ---- building blocks ---------------------------------------------------- */

/* RMSNorm (Hazy instruction list: "RMSNorm"; MPK rmsnorm_linear_layer). */
void orc_rmsnorm(const double *x, const uint16_t *g, int n, double eps, double *y)
{
    double ss = 0.0;
    for (int i = 0; i < n; ++i) ss += x[i] * x[i];
    double inv = 1.0 / sqrt(ss / (double)n + eps);
    for (int i = 0; i < n; ++i) y[i] = x[i] * inv * orc_bf16_to_double(g[i]);
}

/* Matrix-vector product, W row-major [N][K]. */
void orc_gemv(const uint16_t *W, int N, int K, const double *x, double *y)
{
    for (int r = 0; r < N; ++r) {
        const uint16_t *row = W + (size_t)r * (size_t)K;
        double acc = 0.0;
        for (int k = 0; k < K; ++k) acc += orc_bf16_to_double(row[k]) * x[k];
        y[r] = acc;
    }
}

/* Rotary position embedding, half-split pairing (i, i + d/2), as in the
 * cos/sin tables the MPK walkthrough takes from the HF rotary module. */
void orc_rope(double *v, int d, int pos, double theta)
{
    int half = d / 2;
    for (int i = 0; i < half; ++i) {
        double inv_freq = pow(theta, -2.0 * (double)i / (double)d);
        double ang = (double)pos * inv_freq;
        double c = cos(ang), s = sin(ang);
        double a = v[i], b = v[i + half];
        v[i] = a * c - b * s;
        v[i + half] = b * c + a * s;
    }
}

double orc_silu(double x) { return x / (1.0 + exp(-x)); }

int orc_argmax(const double *v, int n)
{
    int best = 0;
    for (int i = 1; i < n; ++i)
        if (v[i] > v[best]) best = i;
    return best;
}

/* Decode attention with grouped KV heads (MPK attention_layer, one query
 * token against the cache; Hazy "attention matmul and reduction"). */
void orc_attention(const double *q, const uint16_t *kc, const uint16_t *vc,
                   int nq, int nkv, int d, int max_seq, int C, double *out)
{
    int group = nq / nkv;
    double scale = 1.0 / sqrt((double)d);
    double *s = (double *)malloc(sizeof(double) * (size_t)(C > 0 ? C : 1));
    for (int i = 0; i < nq; ++i) {
        int h = i / group;
        const uint16_t *K = kc + (size_t)h * (size_t)max_seq * (size_t)d;
        const uint16_t *V = vc + (size_t)h * (size_t)max_seq * (size_t)d;
        const double *qi = q + (size_t)i * (size_t)d;
        double m = -INFINITY;
        for (int j = 0; j < C; ++j) {
            double dot = 0.0;
            for (int t = 0; t < d; ++t)
                dot += qi[t] * orc_bf16_to_double(K[(size_t)j * d + t]);
            s[j] = dot * scale;
            if (s[j] > m) m = s[j];
        }
        double den = 0.0;
        for (int j = 0; j < C; ++j) {
            s[j] = exp(s[j] - m);
            den += s[j];
        }
        for (int t = 0; t < d; ++t) {
            double acc = 0.0;
            for (int j = 0; j < C; ++j)
                acc += s[j] * orc_bf16_to_double(V[(size_t)j * d + t]);
            out[(size_t)i * d + t] = acc / den;
        }
    }
    free(s);
}

static int cfg_ok(const orc_config *c)
{
    return c && c->layers > 0 && c->hidden > 0 && c->n_q_heads > 0 &&
           c->n_kv_heads > 0 && c->n_q_heads % c->n_kv_heads == 0 &&
           c->head_dim > 0 && c->head_dim % 2 == 0 && c->ffn > 0 &&
           c->vocab > 0 && c->max_seq > 0;
}

static double *dalloc(size_t n) { return (double *)calloc(n ? n : 1, sizeof(double)); }

/* ---- one KV-cached decode step ----------------------------------------- */

int orc_decode_step(const orc_config *cfg, const orc_weights *w,
                    uint16_t *const *kcache, uint16_t *const *vcache,
                    int token, int pos,
                    double *logits, double *hidden,
                    double *q_last, double *attn_last, double *act_last)
{
    if (!cfg_ok(cfg) || token < 0 || token >= cfg->vocab || pos < 0 ||
        pos >= cfg->max_seq)
        return -1;
    const int H = cfg->hidden, nq = cfg->n_q_heads, nkv = cfg->n_kv_heads;
    const int d = cfg->head_dim, F = cfg->ffn, V = cfg->vocab, S = cfg->max_seq;
    const int QD = nq * d, KD = nkv * d;

    double *x = dalloc(H), *xn = dalloc(H), *q = dalloc(QD), *k = dalloc(KD);
    double *v = dalloc(KD), *o = dalloc(QD), *t = dalloc(H), *g = dalloc(F);
    double *u = dalloc(F), *lg = dalloc(V);

    /* embed: x = E[token] */
    for (int i = 0; i < H; ++i)
        x[i] = orc_bf16_to_double(w->embed[(size_t)token * H + i]);

    for (int l = 0; l < cfg->layers; ++l) {
        /* RMSNorm -> q, k, v projections */
        orc_rmsnorm(x, w->attn_norm[l], H, cfg->rms_eps, xn);
        orc_gemv(w->wq[l], QD, H, xn, q);
        orc_gemv(w->wk[l], KD, H, xn, k);
        orc_gemv(w->wv[l], KD, H, xn, v);
        /* RoPE on every q and k head */
        for (int h = 0; h < nq; ++h) orc_rope(q + (size_t)h * d, d, pos, cfg->rope_theta);
        for (int h = 0; h < nkv; ++h) orc_rope(k + (size_t)h * d, d, pos, cfg->rope_theta);
        /* append k, v at pos (bf16 storage) */
        for (int h = 0; h < nkv; ++h)
            for (int i = 0; i < d; ++i) {
                size_t at = ((size_t)h * S + (size_t)pos) * d + i;
                kcache[l][at] = orc_double_to_bf16(k[(size_t)h * d + i]);
                vcache[l][at] = orc_double_to_bf16(v[(size_t)h * d + i]);
            }
        /* attention over positions 0..pos */
        orc_attention(q, kcache[l], vcache[l], nq, nkv, d, S, pos + 1, o);
        /* O projection + residual */
        orc_gemv(w->wo[l], H, QD, o, t);
        for (int i = 0; i < H; ++i) x[i] += t[i];
        /* RMSNorm -> gate, up -> SiLU(gate) * up -> down + residual */
        orc_rmsnorm(x, w->mlp_norm[l], H, cfg->rms_eps, xn);
        orc_gemv(w->wg[l], F, H, xn, g);
        orc_gemv(w->wu[l], F, H, xn, u);
        for (int i = 0; i < F; ++i) g[i] = orc_silu(g[i]) * u[i];
        orc_gemv(w->wd[l], H, F, g, t);
        for (int i = 0; i < H; ++i) x[i] += t[i];
        if (l == cfg->layers - 1) {
            if (q_last) memcpy(q_last, q, sizeof(double) * (size_t)QD);
            if (attn_last) memcpy(attn_last, o, sizeof(double) * (size_t)QD);
            if (act_last) memcpy(act_last, g, sizeof(double) * (size_t)F);
        }
    }
    if (hidden) memcpy(hidden, x, sizeof(double) * (size_t)H);
    /* final RMSNorm -> LM head -> argmax */
    orc_rmsnorm(x, w->final_norm, H, cfg->rms_eps, xn);
    orc_gemv(w->lm_head, V, H, xn, lg);
    int next = orc_argmax(lg, V);
    if (logits) memcpy(logits, lg, sizeof(double) * (size_t)V);

    free(x); free(xn); free(q); free(k); free(v); free(o); free(t); free(g);
    free(u); free(lg);
    return next;
}

/* ---- full recompute (no cache input) ------------------------------------ */

int orc_forward_recompute(const orc_config *cfg, const orc_weights *w,
                          const int *tokens, int n,
                          double *logits, double *hidden)
{
    if (!cfg_ok(cfg) || n <= 0 || n > cfg->max_seq) return -1;
    for (int p = 0; p < n; ++p)
        if (tokens[p] < 0 || tokens[p] >= cfg->vocab) return -1;
    const int H = cfg->hidden, nq = cfg->n_q_heads, nkv = cfg->n_kv_heads;
    const int d = cfg->head_dim, F = cfg->ffn, V = cfg->vocab;
    const int QD = nq * d, KD = nkv * d, group = nq / nkv;

    /* residual stream of every position: X[p][H] */
    double *X = dalloc((size_t)n * H);
    double *xn = dalloc(H), *q = dalloc((size_t)n * QD), *t = dalloc(H);
    double *Kf = dalloc((size_t)n * KD), *Vf = dalloc((size_t)n * KD);
    double *o = dalloc(QD), *g = dalloc(F), *u = dalloc(F), *lg = dalloc(V);
    double *s = dalloc((size_t)n);

    for (int p = 0; p < n; ++p)
        for (int i = 0; i < H; ++i)
            X[(size_t)p * H + i] = orc_bf16_to_double(w->embed[(size_t)tokens[p] * H + i]);

    for (int l = 0; l < cfg->layers; ++l) {
        /* projections of all positions; K and V kept at bf16 precision */
        for (int p = 0; p < n; ++p) {
            double *xp = X + (size_t)p * H;
            double *kp = Kf + (size_t)p * KD, *vp = Vf + (size_t)p * KD;
            orc_rmsnorm(xp, w->attn_norm[l], H, cfg->rms_eps, xn);
            orc_gemv(w->wq[l], QD, H, xn, q + (size_t)p * QD);
            orc_gemv(w->wk[l], KD, H, xn, kp);
            orc_gemv(w->wv[l], KD, H, xn, vp);
            for (int h = 0; h < nq; ++h)
                orc_rope(q + (size_t)p * QD + (size_t)h * d, d, p, cfg->rope_theta);
            for (int h = 0; h < nkv; ++h) orc_rope(kp + (size_t)h * d, d, p, cfg->rope_theta);
            for (int i = 0; i < KD; ++i) {
                kp[i] = orc_bf16_to_double(orc_double_to_bf16(kp[i]));
                vp[i] = orc_bf16_to_double(orc_double_to_bf16(vp[i]));
            }
        }
        /* causal attention, then the rest of the layer, per position */
        for (int p = 0; p < n; ++p) {
            double *xp = X + (size_t)p * H;
            for (int i = 0; i < nq; ++i) {
                int h = i / group;
                const double *qi = q + (size_t)p * QD + (size_t)i * d;
                double m = -INFINITY;
                for (int j = 0; j <= p; ++j) {
                    const double *kj = Kf + (size_t)j * KD + (size_t)h * d;
                    double dot = 0.0;
                    for (int e = 0; e < d; ++e) dot += qi[e] * kj[e];
                    s[j] = dot / sqrt((double)d);
                    if (s[j] > m) m = s[j];
                }
                double den = 0.0;
                for (int j = 0; j <= p; ++j) { s[j] = exp(s[j] - m); den += s[j]; }
                for (int e = 0; e < d; ++e) {
                    double acc = 0.0;
                    for (int j = 0; j <= p; ++j)
                        acc += s[j] * Vf[(size_t)j * KD + (size_t)h * d + e];
                    o[(size_t)i * d + e] = acc / den;
                }
            }
            orc_gemv(w->wo[l], H, QD, o, t);
            for (int i = 0; i < H; ++i) xp[i] += t[i];
            orc_rmsnorm(xp, w->mlp_norm[l], H, cfg->rms_eps, xn);
            orc_gemv(w->wg[l], F, H, xn, g);
            orc_gemv(w->wu[l], F, H, xn, u);
            for (int i = 0; i < F; ++i) g[i] = orc_silu(g[i]) * u[i];
            orc_gemv(w->wd[l], H, F, g, t);
            for (int i = 0; i < H; ++i) xp[i] += t[i];
        }
    }
    double *xl = X + (size_t)(n - 1) * H;
    if (hidden) memcpy(hidden, xl, sizeof(double) * (size_t)H);
    orc_rmsnorm(xl, w->final_norm, H, cfg->rms_eps, xn);
    orc_gemv(w->lm_head, V, H, xn, lg);
    int next = orc_argmax(lg, V);
    if (logits) memcpy(logits, lg, sizeof(double) * (size_t)V);

    free(X); free(xn); free(q); free(t); free(Kf); free(Vf); free(o); free(g);
    free(u); free(lg); free(s);
    return next;
}
