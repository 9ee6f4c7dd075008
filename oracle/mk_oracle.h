/*
 * mk_oracle.h -- plain CPU definition of one decode step of a Llama-style
 * decoder, used as the parity oracle for the persistent decode megakernel.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may include, link
 * or call this library: only tests/, __graft_entry__.smoke() and the CPU
 * baseline leg of bench.py use it.  It shares no code, header, table or
 * constant with the CUDA library.
 *
 * What it follows (pages of the reference topic "persistent decode
 * megakernel"):
 *  - the op sequence of one decoder layer and the model tail: the MPK
 *    walkthrough (zizhi168.cn/news/174794, section 3.3.1 "计算图构建过程":
 *    embed_layer, rmsnorm_linear_layer over fused q/k/v grouped per KV head,
 *    attention_layer with k/v caches and cos/sin position tables,
 *    linear_with_residual_layer, rmsnorm_linear_layer over fused gate/up,
 *    silu_mul_linear_with_residual_layer, final rmsnorm_linear_layer to the
 *    LM head, argmax_partial_layer + argmax_reduce_layer) and the Hazy
 *    megakernel instruction list (sfrk.com.cn/ruanjian/202506/86466,
 *    paragraph on the fused instructions: RMSNorm+QKV+RoPE, attention
 *    matmul and reduction, O-projection+residual, MLP RMSNorm+gate SiLU+up,
 *    down projection+residual, final RMSNorm+LM head).
 *  - The pages print no formula; the readings taken (RMSNorm with eps,
 *    half-split RoPE as produced by the HF rotary tables the walkthrough
 *    feeds in, GQA head grouping, 1/sqrt(d) scale, bf16 KV storage,
 *    lowest-index argmax ties) are listed in the design notes.
 *
 * Arithmetic is IEEE double throughout.  Weights and KV entries are bf16
 * bit patterns (uint16) widened exactly to double; a new K/V entry is
 * rounded to bf16 (round to nearest, ties to even) when it is stored, as
 * the cache format requires, and read back widened.
 */
#ifndef MK_ORACLE_H
#define MK_ORACLE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct orc_config {
    int layers;      /* decoder layers */
    int hidden;      /* H */
    int n_q_heads;   /* nq */
    int n_kv_heads;  /* nkv, divides nq */
    int head_dim;    /* d, even */
    int ffn;         /* F */
    int vocab;       /* V */
    int max_seq;     /* KV capacity per sequence (positions 0..max_seq-1) */
    double rope_theta;
    double rms_eps;
} orc_config;

/* All pointers are host pointers to bf16 bit patterns, row-major. */
typedef struct orc_weights {
    const uint16_t *embed;       /* [V][H] */
    const uint16_t *lm_head;     /* [V][H]; may equal embed (tied) */
    const uint16_t *final_norm;  /* [H] */
    const uint16_t *const *attn_norm; /* [layers] -> [H] */
    const uint16_t *const *mlp_norm;  /* [layers] -> [H] */
    const uint16_t *const *wq;   /* [layers] -> [nq*d][H] */
    const uint16_t *const *wk;   /* [layers] -> [nkv*d][H] */
    const uint16_t *const *wv;   /* [layers] -> [nkv*d][H] */
    const uint16_t *const *wo;   /* [layers] -> [H][nq*d] */
    const uint16_t *const *wg;   /* [layers] -> [F][H] */
    const uint16_t *const *wu;   /* [layers] -> [F][H] */
    const uint16_t *const *wd;   /* [layers] -> [H][F] */
} orc_weights;

/* bf16 <-> double.  to_bf16 rounds to nearest, ties to even, directly from
 * the double (no intermediate float rounding); NaN -> 0x7FC0. */
double   orc_bf16_to_double(uint16_t b);
uint16_t orc_double_to_bf16(double x);

/* y = x / sqrt(mean(x^2) + eps) * g   (g bf16 [n]) */
void orc_rmsnorm(const double *x, const uint16_t *g, int n, double eps, double *y);

/* y[N] = W[N][K] x[K] */
void orc_gemv(const uint16_t *W, int N, int K, const double *x, double *y);

/* Rotate one head vector v[d] in place for position pos: pairs (i, i+d/2),
 * angle pos * theta^(-2i/d). */
void orc_rope(double *v, int d, int pos, double theta);

double orc_silu(double x);

/* Index of the maximum of v[n]; ties go to the lowest index. */
int orc_argmax(const double *v, int n);

/* Grouped-query decode attention for one sequence.
 * q[nq][d] (already rotated); kc, vc: bf16 [nkv][max_seq][d];
 * attends positions 0..C-1; out[nq][d]. q head i uses KV head i/(nq/nkv). */
void orc_attention(const double *q, const uint16_t *kc, const uint16_t *vc,
                   int nq, int nkv, int d, int max_seq, int C, double *out);

/* One KV-cached decode step of one sequence at position pos with input
 * token `token`.  kcache[l], vcache[l] point at this sequence's bf16
 * [nkv][max_seq][d] cache of layer l; entry `pos` of every layer is written.
 * Optional outputs (NULL to skip): logits[V], hidden[H] (residual stream
 * after the last layer, before the final norm), and the last layer's
 * q[nq*d] (rotated), attention output attn[nq*d], MLP activation act[F].
 * Returns argmax(logits), or -1 on bad arguments. */
int orc_decode_step(const orc_config *cfg, const orc_weights *w,
                    uint16_t *const *kcache, uint16_t *const *vcache,
                    int token, int pos,
                    double *logits, double *hidden,
                    double *q_last, double *attn_last, double *act_last);

/* Full recompute of positions 0..n-1 with no cache input: every layer is
 * evaluated for all positions (K/V of each position stored as bf16, like the
 * cache), causal attention.  Outputs the logits / hidden state of the last
 * position.  A separate code path from orc_decode_step, used to pin it.
 * Returns argmax(logits) of the last position, or -1 on bad arguments. */
int orc_forward_recompute(const orc_config *cfg, const orc_weights *w,
                          const int *tokens, int n,
                          double *logits, double *hidden);

#ifdef __cplusplus
}
#endif
#endif
