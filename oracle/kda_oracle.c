/*
 * kda_oracle.c — plain, slow, fp64 CPU oracle for the Kimi Delta Attention (KDA)
 * gated delta rule and its layer prologue / epilogue.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may call, link or load
 * this file; only the tests, the package's smoke check and the benchmark's CPU
 * baseline leg do.  It shares no code, header or constant with the CUDA library.
 *
 * Everything here is written straight from the definitions, token by token, with
 * no chunking, blocking or reordering: a reader should be able to check each
 * function against the text it cites by eye.  All arithmetic is double precision;
 * callers pass inputs already rounded to the I/O dtype the GPU sees.
 *
 * Layouts (row-major, last index fastest):
 *   q, k, g        [B, T, H, dk]
 *   v, o           [B, T, H, dv]
 *   beta           [B, T, H]
 *   state          [B, H, dk, dv]
 *
 * Sources (pages about the Kimi-K3 hybrid model):
 *   - open-model-atlas "Kimi-K3 ?inspect=blocks", self.layers: 69 KDA layers keep
 *     a state of fixed size between calls (the dk x dv matrix per head below).
 *   - maxtext PR #5548 review, item 2: the KDA tensors A_log [heads], dt_bias
 *     [heads*dk], {q,k,v}_conv1d.weight [heads*d, 1, 4] and o_norm.weight [dv] are
 *     kept in F32, and exp(A_log) drives the state decay.
 *   - open-model-atlas "Kimi-K3", config.json text_config / linear_attn_config:
 *     head_dim 128, num_heads 96, short_conv_kernel_size 4.
 *   - atlas.klimoza.dev "KDA layers > MoE input", KimiRMSNorm excerpt: fp32
 *     normalise by rsqrt(mean(x^2) + eps), cast back to the input dtype, times gain.
 *   - maxtext PR #5543 "MLA: optional sigmoid output gate", What, item 1: the
 *     output-gate pattern out = attn * sigmoid(g_proj(x)).
 *
 * The recurrence (the KDA gated delta rule), per head, per token t:
 *     alpha_t = exp(g_t)                       (per-channel decay, g_t <= 0)
 *     S'      = Diag(alpha_t) S_{t-1}          (decay first)
 *     u_t     = beta_t (v_t - S'^T k_t)        (delta-rule correction along k_t)
 *     S_t     = S' + k_t u_t^T                 (write with k v^T, strength beta)
 *     o_t     = S_t^T q_t                      (read with q after the update)
 * i.e. S_t = (I - beta_t k_t k_t^T) Diag(alpha_t) S_{t-1} + beta_t k_t v_t^T.
 * Query scale is 1 (no 1/sqrt(dk)); q and k are unit-normalised upstream.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

static void set_threads(int nthreads)
{
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#else
    (void)nthreads;
#endif
}

int kda_oracle_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* One head of the recurrence.  S is the head's dk x dv state (in/out).
 * qh/kh/gh point at token 0 of this head with a row stride of `sk` doubles,
 * vh/oh with row stride `sv`, bh with stride `sb`.
 * delta = 0 drops the correction term (u_t = beta_t v_t); it exists only so the
 * tests can check the write/read wiring against textbook linear attention. */
static void head_recurrence(const double *qh, const double *kh, const double *vh,
                            const double *gh, const double *bh, double *S, double *oh,
                            int T, int dk, int dv, size_t sk, size_t sv, size_t sb,
                            int delta, double *kS, double *u)
{
    for (int t = 0; t < T; ++t) {
        const double *qt = qh + (size_t)t * sk;
        const double *kt = kh + (size_t)t * sk;
        const double *gt = gh + (size_t)t * sk;
        const double *vt = vh + (size_t)t * sv;
        const double beta = bh[(size_t)t * sb];

        /* S' = Diag(exp(g_t)) S */
        for (int c = 0; c < dk; ++c) {
            const double a = exp(gt[c]);
            double *row = S + (size_t)c * dv;
            for (int j = 0; j < dv; ++j) row[j] *= a;
        }
        /* u = beta (v - S'^T k) */
        for (int j = 0; j < dv; ++j) kS[j] = 0.0;
        if (delta) {
            for (int c = 0; c < dk; ++c) {
                const double *row = S + (size_t)c * dv;
                for (int j = 0; j < dv; ++j) kS[j] += kt[c] * row[j];
            }
        }
        for (int j = 0; j < dv; ++j) u[j] = beta * (vt[j] - kS[j]);
        /* S = S' + k u^T */
        for (int c = 0; c < dk; ++c) {
            double *row = S + (size_t)c * dv;
            for (int j = 0; j < dv; ++j) row[j] += kt[c] * u[j];
        }
        /* o = S^T q */
        if (oh) {
            double *ot = oh + (size_t)t * sv;
            for (int j = 0; j < dv; ++j) ot[j] = 0.0;
            for (int c = 0; c < dk; ++c) {
                const double *row = S + (size_t)c * dv;
                for (int j = 0; j < dv; ++j) ot[j] += qt[c] * row[j];
            }
        }
    }
}

/* Token-by-token recurrence over a whole batch.
 * s0 may be NULL (zero initial state); sT may be NULL (final state not wanted);
 * o may be NULL (outputs not wanted).  Heads (b, h) are independent and run in
 * parallel with OpenMP. */
void kda_oracle_recurrent(const double *q, const double *k, const double *v, const double *g,
                          const double *beta, const double *s0, double *o, double *sT,
                          int B, int T, int H, int dk, int dv, int delta, int nthreads)
{
    set_threads(nthreads);
    const size_t sk = (size_t)H * dk, sv = (size_t)H * dv, sb = (size_t)H;
#pragma omp parallel
    {
        double *S = (double *)malloc(sizeof(double) * (size_t)dk * dv);
        double *kS = (double *)malloc(sizeof(double) * (size_t)dv);
        double *u = (double *)malloc(sizeof(double) * (size_t)dv);
#pragma omp for schedule(dynamic, 1)
        for (int bh = 0; bh < B * H; ++bh) {
            const int b = bh / H, h = bh % H;
            const size_t st_off = (size_t)bh * dk * dv;
            if (s0) memcpy(S, s0 + st_off, sizeof(double) * (size_t)dk * dv);
            else memset(S, 0, sizeof(double) * (size_t)dk * dv);
            const size_t tok0 = (size_t)b * T * H + h; /* (b, t=0, h) */
            head_recurrence(q + tok0 * dk, k + tok0 * dk, v + tok0 * dv, g + tok0 * dk,
                            beta + tok0, S, o ? o + tok0 * dv : NULL, T, dk, dv, sk, sv, sb,
                            delta, kS, u);
            if (sT) memcpy(sT + st_off, S, sizeof(double) * (size_t)dk * dv);
        }
        free(S);
        free(kS);
        free(u);
    }
}

/* Gradients of the recurrence (reverse mode, token by token, exact in fp64).
 * Given dO = dL/do [B, T, H, dv] and dST = dL/dS_T [B, H, dk, dv] (NULL: zero), writes
 * dq, dk, dg [B, T, H, dk], dv [B, T, H, dv], dbeta [B, T, H] and ds0 = dL/dS_0
 * [B, H, dk, dv] (NULL: not wanted).  The pages' training runs differentiate the layer
 * (maxtext PR #5550, its jax.grad test and the C4 training steps); the steps below are
 * the chain rule applied to each line of the forward step, last token first:
 *   S' = Diag(a) S_{t-1}, a = exp(g_t);  r = S'^T k;  u = beta (v - r);  S_t = S' + k u^T;
 *   o_t = S_t^T q.
 * The forward states S_0 .. S_{T-1} are kept (one head at a time). */
void kda_oracle_recurrent_backward(const double *q, const double *k, const double *v,
                                   const double *g, const double *beta, const double *s0,
                                   const double *dO, const double *dST, double *dq, double *dk,
                                   double *dv_, double *dg, double *dbeta, double *ds0, int B,
                                   int T, int H, int dk_, int dv, int nthreads)
{
    set_threads(nthreads);
    const size_t sk = (size_t)H * dk_, sv = (size_t)H * dv, DD = (size_t)dk_ * dv;
#pragma omp parallel
    {
        double *Sall = (double *)malloc(sizeof(double) * DD * (size_t)(T + 1));
        double *U = (double *)malloc(sizeof(double) * (size_t)(T > 0 ? T : 1) * dv);
        double *R = (double *)malloc(sizeof(double) * (size_t)(T > 0 ? T : 1) * dv);
        double *Sp = (double *)malloc(sizeof(double) * DD);
        double *dS = (double *)malloc(sizeof(double) * DD);
        double *du = (double *)malloc(sizeof(double) * (size_t)dv);
        double *da = (double *)malloc(sizeof(double) * (size_t)dv);
#pragma omp for schedule(dynamic, 1)
        for (int bh = 0; bh < B * H; ++bh) {
            const int b = bh / H, h = bh % H;
            const size_t tok0 = (size_t)b * T * H + h;
            /* forward: S_0 .. S_T, u_t and r_t = S'^T k */
            if (s0) memcpy(Sall, s0 + (size_t)bh * DD, sizeof(double) * DD);
            else memset(Sall, 0, sizeof(double) * DD);
            for (int t = 0; t < T; ++t) {
                const size_t tk = (tok0 + (size_t)t * H) * dk_, tv = (tok0 + (size_t)t * H) * dv;
                const double *Sprev = Sall + (size_t)t * DD;
                double *Snext = Sall + (size_t)(t + 1) * DD;
                for (int c = 0; c < dk_; ++c) {
                    const double a = exp(g[tk + c]);
                    for (int j = 0; j < dv; ++j) Snext[(size_t)c * dv + j] = a * Sprev[(size_t)c * dv + j];
                }
                const double bt = beta[tok0 + (size_t)t * H];
                for (int j = 0; j < dv; ++j) {
                    double r = 0.0;
                    for (int c = 0; c < dk_; ++c) r += Snext[(size_t)c * dv + j] * k[tk + c];
                    R[(size_t)t * dv + j] = r;
                    U[(size_t)t * dv + j] = bt * (v[tv + j] - r);
                }
                for (int c = 0; c < dk_; ++c)
                    for (int j = 0; j < dv; ++j) Snext[(size_t)c * dv + j] += k[tk + c] * U[(size_t)t * dv + j];
            }
            /* reverse sweep */
            if (dST) memcpy(dS, dST + (size_t)bh * DD, sizeof(double) * DD);
            else memset(dS, 0, sizeof(double) * DD);
            for (int t = T - 1; t >= 0; --t) {
                const size_t tk = (tok0 + (size_t)t * H) * dk_, tv = (tok0 + (size_t)t * H) * dv;
                const size_t tb = tok0 + (size_t)t * H;
                const double *St = Sall + (size_t)(t + 1) * DD, *Sprev = Sall + (size_t)t * DD;
                const double bt = beta[tb];
                /* o_t = S_t^T q_t:  dS_t += q do^T,  dq = S_t do */
                for (int c = 0; c < dk_; ++c) {
                    double acc = 0.0;
                    for (int j = 0; j < dv; ++j) {
                        dS[(size_t)c * dv + j] += q[tk + c] * dO[tv + j];
                        acc += St[(size_t)c * dv + j] * dO[tv + j];
                    }
                    dq[tk + c] = acc;
                }
                /* S_t = S' + k u^T:  du = dS^T k,  dk = dS u */
                for (int j = 0; j < dv; ++j) {
                    double acc = 0.0;
                    for (int c = 0; c < dk_; ++c) acc += dS[(size_t)c * dv + j] * k[tk + c];
                    du[j] = acc;
                }
                double dbt = 0.0;
                for (int j = 0; j < dv; ++j) {
                    /* u = beta (v - r) */
                    dbt += du[j] * (v[tv + j] - R[(size_t)t * dv + j]);
                    dv_[tv + j] = bt * du[j];
                    da[j] = -bt * du[j];
                }
                dbeta[tb] = dbt;
                for (int c = 0; c < dk_; ++c) {
                    const double a = exp(g[tk + c]);
                    double acc_k = 0.0, acc_g = 0.0;
                    for (int j = 0; j < dv; ++j) {
                        const double sp = a * Sprev[(size_t)c * dv + j];
                        acc_k += dS[(size_t)c * dv + j] * U[(size_t)t * dv + j] + sp * da[j];
                        /* r = S'^T k:  dS' = dS + k da^T */
                        const double dsp = dS[(size_t)c * dv + j] + k[tk + c] * da[j];
                        /* S' = Diag(exp g) S_{t-1}:  dg_c = sum_j dS'_cj S'_cj,  dS_{t-1} = Diag(exp g) dS' */
                        acc_g += dsp * sp;
                        dS[(size_t)c * dv + j] = a * dsp;
                    }
                    dk[tk + c] = acc_k;
                    dg[tk + c] = acc_g;
                }
            }
            if (ds0) memcpy(ds0 + (size_t)bh * DD, dS, sizeof(double) * DD);
        }
        free(Sall);
        free(U);
        free(R);
        free(Sp);
        free(dS);
        free(du);
        free(da);
    }
}

/* One decode step: the recurrence for a single token per sequence, state updated
 * in place.  q, k, g: [B, H, dk]; v, o: [B, H, dv]; beta: [B, H]; state [B, H, dk, dv]. */
void kda_oracle_decode(const double *q, const double *k, const double *v, const double *g,
                       const double *beta, double *state, double *o, int B, int H, int dk,
                       int dv, int nthreads)
{
    /* A decode step is the recurrence with T = 1; the batch layout [B, 1, H, .]
     * coincides with [B, H, .]. */
    kda_oracle_recurrent(q, k, v, g, beta, state, o, state, B, 1, H, dk, dv, 1, nthreads);
}

/* ---------------------------------------------------------------- prologue */

static double silu(double x) { return x / (1.0 + exp(-x)); }

static double softplus(double x)
{
    /* log(1 + e^x), evaluated without overflow */
    return x > 0.0 ? x + log1p(exp(-x)) : log1p(exp(x));
}

static double sigmoid(double x) { return 1.0 / (1.0 + exp(-x)); }

/* Depthwise causal short convolution (kernel 4) followed by SiLU.
 * x: [B, T, C] (C = H*d channels), w: [C, 4] (the [C, 1, 4] checkpoint tensor),
 * y: [B, T, C].  PyTorch Conv1d convention with left zero padding 3:
 *   y[t, c] = SiLU( sum_{i=0..3} w[c, i] * x[t - 3 + i, c] ),  x[<0] = 0.
 * (open-model-atlas "Kimi-K3" linear_attn_config: short_conv_kernel_size 4;
 *  maxtext PR #5548 review, item 2: {q,k,v}_conv1d.weight [heads*d, 1, 4].) */
void kda_oracle_short_conv_silu(const double *x, const double *w, double *y, int B, int T,
                                int C, int apply_silu, int nthreads)
{
    set_threads(nthreads);
#pragma omp parallel for schedule(static)
    for (int bc = 0; bc < B * C; ++bc) {
        const int b = bc / C, c = bc % C;
        for (int t = 0; t < T; ++t) {
            double acc = 0.0;
            for (int i = 0; i < 4; ++i) {
                const int ts = t - 3 + i;
                if (ts >= 0) acc += w[(size_t)c * 4 + i] * x[((size_t)b * T + ts) * C + c];
            }
            y[((size_t)b * T + t) * C + c] = apply_silu ? silu(acc) : acc;
        }
    }
}

/* L2 normalisation over the last dim of rows of length d: x / sqrt(sum x^2 + eps). */
void kda_oracle_l2norm(const double *x, double *y, size_t rows, int d, double eps)
{
    for (size_t r = 0; r < rows; ++r) {
        double ss = 0.0;
        for (int c = 0; c < d; ++c) ss += x[r * d + c] * x[r * d + c];
        const double inv = 1.0 / sqrt(ss + eps);
        for (int c = 0; c < d; ++c) y[r * d + c] = x[r * d + c] * inv;
    }
}

/* Per-channel log-decay gate: g = max(-exp(A_log[h]) * softplus(x + dt_bias[h*dk + c]), lb).
 * x: [B, T, H, dk]; A_log: [H]; dt_bias: [H*dk] or NULL (zero); lb = -INFINITY for no bound.
 * (maxtext PR #5548 review, item 2: exp(A_log) drives the state decay, dt_bias is
 *  per channel [heads*dk], both F32.  The Kimi-K3 linear-attention config sets
 *  gate_lower_bound = -5.0 without its formula; the plainest reading, taken here, is a
 *  lower bound on the log-decay itself: per-token decay no stronger than exp(lb).) */
void kda_oracle_gate(const double *x, const double *A_log, const double *dt_bias, double lb,
                     double *g, int B, int T, int H, int dk)
{
    const size_t n = (size_t)B * T * H;
    for (size_t r = 0; r < n; ++r) {
        const int h = (int)(r % H);
        const double scale = exp(A_log[h]);
        for (int c = 0; c < dk; ++c) {
            const double bias = dt_bias ? dt_bias[(size_t)h * dk + c] : 0.0;
            const double v = -scale * softplus(x[r * dk + c] + bias);
            g[r * dk + c] = v < lb ? lb : v;
        }
    }
}

/* beta = sigmoid(x), elementwise. */
void kda_oracle_sigmoid(const double *x, double *y, size_t n)
{
    for (size_t i = 0; i < n; ++i) y[i] = sigmoid(x[i]);
}

/* Round a double to the nearest bfloat16 value (round to nearest, ties to even),
 * returned as a double.  Used only where the cited RMSNorm casts back to the
 * activation dtype. */
static double round_to_bf16(double x)
{
    float f = (float)x;
    uint32_t u;
    memcpy(&u, &f, 4);
    if ((u & 0x7f800000u) == 0x7f800000u) return (double)f; /* inf / nan */
    const uint32_t lsb = (u >> 16) & 1u;
    u += 0x7fffu + lsb;
    u &= 0xffff0000u;
    memcpy(&f, &u, 4);
    return (double)f;
}

/* Layer epilogue, per (token, head) row of length dv:
 *   y   = o * rsqrt(mean(o^2) + eps)           (KimiRMSNorm, computed in high precision)
 *   y   = cast(y, io dtype)                     (cast back to the activation dtype)
 *   y   = gain * y                              (o_norm.weight, [dv], shared by heads)
 *   out = y * sigmoid(z)                        (sigmoid output gate on g_proj(x) = z)
 * gain may be NULL (ones).  io_bf16 != 0 applies the bf16 cast.
 * (atlas.klimoza.dev "KDA layers > MoE input", KimiRMSNorm excerpt;
 *  maxtext PR #5543 What, item 1: out = attn * sigmoid(g_proj(x)).) */
void kda_oracle_out_norm_gate(const double *o, const double *z, const double *gain,
                              double eps, int io_bf16, double *out, size_t rows, int dv)
{
    for (size_t r = 0; r < rows; ++r) {
        const double *orow = o + r * dv;
        double ms = 0.0;
        for (int j = 0; j < dv; ++j) ms += orow[j] * orow[j];
        ms /= (double)dv;
        const double inv = 1.0 / sqrt(ms + eps);
        for (int j = 0; j < dv; ++j) {
            double y = orow[j] * inv;
            if (io_bf16) y = round_to_bf16(y);
            if (gain) y *= gain[j];
            out[r * dv + j] = y * sigmoid(z[r * dv + j]);
        }
    }
}

/* The KDA layer core:
 *   q = l2norm(SiLU(conv_q * q_raw)),  k = l2norm(SiLU(conv_k * k_raw)),
 *   v = SiLU(conv_v * v_raw),
 *   g = max(-exp(A_log) softplus(g_raw + dt_bias), lb),  beta = sigmoid(b_raw),
 *   o = gated delta rule(q, k, v, g, beta; S0) -> (o, S_T),
 *   out = out_norm_gate(o, o_gate_raw).
 * q_raw, k_raw: [B, T, H*dk]; v_raw: [B, T, H*dv]; g_raw: [B, T, H, dk];
 * b_raw: [B, T, H]; o_gate_raw: [B, T, H, dv]; conv_*: [H*d, 4]; A_log: [H];
 * dt_bias: [H*dk] or NULL; lb: the gate's lower bound (-INFINITY: none);
 * o_norm_w: [dv] or NULL; s0, sT: [B, H, dk, dv] or NULL. */
void kda_oracle_layer(const double *q_raw, const double *k_raw, const double *v_raw,
                      const double *conv_q, const double *conv_k, const double *conv_v,
                      const double *g_raw, const double *A_log, const double *dt_bias,
                      double lb, const double *b_raw, const double *o_gate_raw,
                      const double *o_norm_w, double norm_eps, double l2_eps, int io_bf16, const double *s0,
                      double *out, double *sT, int B, int T, int H, int dk, int dv,
                      int nthreads)
{
    const size_t nk = (size_t)B * T * H * dk, nv = (size_t)B * T * H * dv;
    const size_t nb = (size_t)B * T * H;
    double *qc = (double *)malloc(sizeof(double) * nk);
    double *kc = (double *)malloc(sizeof(double) * nk);
    double *vc = (double *)malloc(sizeof(double) * nv);
    double *g = (double *)malloc(sizeof(double) * nk);
    double *beta = (double *)malloc(sizeof(double) * nb);
    double *o = (double *)malloc(sizeof(double) * nv);

    kda_oracle_short_conv_silu(q_raw, conv_q, qc, B, T, H * dk, 1, nthreads);
    kda_oracle_short_conv_silu(k_raw, conv_k, kc, B, T, H * dk, 1, nthreads);
    kda_oracle_short_conv_silu(v_raw, conv_v, vc, B, T, H * dv, 1, nthreads);
    kda_oracle_l2norm(qc, qc, nb, dk, l2_eps);
    kda_oracle_l2norm(kc, kc, nb, dk, l2_eps);
    kda_oracle_gate(g_raw, A_log, dt_bias, lb, g, B, T, H, dk);
    kda_oracle_sigmoid(b_raw, beta, nb);
    kda_oracle_recurrent(qc, kc, vc, g, beta, s0, o, sT, B, T, H, dk, dv, 1, nthreads);
    kda_oracle_out_norm_gate(o, o_gate_raw, o_norm_w, norm_eps, io_bf16, out, nb, dv);

    free(qc);
    free(kc);
    free(vc);
    free(g);
    free(beta);
    free(o);
}
