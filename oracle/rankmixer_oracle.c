/*
 * RankMixer stack forward -- CPU oracle, fp64, plain loops.
 *
 * TEST INFRASTRUCTURE.  Only the test suite, the package smoke check and the
 * benchmark's CPU-baseline leg may load this library.  It shares no code,
 * header, table or helper with the CUDA library, and it never calls into it.
 *
 * What it computes (sources are the pages on RankMixer; the primary one is the
 * fun-rec chapter "Rankmixer: 硬件效率优化"):
 *
 *   block:  S   = LN(TokenMixing(X) + X)                 (section RankMixer整体架构)
 *           X'  = LN(PFFN(S) + S)
 *   mixing: x_t = [x_t^(1) || ... || x_t^(H)]  (SplitHead, chunks of D/H)
 *           s^(h) = Concat(x_1^(h), ..., x_T^(h)),  H = T   (section Token Mixing机制)
 *   PFFN:   v_t = W2_t GELU(W1_t s_t + b1_t) + b2_t        (section Per-Token FFN)
 *   MoE:    G_{t,j} = ReLU(h_t(s_t)),  v_t = sum_j G_{t,j} e_{t,j}(s_t)
 *           with h_t a linear router; experts with G = 0 contribute nothing
 *           (section Sparse MoE扩展, ReLU Routing equation)
 *   pool:   mean over the T tokens of the last block's output
 *           ("特征交叉 —— RankMixer 精读笔记", last paragraph of 模型结构)
 *   Pad-Split: concatenate feature-group embeddings, zero-pad, split into T
 *           equal tokens with no projection ("淘宝闪购-爆品团精排 Scaling Up
 *           迭代实践", section 3.4 Tokenization)
 *
 * Readings where the pages leave a step open:
 *   - LayerNorm normalises each token row over D with the population variance,
 *     eps inside the square root, one (gamma, beta) pair of length D per LN
 *     instance shared by all tokens.
 *   - GELU is the tanh form 0.5 u (1 + tanh(sqrt(2/pi) (u + 0.044715 u^3)))
 *     of Hendrycks & Gimpel (mode 0); mode 1 is the exact erf form; mode 2
 *     is ReLU, the activation of the Mixer backbone timed in Appendix B of
 *     "重新理解 RankMixer：扩参为什么有效，又为什么划算？".
 *   - Variant without the Add & Norm after token mixing (mix_addnorm = 0):
 *     S = TokenMixing(X), the configuration "淘宝闪购-爆品团精排 Scaling Up
 *     迭代实践" reports in section 3.5 (RankMixer 层数).
 *   - Weights are stored out-major, W1_t [kD][D], W2_t [D][kD], router
 *     Wr_t [Ne][D], so u = W1_t s_t is a row-by-vector product as written in
 *     the PFFN equation.
 *   - An expert is active iff its router logit is > 0; its gate multiplies the
 *     whole expert output, second bias included.
 *
 * Numerics: every intermediate is double.  Weights arrive as float (fp32, or
 * bf16 values widened exactly); activations arrive as double or float.  No
 * blocking, fusion or reordering beyond the loops the definitions imply; the
 * only parallelism is OpenMP over independent samples.
 */
#include <math.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

typedef struct {
    const float *W1, *b1, *W2, *b2;        /* dense: [T][kD][D] [T][kD] [T][D][kD] [T][D]    */
                                           /* MoE: [T][Ne][kD][D] [T][Ne][kD] [T][Ne][D][kD] [T][Ne][D] */
    const float *ln1_g, *ln1_b, *ln2_g, *ln2_b;   /* [D] each */
    const float *Wr, *br;                  /* MoE router: [T][Ne][D], [T][Ne] */
} orc_block_params;

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

/* ---- single-sample building blocks ------------------------------------ */

/* Token mixing of one sample.  x: [T][D]; y: [T][D]; H = T heads of width
 * dh = D / T.  Output token h is the concatenation, over t = 0..T-1 in order,
 * of chunk h of input token t. */
static void mix_sample(int T, int D, const double *x, double *y) {
    int dh = D / T;
    for (int h = 0; h < T; ++h)
        for (int t = 0; t < T; ++t)
            for (int j = 0; j < dh; ++j)
                y[(size_t)h * D + (size_t)t * dh + j] = x[(size_t)t * D + (size_t)h * dh + j];
}

/* LayerNorm of one row of length D. */
static void ln_row(int D, const double *z, const float *g, const float *b, double eps, double *out) {
    double mean = 0.0;
    for (int i = 0; i < D; ++i) mean += z[i];
    mean /= D;
    double var = 0.0;
    for (int i = 0; i < D; ++i) var += (z[i] - mean) * (z[i] - mean);
    var /= D;
    double inv = 1.0 / sqrt(var + eps);
    for (int i = 0; i < D; ++i) out[i] = (double)g[i] * ((z[i] - mean) * inv) + (double)b[i];
}

double orc_gelu(double u, int mode) {
    if (mode == 2) return u > 0.0 ? u : 0.0;
    if (mode == 1) return 0.5 * u * (1.0 + erf(u / sqrt(2.0)));
    const double c = sqrt(2.0 / M_PI);
    return 0.5 * u * (1.0 + tanh(c * (u + 0.044715 * u * u * u)));
}

/* One FFN on one token: v = W2 GELU(W1 s + b1) + b2.
 * W1 [Hd][D], b1 [Hd], W2 [D][Hd], b2 [D]; hbuf has Hd doubles. */
static void ffn_vec(int D, int Hd, const double *s, const float *W1, const float *b1,
                    const float *W2, const float *b2, int gelu, double *v, double *hbuf) {
    for (int n = 0; n < Hd; ++n) {
        double u = (double)b1[n];
        const float *w = W1 + (size_t)n * D;
        for (int k = 0; k < D; ++k) u += (double)w[k] * s[k];
        hbuf[n] = orc_gelu(u, gelu);
    }
    for (int d = 0; d < D; ++d) {
        double acc = (double)b2[d];
        const float *w = W2 + (size_t)d * Hd;
        for (int n = 0; n < Hd; ++n) acc += (double)w[n] * hbuf[n];
        v[d] = acc;
    }
}

/* Router logits of one token: r_j = Wr_t[j] . s + br_t[j]. */
static void router_vec(int D, int Ne, const double *s, const float *Wr, const float *br, double *r) {
    for (int j = 0; j < Ne; ++j) {
        double acc = (double)br[j];
        const float *w = Wr + (size_t)j * D;
        for (int k = 0; k < D; ++k) acc += (double)w[k] * s[k];
        r[j] = acc;
    }
}

/* Sparse-MoE FFN of token t of one sample.  Experts with gate 0 are skipped;
 * gate > 0 experts are summed in ascending j. */
static void moe_vec(int t, int D, int Hd, int Ne, const double *s, const orc_block_params *p,
                    int gelu, double *v, double *logits, double *ebuf, double *hbuf) {
    router_vec(D, Ne, s, p->Wr + (size_t)t * Ne * D, p->br + (size_t)t * Ne, logits);
    for (int d = 0; d < D; ++d) v[d] = 0.0;
    for (int j = 0; j < Ne; ++j) {
        double gate = logits[j] > 0.0 ? logits[j] : 0.0;   /* ReLU */
        if (gate == 0.0) continue;                           /* zero gate: expert skipped */
        size_t e = (size_t)t * Ne + j;
        ffn_vec(D, Hd, s, p->W1 + e * Hd * D, p->b1 + e * Hd, p->W2 + e * D * Hd, p->b2 + e * D,
                gelu, ebuf, hbuf);
        for (int d = 0; d < D; ++d) v[d] += gate * ebuf[d];
    }
}

/* One RankMixer block on one sample: x, y are [T][D]. */
static void block_sample(int T, int D, int Hd, int Ne, const double *x, const orc_block_params *p,
                         double eps, int gelu, int mix_addnorm, double *y, double *logits_out, double *work) {
    double *z = work;                       /* [T][D] */
    double *s = z + (size_t)T * D;          /* [T][D] */
    double *v = s + (size_t)T * D;          /* [D]    */
    double *e = v + D;                      /* [D]    */
    double *hb = e + D;                     /* [Hd]   */
    double lg[64];
    /* S = LN(TokenMixing(X) + X), or S = TokenMixing(X) without the Add & Norm */
    mix_sample(T, D, x, z);
    if (mix_addnorm) {
        for (size_t i = 0; i < (size_t)T * D; ++i) z[i] += x[i];
        for (int t = 0; t < T; ++t) ln_row(D, z + (size_t)t * D, p->ln1_g, p->ln1_b, eps, s + (size_t)t * D);
    } else {
        for (size_t i = 0; i < (size_t)T * D; ++i) s[i] = z[i];
    }
    /* X' = LN(PFFN(S) + S) */
    for (int t = 0; t < T; ++t) {
        const double *st = s + (size_t)t * D;
        if (Ne == 0) {
            ffn_vec(D, Hd, st, p->W1 + (size_t)t * Hd * D, p->b1 + (size_t)t * Hd,
                    p->W2 + (size_t)t * D * Hd, p->b2 + (size_t)t * D, gelu, v, hb);
        } else {
            moe_vec(t, D, Hd, Ne, st, p, gelu, v, lg, e, hb);
            if (logits_out)
                for (int j = 0; j < Ne; ++j) logits_out[(size_t)t * Ne + j] = lg[j];
        }
        for (int d = 0; d < D; ++d) v[d] += st[d];
        ln_row(D, v, p->ln2_g, p->ln2_b, eps, y + (size_t)t * D);
    }
}

static size_t block_work_doubles(int T, int D, int Hd) {
    return (size_t)2 * T * D + 2 * (size_t)D + (size_t)Hd;
}

/* ---- exported per-step functions (loops over samples / rows) ---------- */

void orc_token_mix(long B, int T, int D, const double *X, double *Y) {
    #pragma omp parallel for schedule(static)
    for (long b = 0; b < B; ++b)
        mix_sample(T, D, X + (size_t)b * T * D, Y + (size_t)b * T * D);
}

void orc_layernorm(long rows, int D, const double *Z, const float *g, const float *b,
                   double eps, double *out) {
    #pragma omp parallel for schedule(static)
    for (long r = 0; r < rows; ++r) ln_row(D, Z + (size_t)r * D, g, b, eps, out + (size_t)r * D);
}

void orc_gelu_array(long n, const double *u, int mode, double *out) {
    for (long i = 0; i < n; ++i) out[i] = orc_gelu(u[i], mode);
}

/* V[b][t] = PFFN_t(S[b][t]) (no residual, no LN). */
void orc_pffn(long B, int T, int D, int Hd, const double *S, const float *W1, const float *b1,
              const float *W2, const float *b2, int gelu, double *V) {
    #pragma omp parallel
    {
        double *hb = (double *)malloc(sizeof(double) * (size_t)Hd);
        #pragma omp for schedule(dynamic)
        for (long b = 0; b < B; ++b)
            for (int t = 0; t < T; ++t) {
                size_t row = ((size_t)b * T + t) * D;
                ffn_vec(D, Hd, S + row, W1 + (size_t)t * Hd * D, b1 + (size_t)t * Hd,
                        W2 + (size_t)t * D * Hd, b2 + (size_t)t * D, gelu, V + row, hb);
            }
        free(hb);
    }
}

/* V[b][t] = sum_j ReLU(r_j) e_{t,j}(S[b][t]); logits [B][T][Ne] (may be NULL). */
void orc_moe(long B, int T, int D, int Hd, int Ne, const double *S, const orc_block_params *p,
             int gelu, double *V, double *logits) {
    #pragma omp parallel
    {
        double *hb = (double *)malloc(sizeof(double) * (size_t)Hd);
        double *eb = (double *)malloc(sizeof(double) * (size_t)D);
        double lg[64];
        #pragma omp for schedule(dynamic)
        for (long b = 0; b < B; ++b)
            for (int t = 0; t < T; ++t) {
                size_t row = ((size_t)b * T + t) * D;
                moe_vec(t, D, Hd, Ne, S + row, p, gelu, V + row, lg, eb, hb);
                if (logits)
                    for (int j = 0; j < Ne; ++j) logits[((size_t)b * T + t) * Ne + j] = lg[j];
            }
        free(hb);
        free(eb);
    }
}

/* Router logits alone: logits[b][t][j] = Wr_t[j] . S[b][t] + br_t[j]
 * (the linear router h_t of the ReLU routing equation, before the ReLU). */
void orc_router(long B, int T, int D, int Ne, const double *S, const float *Wr, const float *br,
                double *logits) {
    #pragma omp parallel for schedule(static)
    for (long b = 0; b < B; ++b)
        for (int t = 0; t < T; ++t)
            router_vec(D, Ne, S + ((size_t)b * T + t) * D, Wr + (size_t)t * Ne * D, br + (size_t)t * Ne,
                       logits + ((size_t)b * T + t) * Ne);
}

/* One block over B samples. logits [B][T][Ne] (MoE only, may be NULL). */
void orc_block(long B, int T, int D, int Hd, int Ne, const double *X, const orc_block_params *p,
               double eps, int gelu, int mix_addnorm, double *Y, double *logits) {
    #pragma omp parallel
    {
        double *work = (double *)malloc(sizeof(double) * block_work_doubles(T, D, Hd));
        #pragma omp for schedule(dynamic)
        for (long b = 0; b < B; ++b)
            block_sample(T, D, Hd, Ne, X + (size_t)b * T * D, p, eps, gelu, mix_addnorm, Y + (size_t)b * T * D,
                         logits ? logits + (size_t)b * T * Ne : NULL, work);
        free(work);
    }
}

/* L blocks then mean pooling.  X0 [B][T][D] (float).  pooled [B][D].
 * Xall (may be NULL): [L][B][T][D], every block's output.
 * Xlast (may be NULL): [B][T][D], the last block's output. */
void orc_stack(long B, int T, int D, int Hd, int Ne, int L, const float *X0,
               const orc_block_params *blocks, double eps, int gelu, int mix_addnorm,
               double *pooled, double *Xlast, double *Xall) {
    #pragma omp parallel
    {
        size_t td = (size_t)T * D;
        double *work = (double *)malloc(sizeof(double) * block_work_doubles(T, D, Hd));
        double *xa = (double *)malloc(sizeof(double) * td);
        double *xb = (double *)malloc(sizeof(double) * td);
        #pragma omp for schedule(dynamic)
        for (long b = 0; b < B; ++b) {
            for (size_t i = 0; i < td; ++i) xa[i] = (double)X0[(size_t)b * td + i];
            for (int l = 0; l < L; ++l) {
                block_sample(T, D, Hd, Ne, xa, &blocks[l], eps, gelu, mix_addnorm, xb, NULL, work);
                if (Xall) memcpy(Xall + ((size_t)l * B + b) * td, xb, sizeof(double) * td);
                double *tmp = xa; xa = xb; xb = tmp;
            }
            if (Xlast) memcpy(Xlast + (size_t)b * td, xa, sizeof(double) * td);
            for (int d = 0; d < D; ++d) {
                double acc = 0.0;
                for (int t = 0; t < T; ++t) acc += xa[(size_t)t * D + d];
                pooled[(size_t)b * D + d] = acc / T;
            }
        }
        free(work);
        free(xa);
        free(xb);
    }
}

/* Pad-Split: X0[b] = [g_0[b] ; g_1[b] ; ... ; 0 ... 0] of length padded. */
void orc_padsplit(long B, int n_groups, const int *widths, const float *const *groups, int padded,
                  double *X0) {
    for (long b = 0; b < B; ++b) {
        double *row = X0 + (size_t)b * padded;
        int c = 0;
        for (int i = 0; i < n_groups; ++i)
            for (int k = 0; k < widths[i]; ++k) row[c++] = (double)groups[i][(size_t)b * widths[i] + k];
        for (; c < padded; ++c) row[c] = 0.0;
    }
}

/* prob[b] = sigmoid(pooled[b] . w + bias). */
void orc_head(long B, int D, const double *pooled, const float *w, double bias, double *prob) {
    for (long b = 0; b < B; ++b) {
        double acc = bias;
        for (int d = 0; d < D; ++d) acc += pooled[(size_t)b * D + d] * (double)w[d];
        prob[b] = 1.0 / (1.0 + exp(-acc));
    }
}
