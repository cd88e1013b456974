/*
 * Plain fp64 CPU oracle for the hybrid-attention decode path (KDA gated delta rule,
 * its width-4 short convolution, and gated latent attention over the 576-wide MLA cache).
 *
 * TEST INFRASTRUCTURE ONLY. Nothing in the product library links or calls this file; only
 * the test suite, the smoke check and the benchmark's CPU-baseline leg load it. It shares no
 * code, header, table or constant with the CUDA kernels.
 *
 * Sources (web pages on Ling-3.1-flash):
 *   [P1] "Ling-3.1-flash and the 7:1 hybrid: how much KV cache does a 560B model need at 1M
 *        tokens?" (dev.to), sections "How big is the cache per token, exactly?" and
 *        "Why would a model keep only 9 full-attention layers?"
 *   [P2] "Ling-3.1-flash: a 560B hybrid-attention MoE, counted from its safetensors headers"
 *        (ai.thesatyajit.com), sections "How KDA and MLA split the work" and
 *        "Does 292 GiB fit on four Hopper GPUs?"
 *
 * The display equation of the KDA update was lost from [P2] "How KDA and MLA split the work".
 * What survives there: a gated delta-rule linear attention; per token the 128x128 state is
 * decayed channel by channel (alpha_t, one decay per key channel) and the new key-value
 * association is written with a per-head scalar strength beta_t; q, k, v come through a
 * short causal convolution of width 4. [P1] "Why would a model keep only 9..." names the
 * lineage: Gated DeltaNet with finer-grained (per-channel) gating. The readings taken where
 * the page is silent are stated at each function and are:
 *   (i)   the decay is applied before the delta correction (the correction predicts from the
 *         decayed state), Gated-DeltaNet order;
 *   (ii)  alpha scales the key (row) index of S, with S of shape d_k x d_v;
 *   (iii) the readout is o_t = scale * S_t^T q_t, read after the write, scale a parameter;
 *   (iv)  the convolution output passes through SiLU when the caller asks for it.
 *
 * Arithmetic is double precision throughout. Loops follow the definitions directly; the only
 * parallelism is over independent (sequence, head) pairs, which changes no result.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define LADO_OK 0
#define LADO_EINVAL -1
#define LADO_ENOMEM -2

int lado_num_threads_available(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* A bf16 value is the upper 16 bits of an IEEE binary32; widening it is exact. */
static double bf16_bits_to_double(uint16_t bits) {
    uint32_t u = ((uint32_t)bits) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/*
 * KDA gated delta rule, token by token ([P2] "How KDA and MLA split the work"; [P1] "Why
 * would a model keep only 9 full-attention layers?" for the Gated DeltaNet lineage).
 * For every sequence b, head h and token t, with S the d_k x d_v state of (b, h):
 *   S'  = Diag(alpha_t) S_{t-1}            decay, channel by channel (rows = key channels)
 *   w   = S'^T k_t                         what the decayed state predicts for key k_t
 *   u   = beta_t (v_t - w)                 delta-rule correction, strength beta_t
 *   S_t = S' + k_t u^T                     write the new key-value association
 *   o_t = scale * S_t^T q_t                readout after the write
 * Layouts (row-major): q, k, alpha [B][T][H][dk]; v, o [B][T][H][dv]; beta [B][T][H];
 * S [B][H][dk][dv], initial state in, final state out.
 */
int lado_kda_recurrent(int B, int T, int H, int dk, int dv, double scale,
                       const double *q, const double *k, const double *v,
                       const double *alpha, const double *beta,
                       double *S, double *o, int nthreads) {
    if (B < 0 || T < 0 || H < 0 || dk <= 0 || dv <= 0) return LADO_EINVAL;
    if (nthreads < 1) nthreads = 1;
    int err = 0;
#pragma omp parallel for num_threads(nthreads) collapse(2) schedule(dynamic)
    for (int b = 0; b < B; ++b) {
        for (int h = 0; h < H; ++h) {
            double *Sbh = S + ((size_t)b * H + h) * (size_t)dk * dv;
            double *w = (double *)malloc(sizeof(double) * dv);
            double *u = (double *)malloc(sizeof(double) * dv);
            if (!w || !u) {
                free(w); free(u);
#pragma omp atomic write
                err = 1;
                continue;
            }
            for (int t = 0; t < T; ++t) {
                size_t tok = ((size_t)b * T + t) * H + h;
                const double *qt = q + tok * dk;
                const double *kt = k + tok * dk;
                const double *at = alpha + tok * dk;
                const double *vt = v + tok * dv;
                double bt = beta[tok];
                double *ot = o + tok * dv;
                /* S' = Diag(alpha_t) S_{t-1} */
                for (int i = 0; i < dk; ++i)
                    for (int j = 0; j < dv; ++j)
                        Sbh[(size_t)i * dv + j] *= at[i];
                /* w = S'^T k_t */
                for (int j = 0; j < dv; ++j) {
                    double acc = 0.0;
                    for (int i = 0; i < dk; ++i) acc += Sbh[(size_t)i * dv + j] * kt[i];
                    w[j] = acc;
                }
                /* u = beta_t (v_t - w) */
                for (int j = 0; j < dv; ++j) u[j] = bt * (vt[j] - w[j]);
                /* S_t = S' + k_t u^T */
                for (int i = 0; i < dk; ++i)
                    for (int j = 0; j < dv; ++j)
                        Sbh[(size_t)i * dv + j] += kt[i] * u[j];
                /* o_t = scale * S_t^T q_t */
                for (int j = 0; j < dv; ++j) {
                    double acc = 0.0;
                    for (int i = 0; i < dk; ++i) acc += Sbh[(size_t)i * dv + j] * qt[i];
                    ot[j] = scale * acc;
                }
            }
            free(w);
            free(u);
        }
    }
    return err ? LADO_ENOMEM : LADO_OK;
}

/*
 * The same recurrence in chunked (WY / UT) form, chunk length C, a last partial chunk allowed.
 * The pages do not print it; it follows from lado_kda_recurrent by unrolling the recurrence
 * inside a chunk. Within a chunk with rows r = 0..n-1 and initial state S0:
 *   g_r   = prod_{s<=r} alpha_s                 cumulative decay per key channel
 *   Kt    = K * g,  Kh = K / g,  Qt = Q * g     (elementwise, row r uses g_r)
 *   A     = strict_lower(diag(beta) Kt Kh^T)
 *   Tm    = (I + A)^{-1}                        by forward substitution (unit lower triangular)
 *   W     = Tm diag(beta) Kt
 *   U     = Tm diag(beta) V - W S0
 *   O     = scale (Qt S0 + lower(Qt Kh^T) U)    lower() keeps the diagonal
 *   S_new = Diag(g_{n-1}) S0 + (K * (g_{n-1} / g))^T U
 * Same layouts as lado_kda_recurrent.
 */
int lado_kda_chunked(int B, int T, int H, int dk, int dv, int C, double scale,
                     const double *q, const double *k, const double *v,
                     const double *alpha, const double *beta,
                     double *S, double *o, int nthreads) {
    if (B < 0 || T < 0 || H < 0 || dk <= 0 || dv <= 0 || C <= 0) return LADO_EINVAL;
    if (nthreads < 1) nthreads = 1;
    int err = 0;
#pragma omp parallel for num_threads(nthreads) collapse(2) schedule(dynamic)
    for (int b = 0; b < B; ++b) {
        for (int h = 0; h < H; ++h) {
            double *S0 = S + ((size_t)b * H + h) * (size_t)dk * dv;
            size_t nk = (size_t)C * dk, nv = (size_t)C * dv, cc = (size_t)C * C;
            double *g = malloc(sizeof(double) * nk), *Kt = malloc(sizeof(double) * nk);
            double *Kh = malloc(sizeof(double) * nk), *Qt = malloc(sizeof(double) * nk);
            double *A = malloc(sizeof(double) * cc), *Tm = malloc(sizeof(double) * cc);
            double *QK = malloc(sizeof(double) * cc), *W = malloc(sizeof(double) * nk);
            double *U = malloc(sizeof(double) * nv);
            double *Snew = malloc(sizeof(double) * (size_t)dk * dv);
            if (!g || !Kt || !Kh || !Qt || !A || !Tm || !QK || !W || !U || !Snew) {
#pragma omp atomic write
                err = 1;
                goto done;
            }
            for (int c0 = 0; c0 < T; c0 += C) {
                int n = (T - c0) < C ? (T - c0) : C;
#define TOK(r) (((size_t)b * T + (size_t)(c0 + (r))) * H + h)
                /* cumulative decay g and the scaled keys / queries */
                for (int r = 0; r < n; ++r) {
                    const double *ar = alpha + TOK(r) * dk;
                    const double *kr = k + TOK(r) * dk;
                    const double *qr = q + TOK(r) * dk;
                    for (int i = 0; i < dk; ++i) {
                        double prev = (r == 0) ? 1.0 : g[(size_t)(r - 1) * dk + i];
                        double gi = prev * ar[i];
                        g[(size_t)r * dk + i] = gi;
                        Kt[(size_t)r * dk + i] = kr[i] * gi;
                        Kh[(size_t)r * dk + i] = kr[i] / gi;
                        Qt[(size_t)r * dk + i] = qr[i] * gi;
                    }
                }
                /* A = strict_lower(diag(beta) Kt Kh^T); QK = lower(Qt Kh^T) */
                for (int r = 0; r < n; ++r) {
                    double br = beta[TOK(r)];
                    for (int s = 0; s < n; ++s) {
                        double kk = 0.0, qk = 0.0;
                        for (int i = 0; i < dk; ++i) {
                            kk += Kt[(size_t)r * dk + i] * Kh[(size_t)s * dk + i];
                            qk += Qt[(size_t)r * dk + i] * Kh[(size_t)s * dk + i];
                        }
                        A[(size_t)r * C + s] = (s < r) ? br * kk : 0.0;
                        QK[(size_t)r * C + s] = (s <= r) ? qk : 0.0;
                    }
                }
                /* Tm = (I + A)^{-1}: solve (I + A) Tm = I row by row */
                for (int r = 0; r < n; ++r) {
                    for (int col = 0; col < n; ++col) {
                        double acc = (r == col) ? 1.0 : 0.0;
                        for (int s = 0; s < r; ++s) acc -= A[(size_t)r * C + s] * Tm[(size_t)s * C + col];
                        Tm[(size_t)r * C + col] = acc;
                    }
                }
                /* W = Tm diag(beta) Kt */
                for (int r = 0; r < n; ++r)
                    for (int i = 0; i < dk; ++i) {
                        double acc = 0.0;
                        for (int s = 0; s < n; ++s)
                            acc += Tm[(size_t)r * C + s] * beta[TOK(s)] * Kt[(size_t)s * dk + i];
                        W[(size_t)r * dk + i] = acc;
                    }
                /* U = Tm diag(beta) V - W S0 */
                for (int r = 0; r < n; ++r)
                    for (int j = 0; j < dv; ++j) {
                        double acc = 0.0;
                        for (int s = 0; s < n; ++s)
                            acc += Tm[(size_t)r * C + s] * beta[TOK(s)] * v[TOK(s) * dv + j];
                        for (int i = 0; i < dk; ++i) acc -= W[(size_t)r * dk + i] * S0[(size_t)i * dv + j];
                        U[(size_t)r * dv + j] = acc;
                    }
                /* O = scale (Qt S0 + lower(Qt Kh^T) U) */
                for (int r = 0; r < n; ++r)
                    for (int j = 0; j < dv; ++j) {
                        double acc = 0.0;
                        for (int i = 0; i < dk; ++i) acc += Qt[(size_t)r * dk + i] * S0[(size_t)i * dv + j];
                        for (int s = 0; s <= r; ++s) acc += QK[(size_t)r * C + s] * U[(size_t)s * dv + j];
                        o[TOK(r) * dv + j] = scale * acc;
                    }
                /* S_new = Diag(g_last) S0 + (K * (g_last / g))^T U */
                const double *gl = g + (size_t)(n - 1) * dk;
                for (int i = 0; i < dk; ++i)
                    for (int j = 0; j < dv; ++j) {
                        double acc = gl[i] * S0[(size_t)i * dv + j];
                        for (int s = 0; s < n; ++s)
                            acc += k[TOK(s) * dk + i] * (gl[i] / g[(size_t)s * dk + i]) * U[(size_t)s * dv + j];
                        Snew[(size_t)i * dv + j] = acc;
                    }
                memcpy(S0, Snew, sizeof(double) * (size_t)dk * dv);
#undef TOK
            }
        done:
            free(g); free(Kt); free(Kh); free(Qt); free(A); free(Tm);
            free(QK); free(W); free(U); free(Snew);
        }
    }
    return err ? LADO_ENOMEM : LADO_OK;
}

/*
 * Per-vector L2 normalisation y = x / sqrt(sum x^2 + eps), applied to q and k per head before
 * the recurrence. The pages do not mention it; it is the usual input conditioning of delta-rule
 * layers and is kept behind a flag. x and y are [n][d].
 */
int lado_l2norm(long long n, int d, double eps, const double *x, double *y) {
    if (n < 0 || d <= 0) return LADO_EINVAL;
    for (long long r = 0; r < n; ++r) {
        double ss = 0.0;
        for (int i = 0; i < d; ++i) ss += x[r * d + i] * x[r * d + i];
        double inv = 1.0 / sqrt(ss + eps);
        for (int i = 0; i < d; ++i) y[r * d + i] = x[r * d + i] * inv;
    }
    return LADO_OK;
}

/*
 * One decode step of the short causal depthwise convolution that q, k, v pass through
 * ([P2] "How KDA and MLA split the work": width 4; [P2] "Does 292 GiB fit...": the kept
 * "convolution tails"). For every sequence b and channel c, with K taps:
 *   y[b][c] = sum_{i<K-1} w[c][i] tail[b][i][c] + w[c][K-1] x[b][c]  (+ bias[c] if given)
 *   y       = y * sigmoid(y)                      when silu != 0
 * tail[b][0] is the oldest kept input, tail[b][K-2] the newest. Afterwards the tail drops its
 * oldest row and appends x: tail[b][i] = tail[b][i+1] for i < K-2, tail[b][K-2] = x[b].
 * Layouts: x, y [B][Cch]; tail [B][K-1][Cch] (in/out); w [Cch][K]; bias [Cch] or NULL.
 */
int lado_short_conv_step(int B, int Cch, int K, const double *x, double *tail,
                         const double *w, const double *bias, int silu, double *y) {
    if (B < 0 || Cch <= 0 || K < 1) return LADO_EINVAL;
    for (int b = 0; b < B; ++b) {
        double *tb = tail + (size_t)b * (size_t)(K - 1) * Cch;
        for (int c = 0; c < Cch; ++c) {
            double acc = 0.0;
            for (int i = 0; i < K - 1; ++i) acc += w[(size_t)c * K + i] * tb[(size_t)i * Cch + c];
            acc += w[(size_t)c * K + (K - 1)] * x[(size_t)b * Cch + c];
            if (bias) acc += bias[c];
            if (silu) acc = acc / (1.0 + exp(-acc));
            y[(size_t)b * Cch + c] = acc;
        }
        for (int i = 0; i + 1 < K - 1; ++i)
            memcpy(tb + (size_t)i * Cch, tb + (size_t)(i + 1) * Cch, sizeof(double) * Cch);
        if (K > 1) memcpy(tb + (size_t)(K - 2) * Cch, x + (size_t)b * Cch, sizeof(double) * Cch);
    }
    return LADO_OK;
}

/*
 * Gated MLA decode over the compressed latent cache ([P2] "How KDA and MLA split the work":
 * ordinary softmax attention over a cache whose rows are a 512-wide latent plus a 64-wide RoPE
 * key, scaled by a per-head sigmoid gate; [P1] "How big is the cache per token, exactly?": the
 * cached row is kv_lora_rank + qk_rope_head_dim = 576 elements; [P1] "For scale, plain
 * multi-head attention..." gives the 192-wide key behind the softmax scale).
 * The query arrives already absorbed (W_UK folded in), so it is Dc + Dr wide. For every
 * sequence b with L = seq_lens[b] cached rows c_0..c_{L-1} and every head h:
 *   s_t  = scale * <q_h, c_t>                 over all Dc + Dr dimensions
 *   p_t  = exp(s_t - max s) / sum_t exp(s_t - max s)
 *   o_h  = sum_t p_t c_t[0:Dc]                the values are the latent part only
 *   o_h *= sigmoid(gate[b][h])                when gate is given
 *   lse  = max s + log sum_t exp(s_t - max s) (natural log, before the gate)
 * L = 0 gives o_h = 0 and lse = -inf.
 * Layouts: q [B][H][Dc+Dr] (double); cache: bf16 bit patterns, row t of sequence b at
 * element offset b*seq_stride + t*(Dc+Dr); gate [B][H] or NULL; o [B][H][Dc]; lse [B][H] or NULL.
 */
/* Row t of one sequence's cache: contiguous rows (bt == NULL), or the paged layout in which
 * rows [j*P, (j+1)*P) of the sequence are page bt[j] of the pool, P rows per page. */
static size_t mla_row(const int *bt, int P, int D, int t) {
    if (!bt) return (size_t)t * D;
    return ((size_t)bt[t / P] * (size_t)P + (size_t)(t % P)) * (size_t)D;
}

/*
 * FP8 latent cache ([P1] "How big is the cache per token, exactly?": 2 bytes per element in
 * bf16, an FP8 cache halves that; [P2] "Does 292 GiB fit on four Hopper GPUs?": an FP8 cache
 * doubles the tokens that fit). The FP8 the pages name is E4M3 ([P2] "What is in the files": the
 * release's E4M3 weights carry one fp32 scale per 128x128 block). E4M3: 1 sign bit, 4 exponent
 * bits with bias 7, 3 mantissa bits; exponent field 0 holds the subnormals m/8 * 2^-6; there is
 * no infinity, and exponent and mantissa all ones (0x7F, 0xFF) is NaN, so the largest finite
 * value is 1.75 * 2^8 = 448. The pages give no scale for the cache; the reading here is one fp32
 * scale per cache: an element's value is scale * E4M3(code).
 */
static double e4m3_to_double(uint8_t c) {
    const int sign = c >> 7, e = (c >> 3) & 15, m = c & 7;
    double v;
    if (e == 15 && m == 7)
        v = NAN;
    else if (e == 0)
        v = ldexp((double)m, -9); /* m/8 * 2^-6 */
    else
        v = ldexp(8.0 + m, e - 10); /* (1 + m/8) * 2^(e-7) */
    return sign ? -v : v;
}

/* Nearest E4M3 code of v, ties to the even code, magnitudes beyond 448 clamped to 448 (a
 * saturating conversion), NaN to 0x7F. The candidates in v's binade are multiples of the spacing
 * of 4-bit significands there, 2^(e-4) for |v| = m * 2^e, m in [0.5, 1); below 2^-6 the spacing
 * stays at the subnormal step 2^-9. A multiple k of the spacing maps to its code directly: the
 * code's low 7 bits, read as an integer, count steps of the spacing within the format. */
static uint8_t double_to_e4m3(double v) {
    if (v != v) return 0x7Fu;
    const uint8_t sign = signbit(v) ? 0x80u : 0u;
    const double a = fabs(v);
    if (a >= 448.0) return (uint8_t)(sign | 0x7Eu);
    if (a == 0.0) return sign;
    int e;
    frexp(a, &e);
    int q = e - 4;
    if (q < -9) q = -9;
    const double ulp = ldexp(1.0, q);
    const double klo = floor(a / ulp), khi = klo + 1.0;
    const double dlo = a - klo * ulp, dhi = khi * ulp - a;
    double k;
    if (dlo < dhi)
        k = klo;
    else if (dhi < dlo)
        k = khi;
    else
        k = (fmod(klo, 2.0) == 0.0) ? klo : khi;
    const double r = k * ulp; /* <= 448: 448 is a multiple of its binade's spacing 32 */
    if (r == 0.0) return sign;
    /* r = j * 2^-9 for j < 8 (subnormal codes j), else r = (8 + m) * 2^(E-10) with E >= 1 */
    if (r < ldexp(1.0, -6)) return (uint8_t)(sign | (uint8_t)(r * 512.0));
    int E;
    const double f = frexp(r, &E); /* r = f * 2^E, f in [0.5, 1): exponent field E + 6 */
    const int m = (int)(f * 16.0) - 8;
    return (uint8_t)(sign | (uint8_t)(((E + 6) << 3) | m));
}

int lado_e4m3_decode(int n, const uint8_t *c, double *out) {
    if (n < 0) return LADO_EINVAL;
    for (int i = 0; i < n; ++i) out[i] = e4m3_to_double(c[i]);
    return LADO_OK;
}

int lado_e4m3_encode(int n, const double *x, uint8_t *out) {
    if (n < 0) return LADO_EINVAL;
    for (int i = 0; i < n; ++i) out[i] = double_to_e4m3(x[i]);
    return LADO_OK;
}

/* Element i of the cache: bf16 bits (fp8_value == NULL), or an E4M3 code looked up in
 * fp8_value[code] = kv_scale * E4M3(code) (filled once per call from e4m3_to_double). */
static double cache_elem(const void *cache, const double *fp8_value, size_t i) {
    if (fp8_value) return fp8_value[((const uint8_t *)cache)[i]];
    return bf16_bits_to_double(((const uint16_t *)cache)[i]);
}

/* Shared body of the contiguous and paged entry points. With block_table == NULL, sequence b's
 * rows start at cache + b*seq_stride; otherwise cache is the page pool and row b of the block
 * table (bt_stride entries) names its pages of P rows. */
static int mla_decode_impl(int B, int H, int Dc, int Dr, const double *q, const void *cache, int fp8,
                           double kv_scale, long long seq_stride, const int *block_table, int bt_stride, int P,
                           const int *seq_lens, const double *gate, double scale, double *o, double *lse,
                           int nthreads) {
    if (nthreads < 1) nthreads = 1;
    const int D = Dc + Dr;
    int err = 0;
    double fp8_table[256];
    for (int c = 0; c < 256; ++c) fp8_table[c] = kv_scale * e4m3_to_double((uint8_t)c);
    const double *fp8_value = fp8 ? fp8_table : NULL;
#pragma omp parallel for num_threads(nthreads) collapse(2) schedule(dynamic)
    for (int b = 0; b < B; ++b) {
        for (int h = 0; h < H; ++h) {
            const int L = seq_lens[b];
            const double *qh = q + ((size_t)b * H + h) * D;
            double *oh = o + ((size_t)b * H + h) * Dc;
            if (L <= 0) {
                for (int d = 0; d < Dc; ++d) oh[d] = 0.0;
                if (lse) lse[(size_t)b * H + h] = -INFINITY;
                continue;
            }
            double *s = (double *)malloc(sizeof(double) * (size_t)L);
            if (!s) {
#pragma omp atomic write
                err = 1;
                continue;
            }
            const size_t cb = block_table ? 0 : (size_t)b * (size_t)seq_stride;
            const int *bt = block_table ? block_table + (size_t)b * (size_t)bt_stride : NULL;
            double m = -INFINITY;
            for (int t = 0; t < L; ++t) {
                const size_t ct = cb + mla_row(bt, P, D, t);
                double acc = 0.0;
                for (int d = 0; d < D; ++d) acc += qh[d] * cache_elem(cache, fp8_value, ct + (size_t)d);
                s[t] = scale * acc;
                if (s[t] > m) m = s[t];
            }
            double z = 0.0;
            for (int t = 0; t < L; ++t) {
                s[t] = exp(s[t] - m);
                z += s[t];
            }
            for (int d = 0; d < Dc; ++d) oh[d] = 0.0;
            for (int t = 0; t < L; ++t) {
                const size_t ct = cb + mla_row(bt, P, D, t);
                double p = s[t] / z;
                for (int d = 0; d < Dc; ++d) oh[d] += p * cache_elem(cache, fp8_value, ct + (size_t)d);
            }
            if (gate) {
                double sg = 1.0 / (1.0 + exp(-gate[(size_t)b * H + h]));
                for (int d = 0; d < Dc; ++d) oh[d] *= sg;
            }
            if (lse) lse[(size_t)b * H + h] = m + log(z);
            free(s);
        }
    }
    return err ? LADO_ENOMEM : LADO_OK;
}

int lado_mla_decode(int B, int H, int Dc, int Dr, long long seq_stride,
                    const double *q, const uint16_t *cache, const int *seq_lens,
                    const double *gate, double scale, double *o, double *lse, int nthreads) {
    if (B < 0 || H < 0 || Dc <= 0 || Dr < 0) return LADO_EINVAL;
    return mla_decode_impl(B, H, Dc, Dr, q, cache, 0, 1.0, seq_stride, NULL, 0, 1, seq_lens, gate, scale, o, lse,
                           nthreads);
}

/* The same attention over an FP8 cache: E4M3 codes, row t of sequence b at byte offset
 * b*seq_stride + t*(Dc+Dr), each element worth kv_scale * E4M3(code). */
int lado_mla_decode_fp8(int B, int H, int Dc, int Dr, long long seq_stride, const double *q, const uint8_t *cache,
                        double kv_scale, const int *seq_lens, const double *gate, double scale, double *o,
                        double *lse, int nthreads) {
    if (B < 0 || H < 0 || Dc <= 0 || Dr < 0) return LADO_EINVAL;
    return mla_decode_impl(B, H, Dc, Dr, q, cache, 1, kv_scale, seq_stride, NULL, 0, 1, seq_lens, gate, scale, o,
                           lse, nthreads);
}

/*
 * The same attention over a paged cache, the layout serving engines keep the latent cache in
 * ([P2] "How KDA and MLA split the work" and [P1] "How big is the cache per token, exactly?"
 * give the row; the paging is storage only and changes no arithmetic): the pool holds
 * num_pages pages of P rows (pages [num_pages][P][Dc+Dr], bf16 bit patterns) and row t of
 * sequence b is row t % P of page block_table[b*bt_stride + t / P].
 * Returns LADO_EINVAL if a sequence needs more than bt_stride pages or names a page outside
 * [0, num_pages).
 */
static int check_block_table(int B, int P, int num_pages, int bt_stride, const int *block_table,
                             const int *seq_lens) {
    for (int b = 0; b < B; ++b) {
        const long long L = seq_lens[b];
        if (L < 0 || L > (long long)bt_stride * P) return LADO_EINVAL;
        for (long long j = 0; j * P < L; ++j) {
            const int pg = block_table[(size_t)b * bt_stride + (size_t)j];
            if (pg < 0 || pg >= num_pages) return LADO_EINVAL;
        }
    }
    return LADO_OK;
}

int lado_mla_decode_paged(int B, int H, int Dc, int Dr, int P, int num_pages, int bt_stride,
                          const double *q, const uint16_t *pages, const int *block_table, const int *seq_lens,
                          const double *gate, double scale, double *o, double *lse, int nthreads) {
    if (B < 0 || H < 0 || Dc <= 0 || Dr < 0 || P <= 0 || num_pages < 0 || bt_stride < 0) return LADO_EINVAL;
    const int rc = check_block_table(B, P, num_pages, bt_stride, block_table, seq_lens);
    if (rc != LADO_OK) return rc;
    return mla_decode_impl(B, H, Dc, Dr, q, pages, 0, 1.0, 0, block_table, bt_stride, P, seq_lens, gate, scale, o,
                           lse, nthreads);
}

/* The paged attention over an FP8 page pool (E4M3 codes [num_pages][P][Dc+Dr], scale kv_scale). */
int lado_mla_decode_paged_fp8(int B, int H, int Dc, int Dr, int P, int num_pages, int bt_stride, const double *q,
                              const uint8_t *pages, double kv_scale, const int *block_table, const int *seq_lens,
                              const double *gate, double scale, double *o, double *lse, int nthreads) {
    if (B < 0 || H < 0 || Dc <= 0 || Dr < 0 || P <= 0 || num_pages < 0 || bt_stride < 0) return LADO_EINVAL;
    const int rc = check_block_table(B, P, num_pages, bt_stride, block_table, seq_lens);
    if (rc != LADO_OK) return rc;
    return mla_decode_impl(B, H, Dc, Dr, q, pages, 1, kv_scale, 0, block_table, bt_stride, P, seq_lens, gate, scale,
                           o, lse, nthreads);
}

/*
 * Rotary position embedding of the 64-wide RoPE part of a latent-attention query or key ([P2]
 * "Context: 1M in the claims, 262,144 in the config": position enters the model only in the MLA
 * layers, through 64 of each head's 192 query-key dimensions; rope_theta = 6,000,000 with no
 * scaling). The pages do not say how dimensions pair up; the two usual pairings are offered:
 *   interleaved == 0 (rotate-half): pair i is (x[i], x[i + D/2]), i < D/2
 *   interleaved == 1:               pair i is (x[2i], x[2i + 1])
 * Pair i turns by the angle p * theta^(-2i/D):  (a, b) -> (a cos - b sin, b cos + a sin).
 * x, out: [n][D] (out may alias x); positions: [n]; D even.
 */
int lado_rope(int n, int D, const double *x, const long long *positions, double theta, int interleaved,
              double *out) {
    if (n < 0 || D <= 0 || (D & 1) || !(theta > 0.0)) return LADO_EINVAL;
    const int half = D / 2;
    for (int r = 0; r < n; ++r) {
        const double *xr = x + (size_t)r * D;
        double *yr = out + (size_t)r * D;
        double tmp[1024];
        if (D > 1024) return LADO_EINVAL;
        for (int d = 0; d < D; ++d) tmp[d] = xr[d];
        for (int i = 0; i < half; ++i) {
            const double ang = (double)positions[r] * pow(theta, -2.0 * i / D);
            const double c = cos(ang), sn = sin(ang);
            const int ia = interleaved ? 2 * i : i;
            const int ib = interleaved ? 2 * i + 1 : i + half;
            const double a = tmp[ia], b = tmp[ib];
            yr[ia] = a * c - b * sn;
            yr[ib] = b * c + a * sn;
        }
    }
    return LADO_OK;
}

/* IEEE binary64 -> bfloat16 bit pattern, rounded once, to nearest with ties to even: the two
 * bf16 neighbours of |v| are multiples of the spacing 2^(e-8) of 8-bit significands in v's binade
 * (2^-133 below the normal range); the nearer one wins, a tie goes to the even significand. */
static uint16_t double_to_bf16_bits(double v) {
    if (v != v) return 0x7FC0u;
    const uint16_t sign = signbit(v) ? 0x8000u : 0u;
    const double a = fabs(v);
    if (a == 0.0) return sign;
    if (isinf(a)) return (uint16_t)(sign | 0x7F80u);
    int e;
    frexp(a, &e); /* a = m * 2^e, m in [0.5, 1) */
    int q = e - 8;
    if (q < -133) q = -133;
    const double ulp = ldexp(1.0, q);
    const double lo = floor(a / ulp) * ulp, hi = lo + ulp;
    const double dlo = a - lo, dhi = hi - a;
    double r;
    if (dlo < dhi)
        r = lo;
    else if (dhi < dlo)
        r = hi;
    else
        r = (fmod(lo / ulp, 2.0) == 0.0) ? lo : hi;
    if (r >= ldexp(1.0, 128)) return (uint16_t)(sign | 0x7F80u);
    const float f = (float)r; /* exact: r has at most 8 significant bits */
    uint32_t u;
    memcpy(&u, &f, 4);
    return (uint16_t)(sign | (u >> 16));
}

/* For tests: the bf16 rounding above, applied to n values. */
int lado_round_bf16(int n, const double *x, uint16_t *out) {
    if (n < 0) return LADO_EINVAL;
    for (int i = 0; i < n; ++i) out[i] = double_to_bf16_bits(x[i]);
    return LADO_OK;
}

/*
 * A new latent-cache row for each of n tokens ([P1] "How big is the cache per token, exactly?":
 * the row is the 512-wide compressed latent followed by the 64-wide RoPE key, in bf16): the latent
 * is stored as given, the RoPE key is turned to its position (lado_rope, fp64) and rounded to
 * bf16 once. c_kv: [n][Dc] bf16 bits; k_pe: [n][Dr] bf16 bits; out: [n][Dc + Dr] bf16 bits.
 */
int lado_mla_cache_row(int n, int Dc, int Dr, const uint16_t *c_kv, const uint16_t *k_pe, const long long *positions,
                       double theta, int interleaved, uint16_t *out) {
    if (n < 0 || Dc < 0 || Dr <= 0 || Dr > 1024 || (Dr & 1)) return LADO_EINVAL;
    double x[1024], y[1024];
    for (int r = 0; r < n; ++r) {
        uint16_t *o = out + (size_t)r * (Dc + Dr);
        memcpy(o, c_kv + (size_t)r * Dc, sizeof(uint16_t) * (size_t)Dc);
        for (int d = 0; d < Dr; ++d) x[d] = bf16_bits_to_double(k_pe[(size_t)r * Dr + d]);
        const int rc = lado_rope(1, Dr, x, positions + r, theta, interleaved, y);
        if (rc != LADO_OK) return rc;
        for (int d = 0; d < Dr; ++d) o[Dc + d] = double_to_bf16_bits(y[d]);
    }
    return LADO_OK;
}

/*
 * A new FP8 latent-cache row for each of n tokens: the bf16 row of lado_mla_cache_row before its
 * final rounding (the latent as given, the RoPE key turned in fp64), each element x stored as
 * the E4M3 code of x / kv_scale. The quotient is taken in fp32, the precision the code is decided
 * in on the GPU: x rounded to fp32 (exact for the bf16 latent), divided by fp32(kv_scale) with
 * one rounding to nearest, then rounded once more to E4M3 (double_to_e4m3).
 * out: [n][Dc + Dr] E4M3 codes.
 */
int lado_mla_cache_row_fp8(int n, int Dc, int Dr, const uint16_t *c_kv, const uint16_t *k_pe,
                           const long long *positions, double theta, int interleaved, double kv_scale, uint8_t *out) {
    if (n < 0 || Dc < 0 || Dr <= 0 || Dr > 1024 || (Dr & 1) || !(kv_scale > 0.0)) return LADO_EINVAL;
    const float s = (float)kv_scale;
    double x[1024], y[1024];
    for (int r = 0; r < n; ++r) {
        uint8_t *o = out + (size_t)r * (Dc + Dr);
        for (int d = 0; d < Dc; ++d) {
            const float v = (float)bf16_bits_to_double(c_kv[(size_t)r * Dc + d]);
            o[d] = double_to_e4m3((double)(v / s));
        }
        for (int d = 0; d < Dr; ++d) x[d] = bf16_bits_to_double(k_pe[(size_t)r * Dr + d]);
        const int rc = lado_rope(1, Dr, x, positions + r, theta, interleaved, y);
        if (rc != LADO_OK) return rc;
        for (int d = 0; d < Dr; ++d) {
            const float v = (float)y[d];
            o[Dc + d] = double_to_e4m3((double)(v / s));
        }
    }
    return LADO_OK;
}

/*
 * Output gate of a KDA head, the epilogue of the decode step ([P2] "How KDA and MLA split the
 * work": besides q, k, v and the decay, each KDA layer projects an output gate, full-rank). The
 * page does not give its form; the reading is the gated RMSNorm of the published KDA: per head,
 *   out = o / sqrt(mean(o^2) + eps) * w * sigmoid(g)
 * over the head's D output values (w per channel, shared by the heads; w == NULL means 1).
 * o, g, out: [n][D]; w: [D] or NULL.
 */
int lado_gated_rmsnorm(int n, int D, const double *o, const double *g, const double *w, double eps, double *out) {
    if (n < 0 || D <= 0 || !(eps >= 0.0)) return LADO_EINVAL;
    for (int r = 0; r < n; ++r) {
        const double *orow = o + (size_t)r * D;
        const double *grow = g + (size_t)r * D;
        double ss = 0.0;
        for (int d = 0; d < D; ++d) ss += orow[d] * orow[d];
        const double inv = 1.0 / sqrt(ss / D + eps);
        for (int d = 0; d < D; ++d) {
            const double wd = w ? w[d] : 1.0;
            out[(size_t)r * D + d] = orow[d] * inv * wd / (1.0 + exp(-grow[d]));
        }
    }
    return LADO_OK;
}
