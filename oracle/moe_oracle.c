/*
 * moe_oracle.c - plain, slow, fp64 CPU oracle of the mixture-of-experts FFN
 * block (router -> top-k routed SwiGLU experts + always-active shared experts
 * -> gate-weighted combine).
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the parity reference for the CUDA
 * path.  Only the test suite, the smoke check and the benchmark's CPU-baseline
 * leg may load it.  It shares no code, header, table or helper with the CUDA
 * library, and the library never calls it.
 *
 * Source of the method (archdiff.com architecture-comparison pages on
 * Qwen3.5-397B-A17B, DeepSeek-V4-Pro, Qwen3.8, Gemma 4 and DeepSeek-V4.1-Flash):
 *   - Qwen3.5's router: a linear map gives one score per expert, a softmax
 *     turns them into probabilities, the k largest are kept and renormalised,
 *     and no bias takes part in the choice.
 *     (qwen3-5-vs-deepseek-v4, component table, Qwen3.5 router cell;
 *      qwen3-5-vs-gemma-4, component table, Qwen3.5 router cell)
 *   - DeepSeek-V4-Pro's router: sqrt(softplus) affinities; a per-expert bias
 *     is added only while the k experts are chosen; the chosen affinities are
 *     renormalised and multiplied by a constant.  The router node of its
 *     diagram names the sigmoid form beside it.
 *     (qwen3-5-vs-deepseek-v4, DeepSeek-V4-Pro diagram and router cell)
 *   - The routed SwiGLU experts (the top 6 to 22 of 256 to 896) and one or
 *     two shared experts that every token uses; the residual add is drawn as
 *     its own node after the block (qwen3-5-vs-deepseek-v4, Qwen3.5 diagram).
 *   - SwiGLU experts at full model width, no latent projection
 *     (qwen3-5-vs-gemma-4, component table, Qwen3.5 routed-experts cell).
 *   - The shared expert's output is added to the routed sum
 *     (qwen3-5-vs-gemma-4, component table, Qwen3.5 shared-expert cell).
 *
 * Readings where the pages are silent (each also listed in the design notes):
 *   - ties in the top-k order go to the lower expert index;
 *   - the softmax selection key is the softmax probability itself;
 *   - the renormalisation denominator is guarded by max(sum, DBL_MIN);
 *   - the shared experts are ungated (weight 1) unless gate vectors are
 *     given, then scaled by sigma(w_s . x) per token (qwen3-5-vs-gemma-4,
 *     component table, Qwen3.5 shared-expert cell);
 *   - experts carry no biases; the block output is residual-free;
 *   - weights follow the [out, in] (nn.Linear) layout:
 *       W_router [E,d], W_gate/W_up [E,f,d], W_down [E,d,f],
 *       W_shared_gate/up [S,fs,d], W_shared_down [S,d,fs].
 *
 * Every floating-point value is carried in double.  bf16 inputs are widened
 * exactly (a bf16 is the top half of an IEEE binary32).
 */
#include <math.h>
#include <float.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <pthread.h>

#define ORACLE_SOFTMAX 0
#define ORACLE_SIGMOID 1
#define ORACLE_SQRT_SOFTPLUS 2

/* bf16 bits -> double, exact. */
static double bf16_to_double(uint16_t b)
{
    uint32_t u = ((uint32_t)b) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* Linear router: logit_e = sum_i x_i * W_router[e,i]. */
static void router_logits(int d, int E, const uint16_t *x_t, const uint16_t *Wr, double *logit)
{
    for (int e = 0; e < E; ++e) {
        double acc = 0.0;
        const uint16_t *w = Wr + (size_t)e * d;
        for (int i = 0; i < d; ++i)
            acc += bf16_to_double(x_t[i]) * bf16_to_double(w[i]);
        logit[e] = acc;
    }
}

/* softplus(z) = log(1 + exp(z)), written in the overflow-free form
 * max(z,0) + log1p(exp(-|z|)). */
static double softplus(double z)
{
    return (z > 0.0 ? z : 0.0) + log1p(exp(-fabs(z)));
}

/* Scores s_e from the logits.
 *   SOFTMAX:       s_e = exp(l_e - max l) / sum_e' exp(l_e' - max l)
 *   SIGMOID:       s_e = 1 / (1 + exp(-l_e))
 *   SQRT_SOFTPLUS: s_e = sqrt(softplus(l_e)) */
static void scores_from_logits(int E, int score_fn, const double *logit, double *s)
{
    if (score_fn == ORACLE_SOFTMAX) {
        double m = logit[0];
        for (int e = 1; e < E; ++e) if (logit[e] > m) m = logit[e];
        double z = 0.0;
        for (int e = 0; e < E; ++e) { s[e] = exp(logit[e] - m); z += s[e]; }
        for (int e = 0; e < E; ++e) s[e] /= z;
    } else if (score_fn == ORACLE_SIGMOID) {
        for (int e = 0; e < E; ++e) s[e] = 1.0 / (1.0 + exp(-logit[e]));
    } else {
        for (int e = 0; e < E; ++e) s[e] = sqrt(softplus(logit[e]));
    }
}

/* Order used to pick the top k: larger selection key first, and on equal keys
 * the lower expert index first. */
typedef struct { double key; int idx; } keyed;

static int keyed_cmp(const void *pa, const void *pb)
{
    const keyed *a = (const keyed *)pa, *b = (const keyed *)pb;
    if (a->key > b->key) return -1;
    if (a->key < b->key) return 1;
    return (a->idx < b->idx) ? -1 : (a->idx > b->idx);
}

/* SwiGLU expert on one token, accumulated into y with weight w:
 *   g = G x, u = U x, h = SiLU(g) * u with SiLU(z) = z / (1 + exp(-z)),
 *   y += w * (D h).
 * G, U are [ff, d]; D is [d, ff]. */
static void swiglu_expert_accumulate(int d, int ff, const uint16_t *x_t,
                                     const uint16_t *G, const uint16_t *U, const uint16_t *D,
                                     double w, double *h, double *y)
{
    for (int j = 0; j < ff; ++j) {
        double g = 0.0, u = 0.0;
        const uint16_t *gr = G + (size_t)j * d, *ur = U + (size_t)j * d;
        for (int i = 0; i < d; ++i) {
            double xi = bf16_to_double(x_t[i]);
            g += xi * bf16_to_double(gr[i]);
            u += xi * bf16_to_double(ur[i]);
        }
        h[j] = (g / (1.0 + exp(-g))) * u;
    }
    for (int m = 0; m < d; ++m) {
        double acc = 0.0;
        const uint16_t *dr = D + (size_t)m * ff;
        for (int j = 0; j < ff; ++j)
            acc += bf16_to_double(dr[j]) * h[j];
        y[m] += w * acc;
    }
}

typedef struct {
    int T, d, E, k, f, S, fs;
    const uint16_t *x, *Wr;
    const float *bias;
    const uint16_t *Wg, *Wu, *Wd, *Wsg, *Wsu, *Wsd;
    int score_fn, norm_topk;
    double route_scale;
    const int32_t *tokens;   /* n_tokens token ids, or NULL for 0..n_tokens-1 */
    int n_tokens;
    const int32_t *forced;   /* [n_tokens,k] expert ids to use instead of the router's pick, or NULL */
    const double *forced_w;  /* [n_tokens,k] combine weights to use as given (with forced), or NULL */
    const uint16_t *sgate;   /* [S,d] shared-expert gate vectors (bf16), or NULL = ungated */
    int route_only;          /* 1: skip the experts */
    double *out;             /* [n_tokens,d] or NULL */
    int32_t *topk_idx;       /* [n_tokens,k] or NULL */
    double *topk_w;          /* [n_tokens,k] or NULL */
    double *sel_keys;        /* [n_tokens,k+1] selection keys in picked order (k+1-th = -inf if k == E) */
    int32_t *sel_order;      /* [n_tokens,k+1] the experts of those keys (k+1-th = -1 if k == E) */
    double *logits_out;      /* [n_tokens,E] or NULL */
    double *scores_out;      /* [n_tokens,E] or NULL */
    double *keys_out;        /* [n_tokens,E] selection keys, or NULL */
    int next;                /* work counter */
    pthread_mutex_t mu;
    int status;
} oracle_job;

/* One token, the plain definition:
 *  1. logits l = W_router x
 *  2. scores s from l (softmax | sigmoid | sqrt-softplus)
 *  3. selection key c_e = s_e + b_e for sigmoid / sqrt-softplus with a bias,
 *     c_e = s_e otherwise (the bias only picks experts)
 *  4. sel = the k largest keys, descending, ties to the lower index
 *  5. w_j = s_{sel_j}; if norm_topk, w_j /= sum_j s_{sel_j}; w_j *= route_scale
 *     (external routing: the given experts and weights replace 4 and 5)
 *  6. out = sum_j w_j SwiGLU_{sel_j}(x) + sum_s g_s SwiGLU_shared_s(x),
 *     g_s = 1, or sigma(w_s . x) with gate vectors */
static int oracle_token(oracle_job *J, int n, double *logit, double *s, keyed *kv,
                        double *h, double *y)
{
    const int d = J->d, E = J->E, k = J->k;
    const int t = J->tokens ? J->tokens[n] : n;
    if (t < 0 || t >= J->T) return -1;
    const uint16_t *x_t = J->x + (size_t)t * d;

    router_logits(d, E, x_t, J->Wr, logit);
    scores_from_logits(E, J->score_fn, logit, s);
    if (J->logits_out) memcpy(J->logits_out + (size_t)n * E, logit, sizeof(double) * E);
    if (J->scores_out) memcpy(J->scores_out + (size_t)n * E, s, sizeof(double) * E);

    const int use_bias = (J->bias != NULL) && (J->score_fn != ORACLE_SOFTMAX);
    for (int e = 0; e < E; ++e) {
        kv[e].key = s[e] + (use_bias ? (double)J->bias[e] : 0.0);
        kv[e].idx = e;
    }
    if (J->keys_out)
        for (int e = 0; e < E; ++e) J->keys_out[(size_t)n * E + e] = kv[e].key;
    qsort(kv, (size_t)E, sizeof(keyed), keyed_cmp);
    if (J->sel_keys) {
        double *sk = J->sel_keys + (size_t)n * (k + 1);
        for (int j = 0; j <= k; ++j) sk[j] = (j < E) ? kv[j].key : -INFINITY;
    }
    if (J->sel_order) {
        int32_t *so = J->sel_order + (size_t)n * (k + 1);
        for (int j = 0; j <= k; ++j) so[j] = (j < E) ? kv[j].idx : -1;
    }

    int sel[64];
    if (J->forced) {
        for (int j = 0; j < k; ++j) {
            int e = J->forced[(size_t)n * k + j];
            if (e < 0 || e >= E) return -1;
            sel[j] = e;
        }
    } else {
        for (int j = 0; j < k; ++j) sel[j] = kv[j].idx;
    }

    double w[64], denom = 0.0;
    if (J->forced && J->forced_w) {
        /* external routing: the caller's weights, as given */
        for (int j = 0; j < k; ++j) w[j] = J->forced_w[(size_t)n * k + j];
    } else {
        for (int j = 0; j < k; ++j) { w[j] = s[sel[j]]; denom += w[j]; }
        if (J->norm_topk) {
            if (denom < DBL_MIN) denom = DBL_MIN;
            for (int j = 0; j < k; ++j) w[j] /= denom;
        }
        for (int j = 0; j < k; ++j) w[j] *= J->route_scale;
    }

    if (J->topk_idx) for (int j = 0; j < k; ++j) J->topk_idx[(size_t)n * k + j] = sel[j];
    if (J->topk_w) for (int j = 0; j < k; ++j) J->topk_w[(size_t)n * k + j] = w[j];
    if (J->route_only || !J->out) return 0;

    for (int m = 0; m < d; ++m) y[m] = 0.0;
    const size_t fsz = (size_t)J->f * d;
    for (int j = 0; j < k; ++j) {
        const size_t e = (size_t)sel[j];
        swiglu_expert_accumulate(d, J->f, x_t, J->Wg + e * fsz, J->Wu + e * fsz, J->Wd + e * fsz,
                                 w[j], h, y);
    }
    const size_t ssz = (size_t)J->fs * d;
    for (int sh = 0; sh < J->S; ++sh) {
        /* shared expert weight: 1 (ungated), or sigma(w_s . x) with the
         * per-token gate of the Qwen3.5 shared expert */
        double gw = 1.0;
        if (J->sgate) {
            double z = 0.0;
            const uint16_t *gv = J->sgate + (size_t)sh * d;
            for (int i = 0; i < d; ++i) z += bf16_to_double(gv[i]) * bf16_to_double(x_t[i]);
            gw = 1.0 / (1.0 + exp(-z));
        }
        swiglu_expert_accumulate(d, J->fs, x_t, J->Wsg + sh * ssz, J->Wsu + sh * ssz,
                                 J->Wsd + sh * ssz, gw, h, y);
    }
    memcpy(J->out + (size_t)n * d, y, sizeof(double) * d);
    return 0;
}

static void *oracle_worker(void *arg)
{
    oracle_job *J = (oracle_job *)arg;
    const int E = J->E, d = J->d;
    const int hmax = J->f > J->fs ? J->f : J->fs;
    double *logit = (double *)malloc(sizeof(double) * E);
    double *s = (double *)malloc(sizeof(double) * E);
    keyed *kv = (keyed *)malloc(sizeof(keyed) * E);
    double *h = (double *)malloc(sizeof(double) * (hmax > 0 ? hmax : 1));
    double *y = (double *)malloc(sizeof(double) * d);
    int bad = (!logit || !s || !kv || !h || !y);
    for (;;) {
        pthread_mutex_lock(&J->mu);
        int n = J->next++;
        if (bad) J->status = -2;
        pthread_mutex_unlock(&J->mu);
        if (bad || n >= J->n_tokens) break;
        if (oracle_token(J, n, logit, s, kv, h, y) != 0) {
            pthread_mutex_lock(&J->mu);
            J->status = -1;
            pthread_mutex_unlock(&J->mu);
        }
    }
    free(logit); free(s); free(kv); free(h); free(y);
    return NULL;
}

/* Entry point.  Returns 0 on success, -1 on invalid arguments, -2 on
 * allocation failure.  Outputs are per evaluated token n (0..n_tokens-1),
 * token id tokens[n] (or n when tokens is NULL). */
int oracle_moe_forward(int T, int d, int E, int k, int f, int S, int fs,
                       const uint16_t *x, const uint16_t *Wr, const float *bias,
                       const uint16_t *Wg, const uint16_t *Wu, const uint16_t *Wd,
                       const uint16_t *Wsg, const uint16_t *Wsu, const uint16_t *Wsd,
                       int score_fn, int norm_topk, double route_scale,
                       const int32_t *tokens, int n_tokens, const int32_t *forced,
                       const double *forced_w, const uint16_t *sgate, int route_only,
                       double *out, int32_t *topk_idx, double *topk_w, double *sel_keys,
                       int32_t *sel_order, double *logits_out, double *scores_out, double *keys_out,
                       int n_threads)
{
    if (T < 1 || d < 1 || E < 1 || k < 1 || k > E || k > 64 || n_tokens < 0) return -1;
    if (score_fn < 0 || score_fn > 2 || !x || !Wr) return -1;
    if (!route_only && (f < 1 || !Wg || !Wu || !Wd || S < 0)) return -1;
    if (!route_only && S > 0 && (fs < 1 || !Wsg || !Wsu || !Wsd)) return -1;
    if (n_threads < 1) n_threads = 1;
    if (n_threads > 512) n_threads = 512;

    oracle_job J;
    memset(&J, 0, sizeof J);
    J.T = T; J.d = d; J.E = E; J.k = k; J.f = f; J.S = S; J.fs = fs;
    J.x = x; J.Wr = Wr; J.bias = bias;
    J.Wg = Wg; J.Wu = Wu; J.Wd = Wd; J.Wsg = Wsg; J.Wsu = Wsu; J.Wsd = Wsd;
    J.score_fn = score_fn; J.norm_topk = norm_topk; J.route_scale = route_scale;
    J.tokens = tokens; J.n_tokens = n_tokens; J.forced = forced; J.route_only = route_only;
    J.forced_w = forced_w; J.sgate = sgate;
    J.out = out; J.topk_idx = topk_idx; J.topk_w = topk_w; J.sel_keys = sel_keys;
    J.sel_order = sel_order;
    J.logits_out = logits_out; J.scores_out = scores_out; J.keys_out = keys_out;
    pthread_mutex_init(&J.mu, NULL);

    pthread_t th[512];
    int started = 0;
    for (int i = 0; i < n_threads; ++i) {
        if (pthread_create(&th[i], NULL, oracle_worker, &J) != 0) break;
        ++started;
    }
    if (started == 0) oracle_worker(&J);
    for (int i = 0; i < started; ++i) pthread_join(th[i], NULL);
    pthread_mutex_destroy(&J.mu);
    return J.status;
}

/* ------------------------------------------------------------------ RMSNorm
 * The pre-norm RMSNorm that produces the block's input (qwen3-5-vs-deepseek-v4,
 * Qwen3.5 diagram: the pre-norm RMSNorm node right before the router), with
 * zero-centred gains (same page, component table, Qwen3.5 residual-stream
 * cell): the stored gain g is centred on zero, so the scale applied is 1 + g.
 *
 *   y[t,i] = x[t,i] / sqrt(mean_j x[t,j]^2 + eps) * (1 + g[i])
 *
 * in double, then rounded to bf16 (nearest, ties to even) because the block
 * takes bf16 input.  eps is not given on the pages; the caller passes it. */

/* double -> bf16 bits, round to nearest, ties to even, straight from the
 * double (no intermediate float rounding).  bf16 keeps 8 significant bits; a
 * value in [2^(e-1), 2^e) is rounded to a multiple of 2^(e-8), and below the
 * smallest normal (2^-126) to a multiple of 2^-133.  The rounded value is
 * exactly representable in binary32, whose top 16 bits are the bf16. */
uint16_t oracle_double_to_bf16(double v)
{
    if (isnan(v)) return 0x7FC0;
    const uint16_t sign = signbit(v) ? 0x8000 : 0;
    double a = fabs(v);
    if (a == 0.0) return sign;
    if (isinf(a)) return (uint16_t)(sign | 0x7F80);
    int e;
    frexp(a, &e);                       /* a = m * 2^e, 0.5 <= m < 1 */
    int qe = e - 8;
    if (qe < -133) qe = -133;
    double q = nearbyint(ldexp(a, -qe)); /* exact scaling; default mode = ties to even */
    double r = ldexp(q, qe);
    if (r >= 0x1p128) return (uint16_t)(sign | 0x7F80);
    float f = (float)r;                 /* exact */
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    return (uint16_t)(sign | (u >> 16));
}

int oracle_rmsnorm(int T, int d, const uint16_t *x, const uint16_t *gain, double eps,
                   double *y, uint16_t *y_bf16)
{
    if (T < 0 || d < 1 || !x || !gain || !(eps >= 0.0)) return -1;
    for (int t = 0; t < T; ++t) {
        const uint16_t *xr = x + (size_t)t * d;
        double ss = 0.0;
        for (int i = 0; i < d; ++i) {
            const double v = bf16_to_double(xr[i]);
            ss += v * v;
        }
        const double rstd = 1.0 / sqrt(ss / d + eps);
        for (int i = 0; i < d; ++i) {
            const double v = bf16_to_double(xr[i]) * rstd * (1.0 + bf16_to_double(gain[i]));
            if (y) y[(size_t)t * d + i] = v;
            if (y_bf16) y_bf16[(size_t)t * d + i] = oracle_double_to_bf16(v);
        }
    }
    return 0;
}

/* ------------------------------------------------------------------ FP8 weights
 * Block-scaled FP8 expert weights (the pages mention an FP8 release of the
 * Qwen3.5 weights and block-scaled FP8 in the training blueprint:
 * qwen3-5-vs-gemma-4, component table, Qwen3.5 routed-experts cell;
 * qwen3-5-vs-deepseek-v4, blueprint diagram).
 * The pages give no block size or scale format.  Reading: OCP MX-style
 * blocks of 32 consecutive elements along the input dimension K, each with
 * one power-of-two scale stored as an unbiased-exponent byte (UE8M0):
 *   w[g, r, c] = e4m3(q[g, r, c]) * 2^(s[g, c / 32, r] - 127)
 * Scales are stored block-major ([G, K/32, rows]).
 *
 * E4M3 (the OCP "E4M3FN" encoding): 1 sign bit, 4 exponent bits with bias 7,
 * 3 mantissa bits.  Exponent field 0 is subnormal, m/8 * 2^-6; exponent
 * field 15 with mantissa 7 is NaN; there are no infinities, so the largest
 * finite magnitude is 1.75 * 2^8 = 448. */
double oracle_e4m3_to_double(uint8_t b)
{
    const int s = b >> 7, e = (b >> 3) & 15, m = b & 7;
    double v;
    if (e == 15 && m == 7) return NAN;
    if (e == 0) v = ldexp((double)m / 8.0, -6);
    else v = ldexp(1.0 + (double)m / 8.0, e - 7);
    return s ? -v : v;
}

/* Dequantises G x rows x K weights to bf16 bits.  Returns 0, -1 for bad
 * arguments (K not a multiple of 32), or -2 when some value is NaN or not
 * exactly representable in bf16 (the block then has no exact bf16 form). */
int oracle_dequant_mxfp8(int G, int rows, int K, const uint8_t *q, const uint8_t *scale, uint16_t *w_bf16)
{
    if (G < 0 || rows < 0 || K < 32 || K % 32 != 0 || !q || !scale || !w_bf16) return -1;
    const int nb = K / 32;
    for (int g = 0; g < G; ++g)
        for (int r = 0; r < rows; ++r)
            for (int c = 0; c < K; ++c) {
                const uint8_t u = scale[((size_t)g * nb + c / 32) * rows + r];
                if (u == 255) return -2;
                const double v = oracle_e4m3_to_double(q[((size_t)g * rows + r) * K + c]) * ldexp(1.0, (int)u - 127);
                if (isnan(v)) return -2;
                const uint16_t b = oracle_double_to_bf16(v);
                if (bf16_to_double(b) != v) return -2;
                w_bf16[((size_t)g * rows + r) * K + c] = b;
            }
    return 0;
}
