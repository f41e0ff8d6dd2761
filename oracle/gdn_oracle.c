/*
 * gdn_oracle.c -- plain FP64 CPU definition of the Gated DeltaNet token mixer.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the checker the CUDA library is
 * compared against.  Only the tests, the package's smoke check and the
 * benchmark's CPU-baseline leg may load it; the library never calls it and
 * shares no code, header or table with it.
 *
 * Every stage is written as its plain definition, one token at a time, with
 * no blocking, chunking or reordering:
 *
 *   conv   : depthwise causal convolution of kernel 4 over the q, k and v
 *            channels, followed by SiLU ("Qwen3.8-2.4T-A95B vs Inkling",
 *            component table, Gated DeltaNet row; "Qwen3.8 2.4T A95B", raw
 *            config fields, linear_conv_kernel_dim = 4).
 *   l2norm : q and k of every q/k head divided by their Euclidean norm
 *            (the Gated DeltaNet layer normalises q and k before the
 *            recurrence; the pages state the same normalisation for KDA in
 *            "Inkling vs Kimi K3", component table, linear-attention row).
 *   gates  : g = -exp(A_log) * softplus(a + dt_bias), beta = sigmoid(b),
 *            one scalar per value head and token ("Qwen3.8-2.4T-A95B vs
 *            Inkling", component table, Gated DeltaNet row).
 *   delta  : the gated delta rule on a d_v x d_k FP32-or-wider state per
 *            value head,
 *               S_t = exp(g_t) S_{t-1} (I - beta_t k_t k_t^T) + beta_t v_t k_t^T,
 *               o_t = S_t q_t,
 *            where value head h reads q/k head floor(h / G), G = H_v / H_k
 *            ("Qwen3.8-2.4T-A95B vs Inkling", Gated DeltaNet row: 16 q/k heads
 *            serve 128 value heads, 8 each; "Qwen3.8 2.4T A95B", raw config
 *            fields, mamba_ssm_dtype = float32 for the state).
 *   norm   : per value head RMSNorm of o, times a weight, times SiLU(z)
 *            ("Qwen3.8-2.4T-A95B vs Inkling", component table, output-gate
 *            row: output_gate_type swish after a per-head RMSNorm;
 *            "Qwen3.8 2.4T A95B", raw config fields, rms_norm_eps = 1e-6).
 *
 * Kimi Delta Attention (KDA), the per-channel-decay variant ("Inkling vs Kimi
 * K3", component table, linear-attention and output-gate rows), adds
 *
 *   kda gates : g = -5 sigmoid(exp(A_log) z), one log-decay per key channel,
 *               token and head (z is the decay input of the channel), and
 *               beta = sigmoid(b);
 *   kda delta : S_t = S_{t-1} Diag(exp(g_t)) (I - beta_t k_t k_t^T) + beta_t v_t k_t^T,
 *               o_t = S_t q_t, one state per head (no head sharing);
 *   kda norm  : per head RMSNorm of o, times a weight, times sigmoid(gate)
 *               (a full-rank channel-wise sigmoid gate).
 *
 * All arrays are row-major, contiguous, double precision.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------ conv */

/*
 * Depthwise causal convolution + SiLU.
 *
 *   xc_t[c] = sum_{i=0..K-1} w[c][i] * x_{t-(K-1)+i}[c]
 *   out_t[c] = xc_t[c] * sigmoid(xc_t[c])
 *
 * so w[c][K-1] multiplies the current token.  Positions before the first
 * token come from `window` ([K-1, C], oldest row first) or are zero when
 * `window` is NULL.  There is no bias.
 *   x   : [T, C] pre-convolution rows
 *   w   : [C, K]
 *   out : [T, C]
 */
void gdn_oracle_conv_silu(const double *x, const double *window, const double *w,
                          int64_t T, int64_t C, int64_t K, double *out)
{
    for (int64_t t = 0; t < T; ++t) {
        for (int64_t c = 0; c < C; ++c) {
            double acc = 0.0;
            for (int64_t i = 0; i < K; ++i) {
                int64_t src = t - (K - 1) + i; /* token index of this tap */
                double xv;
                if (src >= 0)
                    xv = x[src * C + c];
                else if (window)
                    xv = window[(K - 1 + src) * C + c]; /* row K-1+src of the window */
                else
                    xv = 0.0;
                acc += w[c * K + i] * xv;
            }
            out[t * C + c] = acc / (1.0 + exp(-acc));
        }
    }
}

/* ---------------------------------------------------------------- l2norm */

/*
 * In place: every row of length d becomes row * scale / sqrt(sum(row^2) + eps).
 */
void gdn_oracle_l2norm_rows(double *x, int64_t rows, int64_t d, double eps, double scale)
{
    for (int64_t r = 0; r < rows; ++r) {
        double ss = 0.0;
        for (int64_t i = 0; i < d; ++i)
            ss += x[r * d + i] * x[r * d + i];
        double f = scale / sqrt(ss + eps);
        for (int64_t i = 0; i < d; ++i)
            x[r * d + i] *= f;
    }
}

/* ----------------------------------------------------------------- gates */

static double softplus(double x)
{
    /* log(1 + e^x) without overflow: max(x, 0) + log1p(e^{-|x|}) */
    return (x > 0.0 ? x : 0.0) + log1p(exp(-fabs(x)));
}

/*
 * Per token t and value head h:
 *   g[t][h]    = -exp(A_log[h]) * softplus(a[t][h] + dt_bias[h])
 *   beta[t][h] = 1 / (1 + exp(-b[t][h]))
 * a, b, g, beta are [T, H]; A_log and dt_bias are [H].
 */
void gdn_oracle_gates(const double *a, const double *b, const double *A_log,
                      const double *dt_bias, int64_t T, int64_t H, double *g, double *beta)
{
    for (int64_t t = 0; t < T; ++t) {
        for (int64_t h = 0; h < H; ++h) {
            g[t * H + h] = -exp(A_log[h]) * softplus(a[t * H + h] + dt_bias[h]);
            beta[t * H + h] = 1.0 / (1.0 + exp(-b[t * H + h]));
        }
    }
}

/* ------------------------------------------------------------- delta rule */

typedef struct {
    const double *q, *k, *v, *g, *beta;
    int64_t T, H_k, H_v, d_k, d_v;
    double *state, *o;
    int64_t next_head; /* shared job counter, guarded by mu */
    pthread_mutex_t mu;
} delta_job;

/*
 * One value head h over all T tokens.  The state S is [d_v][d_k] (row i is
 * the value channel, column j the key channel), so S k is a d_v vector.
 * Per token:  S <- alpha S;  p = S k;  u = beta (v - p);  S <- S + u k^T;
 * o = S q.  Expanding, S_t = alpha S_{t-1} - beta alpha S_{t-1} k k^T
 * + beta v k^T, which is the defining update written above.
 */
static void delta_one_head(delta_job *J, int64_t h)
{
    const int64_t G = J->H_v / J->H_k;
    const int64_t j = h / G; /* the q/k head this value head reads */
    const int64_t dk = J->d_k, dv = J->d_v;
    double *S = J->state + h * dv * dk;
    double *p = (double *)malloc(sizeof(double) * (size_t)dv);
    for (int64_t t = 0; t < J->T; ++t) {
        const double *kt = J->k + (t * J->H_k + j) * dk;
        const double *qt = J->q + (t * J->H_k + j) * dk;
        const double *vt = J->v + (t * J->H_v + h) * dv;
        const double alpha = exp(J->g[t * J->H_v + h]);
        const double bt = J->beta[t * J->H_v + h];
        for (int64_t i = 0; i < dv * dk; ++i)
            S[i] *= alpha;
        for (int64_t i = 0; i < dv; ++i) {
            double acc = 0.0;
            for (int64_t c = 0; c < dk; ++c)
                acc += S[i * dk + c] * kt[c];
            p[i] = acc;
        }
        for (int64_t i = 0; i < dv; ++i) {
            double u = bt * (vt[i] - p[i]);
            for (int64_t c = 0; c < dk; ++c)
                S[i * dk + c] += u * kt[c];
        }
        double *ot = J->o + (t * J->H_v + h) * dv;
        for (int64_t i = 0; i < dv; ++i) {
            double acc = 0.0;
            for (int64_t c = 0; c < dk; ++c)
                acc += S[i * dk + c] * qt[c];
            ot[i] = acc;
        }
    }
    free(p);
}

static void *delta_worker(void *arg)
{
    delta_job *J = (delta_job *)arg;
    for (;;) {
        pthread_mutex_lock(&J->mu);
        int64_t h = J->next_head++;
        pthread_mutex_unlock(&J->mu);
        if (h >= J->H_v)
            break;
        delta_one_head(J, h);
    }
    return NULL;
}

/*
 * Gated delta rule over one sequence of T tokens, all value heads.
 *   q, k  : [T, H_k, d_k]  (already convolved, activated and L2-normalised)
 *   v     : [T, H_v, d_v]
 *   g     : [T, H_v] log-decay;  beta : [T, H_v] write strength
 *   state : [H_v, d_v, d_k] initial state on entry, final state on return
 *   o     : [T, H_v, d_v]
 * Value heads are independent; they are spread over n_threads threads
 * (each head runs its tokens strictly in order).  Returns 0, or -1 if H_v
 * is not a multiple of H_k.
 */
int gdn_oracle_delta_rule(const double *q, const double *k, const double *v,
                          const double *g, const double *beta, int64_t T, int64_t H_k,
                          int64_t H_v, int64_t d_k, int64_t d_v, double *state, double *o,
                          int n_threads)
{
    if (H_k <= 0 || H_v <= 0 || H_v % H_k != 0)
        return -1;
    delta_job J = {q, k, v, g, beta, T, H_k, H_v, d_k, d_v, state, o, 0,
                   PTHREAD_MUTEX_INITIALIZER};
    if (n_threads < 1)
        n_threads = 1;
    if (n_threads > H_v)
        n_threads = (int)H_v;
    if (n_threads == 1) {
        delta_worker(&J);
        return 0;
    }
    pthread_t *th = (pthread_t *)malloc(sizeof(pthread_t) * (size_t)n_threads);
    for (int i = 0; i < n_threads; ++i)
        pthread_create(&th[i], NULL, delta_worker, &J);
    for (int i = 0; i < n_threads; ++i)
        pthread_join(th[i], NULL);
    free(th);
    return 0;
}

/* ----------------------------------------------------------- gated norm */

/*
 * Per row of length d:  y = o / sqrt(mean(o^2) + eps) * w * z * sigmoid(z).
 *   o, z, y : [rows, d];  w : [d]
 */
void gdn_oracle_gated_rmsnorm(const double *o, const double *z, const double *w,
                              int64_t rows, int64_t d, double eps, double *y)
{
    for (int64_t r = 0; r < rows; ++r) {
        double ss = 0.0;
        for (int64_t i = 0; i < d; ++i)
            ss += o[r * d + i] * o[r * d + i];
        double inv = 1.0 / sqrt(ss / (double)d + eps);
        for (int64_t i = 0; i < d; ++i) {
            double zi = z[r * d + i];
            y[r * d + i] = o[r * d + i] * inv * w[i] * (zi / (1.0 + exp(-zi)));
        }
    }
}

/* ------------------------------------------------------------------ KDA */

/*
 * Per token t, head h and key channel c:
 *   g[t][h][c] = -5 * sigmoid(exp(A_log[h]) * z[t][h][c])
 *   beta[t][h] = 1 / (1 + exp(-b[t][h]))
 * z, g are [T, H, d_k]; b, beta are [T, H]; A_log is [H].
 */
void gdn_oracle_kda_gates(const double *z, const double *b, const double *A_log, int64_t T,
                          int64_t H, int64_t d_k, double *g, double *beta)
{
    for (int64_t t = 0; t < T; ++t) {
        for (int64_t h = 0; h < H; ++h) {
            const double eA = exp(A_log[h]);
            for (int64_t c = 0; c < d_k; ++c) {
                const double x = eA * z[(t * H + h) * d_k + c];
                g[(t * H + h) * d_k + c] = -5.0 / (1.0 + exp(-x));
            }
            beta[t * H + h] = 1.0 / (1.0 + exp(-b[t * H + h]));
        }
    }
}

typedef struct {
    const double *q, *k, *v, *g, *beta;
    int64_t T, H, d_k, d_v;
    double *state, *o;
    int64_t next_head;
    pthread_mutex_t mu;
} kda_job;

/*
 * One head over all T tokens, S = [d_v][d_k].  Per token:
 *   S[i][c] <- S[i][c] * exp(g[c])   (the decay of key channel c, every row);
 *   p = S k;  u = beta (v - p);  S <- S + u k^T;  o = S q,
 * which expands to S_t = S_{t-1} D - beta S_{t-1} D k k^T + beta v k^T with
 * D = Diag(exp(g_t)): the defining update written above.
 */
static void kda_one_head(kda_job *J, int64_t h)
{
    const int64_t dk = J->d_k, dv = J->d_v, H = J->H;
    double *S = J->state + h * dv * dk;
    double *p = (double *)malloc(sizeof(double) * (size_t)dv);
    double *alpha = (double *)malloc(sizeof(double) * (size_t)dk);
    for (int64_t t = 0; t < J->T; ++t) {
        const double *kt = J->k + (t * H + h) * dk;
        const double *qt = J->q + (t * H + h) * dk;
        const double *vt = J->v + (t * H + h) * dv;
        const double *gt = J->g + (t * H + h) * dk;
        const double bt = J->beta[t * H + h];
        for (int64_t c = 0; c < dk; ++c)
            alpha[c] = exp(gt[c]);
        for (int64_t i = 0; i < dv; ++i)
            for (int64_t c = 0; c < dk; ++c)
                S[i * dk + c] *= alpha[c];
        for (int64_t i = 0; i < dv; ++i) {
            double acc = 0.0;
            for (int64_t c = 0; c < dk; ++c)
                acc += S[i * dk + c] * kt[c];
            p[i] = acc;
        }
        for (int64_t i = 0; i < dv; ++i) {
            double u = bt * (vt[i] - p[i]);
            for (int64_t c = 0; c < dk; ++c)
                S[i * dk + c] += u * kt[c];
        }
        double *ot = J->o + (t * H + h) * dv;
        for (int64_t i = 0; i < dv; ++i) {
            double acc = 0.0;
            for (int64_t c = 0; c < dk; ++c)
                acc += S[i * dk + c] * qt[c];
            ot[i] = acc;
        }
    }
    free(alpha);
    free(p);
}

static void *kda_worker(void *arg)
{
    kda_job *J = (kda_job *)arg;
    for (;;) {
        pthread_mutex_lock(&J->mu);
        int64_t h = J->next_head++;
        pthread_mutex_unlock(&J->mu);
        if (h >= J->H)
            break;
        kda_one_head(J, h);
    }
    return NULL;
}

/*
 * The KDA recurrence over one sequence of T tokens, all heads.
 *   q, k  : [T, H, d_k]  (convolved, activated and L2-normalised)
 *   v     : [T, H, d_v]
 *   g     : [T, H, d_k] per-channel log-decay;  beta : [T, H]
 *   state : [H, d_v, d_k] initial state on entry, final state on return
 *   o     : [T, H, d_v]
 * Heads are spread over n_threads threads (each runs its tokens in order).
 */
void gdn_oracle_kda_rule(const double *q, const double *k, const double *v, const double *g,
                         const double *beta, int64_t T, int64_t H, int64_t d_k, int64_t d_v,
                         double *state, double *o, int n_threads)
{
    kda_job J = {q, k, v, g, beta, T, H, d_k, d_v, state, o, 0, PTHREAD_MUTEX_INITIALIZER};
    if (n_threads < 1)
        n_threads = 1;
    if (n_threads > H)
        n_threads = (int)H;
    if (n_threads == 1) {
        kda_worker(&J);
        return;
    }
    pthread_t *th = (pthread_t *)malloc(sizeof(pthread_t) * (size_t)n_threads);
    for (int i = 0; i < n_threads; ++i)
        pthread_create(&th[i], NULL, kda_worker, &J);
    for (int i = 0; i < n_threads; ++i)
        pthread_join(th[i], NULL);
    free(th);
}

/*
 * Per row of length d:  y = o / sqrt(mean(o^2) + eps) * w * sigmoid(gate).
 *   o, gate, y : [rows, d];  w : [d]
 */
void gdn_oracle_sigmoid_rmsnorm(const double *o, const double *gate, const double *w,
                                int64_t rows, int64_t d, double eps, double *y)
{
    for (int64_t r = 0; r < rows; ++r) {
        double ss = 0.0;
        for (int64_t i = 0; i < d; ++i)
            ss += o[r * d + i] * o[r * d + i];
        double inv = 1.0 / sqrt(ss / (double)d + eps);
        for (int64_t i = 0; i < d; ++i)
            y[r * d + i] = o[r * d + i] * inv * w[i] / (1.0 + exp(-gate[r * d + i]));
    }
}
