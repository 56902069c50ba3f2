/*
 * KDA forward oracle -- TEST INFRASTRUCTURE ONLY.
 *
 * A plain, slow, fp64 CPU implementation of the Kimi Delta Attention forward
 * pass, written token by token in the order the AliceAI-Foundation KDA write-up
 * gives it ("二、KDA 线性注意力": the _torch_kda loop, the gate formula, the
 * depthwise causal conv with kernel 4 / padding 3 / no bias followed by SiLU,
 * L2-normalised q and k) and the Ling-3.0-flash-VL config table (kda_safe_gate,
 * kda_lower_bound = -5.0).  It shares no code with the CUDA library and is
 * never linked into it; only the tests, the bench's CPU-baseline leg and the
 * smoke check load it.
 *
 * Readings where the pages are silent or garbled (the "+" between alpha and
 * dt_bias lost in extraction; the safe gate as a hard clamp g = max(g, lb);
 * the L2-norm epsilon inside the square root; PyTorch Conv1d tap order; conv
 * channel blocks q | k | v) are the plain ones and are listed with the
 * project's design notes.
 *
 * Layouts (row-major, packed tokens):
 *   q, k, v        [Ttot, H*D]     raw, pre-conv
 *   conv_w         [3, H*D, 4]     w[.., 3] multiplies the current token
 *   alpha          [Ttot, H, D]
 *   b              [Ttot, H]
 *   A_log          [H]
 *   dt_bias        [H, D]
 *   state          [N, H, D, D]    S[i][j]: i = key channel, j = value channel
 *   conv_state     [N, 3, 3*H*D]   raw inputs of the 3 tokens before the
 *                                  sequence start, oldest first
 *   o              [Ttot, H, D]
 *   ogate          [Ttot, H, D]    output gate (pre-sigmoid), optional
 *   onw            [D]             o_norm weight, shared by the heads
 *
 * Output epilogue (optional): the layer's o_norm and sigmoid output gating
 * (same write-up: the KDA layer projects an output_gate, section "二", and ends
 * in o_norm plus sigmoid gating, section "三"; the Ling-3.0-flash-VL weight list
 * names o_norm and g_proj).  Read as an RMS norm over the head's D channels with
 * a per-channel weight, then the elementwise sigmoid gate:
 *   o[j] <- o[j] / sqrt(mean_j o^2 + oeps) * onw[j] * sigmoid(ogate[j]).
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <unistd.h>

#define KCONV 4

typedef struct {
    int64_t N, H, D;
    const int64_t *cu;
    const double *q, *k, *v, *conv_w, *alpha, *b, *A_log, *dt_bias;
    const double *state0, *conv0;
    double lower_bound, eps, scale;
    int beta2;              /* kda_allow_negative_eigenvalues: beta = 2 sigmoid(b) */
    const double *ogate, *onw;   /* output epilogue, or NULL */
    double oeps;
    double *o, *state1, *conv1;
    /* prologue-only outputs (any may be NULL) */
    double *qn, *kn, *vc, *g, *beta;
    int run_recurrence;
} job_t;

/* log(1 + e^x), the softplus of the gate formula, in an overflow-free form. */
static double softplus(double x) { return (x > 0 ? x : 0.0) + log1p(exp(-fabs(x))); }

static double sigmoid(double x) { return 1.0 / (1.0 + exp(-x)); }

static double silu(double x) { return x * sigmoid(x); }

/* Raw input of channel c (0 .. 3*H*D-1, blocks q | k | v) at token offset t
 * relative to the sequence start; t < 0 reads the conv history. */
static double raw_at(const job_t *J, int64_t n, int64_t t, int64_t c)
{
    int64_t HD = J->H * J->D;
    if (t < 0) {
        if (!J->conv0) return 0.0;
        return J->conv0[(n * 3 + (t + 3)) * 3 * HD + c];
    }
    int64_t row = J->cu[n] + t;
    int64_t blk = c / HD, cc = c % HD;
    const double *x = blk == 0 ? J->q : (blk == 1 ? J->k : J->v);
    return x[row * HD + cc];
}

/* One (sequence, head) pair: prologue then the token recurrence. */
static void run_pair(const job_t *J, int64_t n, int64_t h)
{
    const int64_t H = J->H, D = J->D, HD = H * D;
    const int64_t L = J->cu[n + 1] - J->cu[n];
    double *S = malloc(sizeof(double) * D * D);
    double *qt = malloc(sizeof(double) * D), *kt = malloc(sizeof(double) * D);
    double *vt = malloc(sizeof(double) * D), *gt = malloc(sizeof(double) * D);
    double *p = malloc(sizeof(double) * D), *dl = malloc(sizeof(double) * D);

    if (J->state0)
        memcpy(S, J->state0 + (n * H + h) * D * D, sizeof(double) * D * D);
    else
        memset(S, 0, sizeof(double) * D * D);

    const double A = exp(J->A_log[h]);

    for (int64_t t = 0; t < L; ++t) {
        const int64_t row = J->cu[n] + t;
        /* depthwise causal conv, kernel 4, no bias, then SiLU (q, k, v) */
        for (int blk = 0; blk < 3; ++blk) {
            double *dst = blk == 0 ? qt : (blk == 1 ? kt : vt);
            for (int64_t i = 0; i < D; ++i) {
                int64_t c = blk * HD + h * D + i;
                double acc = 0.0;
                for (int j = 0; j < KCONV; ++j)
                    acc += J->conv_w[c * KCONV + j] * raw_at(J, n, t - (KCONV - 1) + j, c);
                dst[i] = silu(acc);
            }
        }
        /* L2 normalisation of q and k over the head dimension */
        double sq = 0.0, sk = 0.0;
        for (int64_t i = 0; i < D; ++i) { sq += qt[i] * qt[i]; sk += kt[i] * kt[i]; }
        double rq = 1.0 / sqrt(sq + J->eps), rk = 1.0 / sqrt(sk + J->eps);
        for (int64_t i = 0; i < D; ++i) { qt[i] *= rq; kt[i] *= rk; }
        /* gate g = max(-exp(A_log) * softplus(alpha + dt_bias), lower_bound); beta = sigmoid(b),
         * doubled when negative eigenvalues are allowed (section "二": with
         * kda_allow_negative_eigenvalues off, beta is not multiplied by 2) */
        for (int64_t i = 0; i < D; ++i) {
            double x = J->alpha[(row * H + h) * D + i] + J->dt_bias[h * D + i];
            double g = -A * softplus(x);
            gt[i] = g < J->lower_bound ? J->lower_bound : g;
        }
        const double beta = (J->beta2 ? 2.0 : 1.0) * sigmoid(J->b[row * H + h]);

        if (J->qn) for (int64_t i = 0; i < D; ++i) J->qn[(row * H + h) * D + i] = qt[i];
        if (J->kn) for (int64_t i = 0; i < D; ++i) J->kn[(row * H + h) * D + i] = kt[i];
        if (J->vc) for (int64_t i = 0; i < D; ++i) J->vc[(row * H + h) * D + i] = vt[i];
        if (J->g) for (int64_t i = 0; i < D; ++i) J->g[(row * H + h) * D + i] = gt[i];
        if (J->beta) J->beta[row * H + h] = beta;
        if (!J->run_recurrence) continue;

        /* the delta-rule step: decay, predict, correct, write, read */
        for (int64_t i = 0; i < D; ++i) {
            double e = exp(gt[i]);
            for (int64_t j = 0; j < D; ++j) S[i * D + j] *= e;
        }
        for (int64_t j = 0; j < D; ++j) {
            double acc = 0.0;
            for (int64_t i = 0; i < D; ++i) acc += kt[i] * S[i * D + j];
            p[j] = acc;
        }
        for (int64_t j = 0; j < D; ++j) dl[j] = (vt[j] - p[j]) * beta;
        for (int64_t i = 0; i < D; ++i)
            for (int64_t j = 0; j < D; ++j) S[i * D + j] += kt[i] * dl[j];
        double *ot = J->o + (row * H + h) * D;
        for (int64_t j = 0; j < D; ++j) {
            double acc = 0.0;
            for (int64_t i = 0; i < D; ++i) acc += qt[i] * S[i * D + j];
            ot[j] = J->scale * acc;
        }
        if (J->ogate) {   /* o_norm (RMS over the head's D channels, weighted), then the gate */
            double ms = 0.0;
            for (int64_t j = 0; j < D; ++j) ms += ot[j] * ot[j];
            const double r = 1.0 / sqrt(ms / (double)D + J->oeps);
            for (int64_t j = 0; j < D; ++j)
                ot[j] = ot[j] * r * J->onw[j] * sigmoid(J->ogate[(row * H + h) * D + j]);
        }
    }

    if (J->run_recurrence && J->state1)
        memcpy(J->state1 + (n * H + h) * D * D, S, sizeof(double) * D * D);

    /* conv history after the sequence: raw inputs of its last 3 tokens */
    if (J->conv1) {
        for (int blk = 0; blk < 3; ++blk)
            for (int64_t i = 0; i < D; ++i) {
                int64_t c = blk * HD + h * D + i;
                for (int m = 0; m < 3; ++m)
                    J->conv1[(n * 3 + m) * 3 * HD + c] = raw_at(J, n, L - 3 + m, c);
            }
    }
    free(S); free(qt); free(kt); free(vt); free(gt); free(p); free(dl);
}

typedef struct { const job_t *J; int64_t next; pthread_mutex_t mu; } pool_t;

static void *worker(void *arg)
{
    pool_t *P = arg;
    const int64_t total = P->J->N * P->J->H;
    for (;;) {
        pthread_mutex_lock(&P->mu);
        int64_t task = P->next++;
        pthread_mutex_unlock(&P->mu);
        if (task >= total) break;
        run_pair(P->J, task / P->J->H, task % P->J->H);
    }
    return NULL;
}

static int run_all(const job_t *J, int nthreads)
{
    if (nthreads <= 0) nthreads = (int)sysconf(_SC_NPROCESSORS_ONLN);
    if (nthreads < 1) nthreads = 1;
    pool_t P = { J, 0 };
    pthread_mutex_init(&P.mu, NULL);
    pthread_t *th = malloc(sizeof(pthread_t) * nthreads);
    for (int i = 0; i < nthreads; ++i) pthread_create(&th[i], NULL, worker, &P);
    for (int i = 0; i < nthreads; ++i) pthread_join(th[i], NULL);
    free(th);
    pthread_mutex_destroy(&P.mu);
    return nthreads;
}

/* Full forward over N packed sequences.  state0 / conv0 may be NULL (zeros);
 * state1 / conv1 may be NULL (not wanted).  Returns the thread count used. */
int kda_oracle_forward(int64_t N, const int64_t *cu_seqlens, int64_t H, int64_t D,
                       const double *q, const double *k, const double *v,
                       const double *conv_w, const double *alpha, const double *b,
                       const double *A_log, const double *dt_bias,
                       const double *state0, const double *conv0,
                       double lower_bound, double eps, double scale, int beta2,
                       const double *ogate, const double *onw, double oeps,
                       double *o, double *state1, double *conv1, int nthreads)
{
    job_t J;
    memset(&J, 0, sizeof J);
    J.N = N; J.H = H; J.D = D; J.cu = cu_seqlens;
    J.q = q; J.k = k; J.v = v; J.conv_w = conv_w; J.alpha = alpha; J.b = b;
    J.A_log = A_log; J.dt_bias = dt_bias; J.state0 = state0; J.conv0 = conv0;
    J.lower_bound = lower_bound; J.eps = eps; J.scale = scale; J.beta2 = beta2;
    J.ogate = ogate; J.onw = onw; J.oeps = oeps;
    J.o = o; J.state1 = state1; J.conv1 = conv1;
    J.run_recurrence = 1;
    return run_all(&J, nthreads);
}

/* Prologue only: conv + SiLU, L2 norm, gate, beta.  Outputs [Ttot, H, D] and [Ttot, H]. */
int kda_oracle_prologue(int64_t N, const int64_t *cu_seqlens, int64_t H, int64_t D,
                        const double *q, const double *k, const double *v,
                        const double *conv_w, const double *alpha, const double *b,
                        const double *A_log, const double *dt_bias, const double *conv0,
                        double lower_bound, double eps, int beta2,
                        double *qn, double *kn, double *vc, double *g, double *beta,
                        int nthreads)
{
    job_t J;
    memset(&J, 0, sizeof J);
    J.N = N; J.H = H; J.D = D; J.cu = cu_seqlens;
    J.q = q; J.k = k; J.v = v; J.conv_w = conv_w; J.alpha = alpha; J.b = b;
    J.A_log = A_log; J.dt_bias = dt_bias; J.conv0 = conv0;
    J.lower_bound = lower_bound; J.eps = eps; J.scale = 1.0; J.beta2 = beta2;
    J.qn = qn; J.kn = kn; J.vc = vc; J.g = g; J.beta = beta;
    J.run_recurrence = 0;
    return run_all(&J, nthreads);
}

/* The recurrence alone, on already-prepared per-token q, k, v [Ttot, H, D],
 * g [Ttot, H, D] and beta [Ttot, H] (one sequence per (n), state [N, H, D, D]). */
int kda_oracle_recurrence(int64_t N, const int64_t *cu_seqlens, int64_t H, int64_t D,
                          const double *q, const double *k, const double *v,
                          const double *g, const double *beta, const double *state0,
                          double scale, double *o, double *state1)
{
    double *S = malloc(sizeof(double) * D * D);
    double *p = malloc(sizeof(double) * D), *dl = malloc(sizeof(double) * D);
    for (int64_t n = 0; n < N; ++n)
        for (int64_t h = 0; h < H; ++h) {
            if (state0) memcpy(S, state0 + (n * H + h) * D * D, sizeof(double) * D * D);
            else memset(S, 0, sizeof(double) * D * D);
            for (int64_t row = cu_seqlens[n]; row < cu_seqlens[n + 1]; ++row) {
                const double *qt = q + (row * H + h) * D, *kt = k + (row * H + h) * D;
                const double *vt = v + (row * H + h) * D, *gt = g + (row * H + h) * D;
                const double bt = beta[row * H + h];
                for (int64_t i = 0; i < D; ++i) {
                    double e = exp(gt[i]);
                    for (int64_t j = 0; j < D; ++j) S[i * D + j] *= e;
                }
                for (int64_t j = 0; j < D; ++j) {
                    double acc = 0.0;
                    for (int64_t i = 0; i < D; ++i) acc += kt[i] * S[i * D + j];
                    p[j] = acc;
                }
                for (int64_t j = 0; j < D; ++j) dl[j] = (vt[j] - p[j]) * bt;
                for (int64_t i = 0; i < D; ++i)
                    for (int64_t j = 0; j < D; ++j) S[i * D + j] += kt[i] * dl[j];
                for (int64_t j = 0; j < D; ++j) {
                    double acc = 0.0;
                    for (int64_t i = 0; i < D; ++i) acc += qt[i] * S[i * D + j];
                    o[(row * H + h) * D + j] = scale * acc;
                }
            }
            if (state1) memcpy(state1 + (n * H + h) * D * D, S, sizeof(double) * D * D);
        }
    free(S); free(p); free(dl);
    return 0;
}
