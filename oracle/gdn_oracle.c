/*
 * Gated delta rule: plain fp64 CPU oracle.  TEST INFRASTRUCTURE ONLY.
 *
 * Only the test suite, the smoke check and the bench's CPU-baseline leg may call this code.  It
 * shares nothing with the CUDA library: no header, helper, table or kernel.  It is slow on
 * purpose: every function below is the plain definition, token by token, in double precision.
 *
 * Sources (page titles as printed at each page header; sections in parentheses):
 *   [HYB]  "L'attention hybride" (mkdocs.reaper.mx, Qwen3.8-27B architecture chapter):
 *          (Les 48 couches Gated DeltaNet) dims 16 key / 48 value heads of 128, conv kernel 4,
 *          swish output gate, fp32 state; (La récurrence) the symbol table: alpha_t in ]0,1[ a
 *          global decay that fades the whole state, beta_t in ]0,1[ a write rate that replaces
 *          the association bound to k_t, I the 128x128 identity; (L'état, en mémoire) the state
 *          has a constant size whatever the length; (Le décompte) conv 4 taps per channel and no
 *          bias, one 128-wide normalisation gain.
 *   [BRK]  "Les briques d'un réseau de neurones" (same site, Kimi K3 foundations): (2. Les
 *          fonctions d'activation) sigmoid and SiLU = x * sigmoid(x); (4. Les normalisations)
 *          RMSNorm with eps = 1e-5 and a per-coordinate gain.
 *   [KIMI] "Chapitre 16 - Assembler un système de type Kimi K3" (cours.spawnkit.ai, session 21):
 *          (16.2) prefill processes blocks and hands the state from block to block; (16.3) a
 *          decode step reads the fixed state, computes the output and updates the state.
 *
 * The equation of the recurrence was lost when the page was extracted; its symbols survive.
 * This oracle uses the gated delta rule written with exactly those symbols:
 *
 *      S_t = alpha_t * S_{t-1} (I - beta_t k_t k_t^T) + beta_t v_t k_t^T,     o_t = scale * S_t q_t
 *
 * with S_t of shape d_v x d_k for each value head.  Value head h reads key/query head
 * h / (Hv / Hk) (contiguous groups of Hv/Hk value heads per key head, [HYB] "La dissymétrie").
 *
 * Memory layout of the state at this interface: M = S^T, i.e. state[b][h][i][j] = S[j][i] with i
 * over d_k and j over d_v (d_v contiguous).  Inside the recurrence the oracle keeps S in the
 * orientation of the equation above and transposes only when reading S0 and writing S_T.
 *
 * Pins that tie this code to the pages and to mathematics, not to itself, live in the test suite:
 * closed forms for alpha = 1 / beta = 0, exact retrieval with orthonormal keys, the overwrite of a
 * repeated key, brute-force products of explicit d_k x d_k transition matrices, the Frobenius-norm
 * bound, a library convolution, and unit norms after the L2 / RMS normalisations.
 */
#include <math.h>
#include <pthread.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------------------------------ */
/* Gated delta recurrence, one (batch, value head) pair                                        */
/* ------------------------------------------------------------------------------------------ */

typedef struct {
    const double *q, *k, *v, *log_alpha, *beta, *S0;
    double *o, *S_T;
    long B, T;
    int Hk, Hv, dk, dv;
    double scale;
    int nthreads, tid;
} recur_job;

static void recur_one_head(const recur_job *J, long b, int h, double *S, double *Sk)
{
    const int dk = J->dk, dv = J->dv, Hk = J->Hk, Hv = J->Hv;
    const int hk = h / (Hv / Hk);                      /* GQA: contiguous groups */
    /* S0 (stored transposed) or the zero state of a fresh request ([KIMI] 16.1: reset per request) */
    for (int a = 0; a < dv; ++a)
        for (int c = 0; c < dk; ++c)
            S[(long)a * dk + c] = J->S0 ? J->S0[(((long)b * Hv + h) * dk + c) * dv + a] : 0.0;

    for (long t = 0; t < J->T; ++t) {
        const double *q = J->q + ((b * J->T + t) * Hk + hk) * (long)dk;
        const double *k = J->k + ((b * J->T + t) * Hk + hk) * (long)dk;
        const double *v = J->v + ((b * J->T + t) * Hv + h) * (long)dv;
        const double alpha = exp(J->log_alpha[(b * J->T + t) * Hv + h]);
        const double beta = J->beta[(b * J->T + t) * Hv + h];

        /* S (I - beta k k^T) = S - beta (S k) k^T */
        for (int a = 0; a < dv; ++a) {
            double acc = 0.0;
            for (int c = 0; c < dk; ++c) acc += S[(long)a * dk + c] * k[c];
            Sk[a] = acc;
        }
        /* S_t = alpha * [S - beta (S k) k^T] + beta v k^T */
        for (int a = 0; a < dv; ++a)
            for (int c = 0; c < dk; ++c) {
                const double x = S[(long)a * dk + c] - beta * Sk[a] * k[c];
                S[(long)a * dk + c] = alpha * x + beta * v[a] * k[c];
            }
        /* o_t = scale * S_t q_t  (the output reads the state after this token's update) */
        double *o = J->o + ((b * J->T + t) * Hv + h) * (long)dv;
        for (int a = 0; a < dv; ++a) {
            double acc = 0.0;
            for (int c = 0; c < dk; ++c) acc += S[(long)a * dk + c] * q[c];
            o[a] = J->scale * acc;
        }
    }
    if (J->S_T)
        for (int a = 0; a < dv; ++a)
            for (int c = 0; c < dk; ++c)
                J->S_T[(((long)b * Hv + h) * dk + c) * dv + a] = S[(long)a * dk + c];
}

static void *recur_worker(void *arg)
{
    const recur_job *J = (const recur_job *)arg;
    double *S = (double *)malloc(sizeof(double) * (size_t)J->dk * J->dv);
    double *Sk = (double *)malloc(sizeof(double) * (size_t)J->dv);
    const long pairs = J->B * J->Hv;
    for (long p = J->tid; p < pairs; p += J->nthreads)
        recur_one_head(J, p / J->Hv, (int)(p % J->Hv), S, Sk);
    free(S);
    free(Sk);
    return NULL;
}

/*
 * q, k: [B, T, Hk, dk]; v, o: [B, T, Hv, dv]; log_alpha, beta: [B, T, Hv];
 * S0 (nullable = zero state), S_T (nullable): [B, Hv, dk, dv] holding S^T.
 * The (b, h) recurrences are independent; they are spread over `nthreads` host threads and each
 * token loop stays sequential.  Returns 0, or -1 on bad sizes.
 */
int oracle_gated_delta(const double *q, const double *k, const double *v,
                       const double *log_alpha, const double *beta, const double *S0,
                       double *o, double *S_T, long B, long T, int Hk, int Hv, int dk, int dv,
                       double scale, int nthreads)
{
    if (B < 0 || T < 0 || Hk <= 0 || Hv <= 0 || dk <= 0 || dv <= 0 || Hv % Hk) return -1;
    if (nthreads < 1) nthreads = 1;
    if (nthreads > 1024) nthreads = 1024;
    recur_job *jobs = (recur_job *)calloc((size_t)nthreads, sizeof(recur_job));
    pthread_t *th = (pthread_t *)calloc((size_t)nthreads, sizeof(pthread_t));
    for (int i = 0; i < nthreads; ++i) {
        recur_job J = {q, k, v, log_alpha, beta, S0, o, S_T, B, T, Hk, Hv, dk, dv,
                       scale, nthreads, i};
        jobs[i] = J;
    }
    char *started = (char *)calloc((size_t)nthreads, 1);
    for (int i = 1; i < nthreads; ++i)
        started[i] = pthread_create(&th[i], NULL, recur_worker, &jobs[i]) == 0;
    recur_worker(&jobs[0]);
    for (int i = 1; i < nthreads; ++i) {
        if (started[i]) pthread_join(th[i], NULL);
        else recur_worker(&jobs[i]);            /* a thread that failed to start: run its share */
    }
    free(started);
    free(jobs);
    free(th);
    return 0;
}

/* ------------------------------------------------------------------------------------------ */
/* Prologue pieces: causal depthwise conv (4 taps, no bias) then SiLU; L2 normalisation       */
/* ------------------------------------------------------------------------------------------ */

static double sigmoid(double x) { return 1.0 / (1.0 + exp(-x)); }     /* [BRK] 2. */

/*
 * x, y: [B, T, C]; w: [C, 4], tap j multiplies x[t - 3 + j] (tap 3 is the current token), and
 * positions before t = 0 hold zeros (a fresh request).  y = SiLU(conv(x)).  ([HYB] Le décompte:
 * 4 weights per channel and no bias; SiLU is the swish of [BRK] 2.)
 */
void oracle_causal_conv_silu(const double *x, const double *w, double *y, long B, long T, long C)
{
    for (long b = 0; b < B; ++b)
        for (long t = 0; t < T; ++t)
            for (long c = 0; c < C; ++c) {
                double acc = 0.0;
                for (int j = 0; j < 4; ++j) {
                    const long s = t - 3 + j;
                    if (s >= 0) acc += w[c * 4 + j] * x[(b * T + s) * C + c];
                }
                y[(b * T + t) * C + c] = acc * sigmoid(acc);
            }
}

/* x, y: [rows, d]; y = x / sqrt(sum x^2 + eps). */
void oracle_l2_normalize(const double *x, double *y, long rows, int d, double eps)
{
    for (long r = 0; r < rows; ++r) {
        double ss = 0.0;
        for (int i = 0; i < d; ++i) ss += x[r * d + i] * x[r * d + i];
        const double inv = 1.0 / sqrt(ss + eps);
        for (int i = 0; i < d; ++i) y[r * d + i] = x[r * d + i] * inv;
    }
}

/*
 * Output gate: y = RMSNorm(o) * w (.) SiLU(z) per (token, head) row of length d
 * ([HYB] output_gate_type swish, one 128-wide gain; [BRK] 4. RMSNorm).
 * RMSNorm(o) = o / sqrt(mean(o^2) + eps).  o, z, y: [rows, d]; w: [d].
 */
void oracle_gated_rmsnorm(const double *o, const double *z, const double *w, double *y,
                          long rows, int d, double eps)
{
    for (long r = 0; r < rows; ++r) {
        double ss = 0.0;
        for (int i = 0; i < d; ++i) ss += o[r * d + i] * o[r * d + i];
        const double inv = 1.0 / sqrt(ss / d + eps);
        for (int i = 0; i < d; ++i) {
            const double zz = z[r * d + i];
            y[r * d + i] = (o[r * d + i] * inv) * w[i] * (zz * sigmoid(zz));
        }
    }
}

/*
 * Gates of one (token, value head) from the in_proj_ba outputs ([HYB] Le décompte: in_proj_ba
 * makes one beta and one alpha per value head, 2 x 48 outputs, and no other gate parameter is
 * counted; [BRK] 2.: the sigmoid is the gate that squashes into (0, 1), softplus is
 * log(1 + e^x)).  Reading: beta = sigmoid(b), alpha = sigmoid(a), so log alpha = -softplus(-a).
 * ba: [rows, 2 * Hv], the Hv b values then the Hv a values; log_alpha, beta: [rows, Hv].
 */
static double softplus(double x) { return x > 0.0 ? x + log1p(exp(-x)) : log1p(exp(x)); }

void oracle_gates(const double *ba, double *log_alpha, double *beta, long rows, int Hv)
{
    for (long r = 0; r < rows; ++r)
        for (int h = 0; h < Hv; ++h) {
            const double b = ba[r * 2 * Hv + h], a = ba[r * 2 * Hv + Hv + h];
            beta[r * Hv + h] = sigmoid(b);
            log_alpha[r * Hv + h] = -softplus(-a);
        }
}
