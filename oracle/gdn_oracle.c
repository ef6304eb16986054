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

/* ------------------------------------------------------------------------------------------ */
/* Backward pass of the recurrence: reverse-mode derivative of the loss through every token    */
/* ------------------------------------------------------------------------------------------ */
/*
 * The pages train their models ([HYB], [KIMI]) but give the layer for inference only; the
 * gradient here is the exact derivative of the recurrence above, taken by the chain rule one
 * token at a time in reverse, in the equation's own order.  Per token, with P = S_{t-1}:
 *
 *      x = P k,   A = P - beta x k^T,   S_t = alpha A + beta v k^T,   o_t = scale S_t q_t.
 *
 * Given G = dL/dS_t (the state gradient from later tokens plus this token's output):
 *      G     += scale do q^T                         (o_t = scale S_t q_t)
 *      dq    += scale S_t^T do
 *      dlog_alpha = alpha <G, A>,  dA = alpha G      (S_t = alpha A + ...)
 *      dbeta += v^T G k,  dv = beta G k,  dk += beta G^T v        (... + beta v k^T)
 *      dP = dA,  dbeta -= x^T dA k,  dx = -beta dA k,  dk -= beta dA^T x   (A = P - beta x k^T)
 *      dP += dx k^T,  dk += P^T dx                    (x = P k)
 *      dL/dS_{t-1} = dP.
 * The states S_0 .. S_T of a (batch, value head) are recomputed forward first and kept (the
 * tape).  The loss is L = sum <dO, o> + <dS_T, S_T>; dq and dk sum over the value heads that
 * share a key head, so one worker owns all value heads of a (batch, key head).
 */
typedef struct {
    const double *q, *k, *v, *log_alpha, *beta, *S0, *dO, *dST;
    double *dq, *dk, *dv, *dla, *dbeta, *dS0;
    long B, T;
    int Hk, Hv, dk_, dv_;
    double scale;
    int nthreads, tid;
} bwd_job;

static void bwd_one_head(const bwd_job *J, long b, int h, double *tape, double *G, double *dP,
                         double *x, double *dx, double *Gk, double *A)
{
    const int dk = J->dk_, dv = J->dv_, Hk = J->Hk, Hv = J->Hv;
    const int group = Hv / Hk, hk = h / group;         /* GQA: contiguous groups */
    const long T = J->T, SS = (long)dv * dk;
    const long st0 = ((long)b * Hv + h) * dk * dv;      /* this head's [dk][dv] state slot */
    /* forward: the tape of states, tape[t] = S_t (S_0 the initial state) */
    for (int a = 0; a < dv; ++a)
        for (int c = 0; c < dk; ++c)
            tape[(long)a * dk + c] = J->S0 ? J->S0[st0 + (long)c * dv + a] : 0.0;
    for (long t = 0; t < T; ++t) {
        const double *P = tape + t * SS;
        double *S = tape + (t + 1) * SS;
        const double *k = J->k + ((b * T + t) * Hk + hk) * (long)dk;
        const double *v = J->v + ((b * T + t) * Hv + h) * (long)dv;
        const double alpha = exp(J->log_alpha[(b * T + t) * Hv + h]);
        const double beta = J->beta[(b * T + t) * Hv + h];
        for (int a = 0; a < dv; ++a) {
            double acc = 0.0;
            for (int c = 0; c < dk; ++c) acc += P[(long)a * dk + c] * k[c];
            x[a] = acc;
        }
        for (int a = 0; a < dv; ++a)
            for (int c = 0; c < dk; ++c)
                S[(long)a * dk + c] = alpha * (P[(long)a * dk + c] - beta * x[a] * k[c]) +
                                      beta * v[a] * k[c];
    }
    /* reverse */
    for (int a = 0; a < dv; ++a)
        for (int c = 0; c < dk; ++c)
            G[(long)a * dk + c] = J->dST ? J->dST[st0 + (long)c * dv + a] : 0.0;
    for (long t = T - 1; t >= 0; --t) {
        const double *P = tape + t * SS, *S = tape + (t + 1) * SS;
        const long row = (b * T + t) * Hv + h;
        const double *q = J->q + ((b * T + t) * Hk + hk) * (long)dk;
        const double *k = J->k + ((b * T + t) * Hk + hk) * (long)dk;
        const double *v = J->v + row * (long)dv;
        const double *dO = J->dO + row * (long)dv;
        double *dq = J->dq + ((b * T + t) * Hk + hk) * (long)dk;
        double *dkk = J->dk + ((b * T + t) * Hk + hk) * (long)dk;
        double *dvv = J->dv + row * (long)dv;
        const double alpha = exp(J->log_alpha[row]);
        const double beta = J->beta[row];
        /* o_t = scale S_t q_t */
        for (int a = 0; a < dv; ++a)
            for (int c = 0; c < dk; ++c) G[(long)a * dk + c] += J->scale * dO[a] * q[c];
        for (int c = 0; c < dk; ++c) {
            double acc = 0.0;
            for (int a = 0; a < dv; ++a) acc += S[(long)a * dk + c] * dO[a];
            dq[c] += J->scale * acc;
        }
        /* x = P k and A = P - beta x k^T, recomputed from the tape */
        for (int a = 0; a < dv; ++a) {
            double acc = 0.0;
            for (int c = 0; c < dk; ++c) acc += P[(long)a * dk + c] * k[c];
            x[a] = acc;
        }
        for (int a = 0; a < dv; ++a)
            for (int c = 0; c < dk; ++c) A[(long)a * dk + c] = P[(long)a * dk + c] - beta * x[a] * k[c];
        /* S_t = alpha A + beta v k^T */
        double ga = 0.0;
        for (long i = 0; i < SS; ++i) ga += G[i] * A[i];
        J->dla[row] = alpha * ga;
        for (int a = 0; a < dv; ++a) {
            double acc = 0.0;
            for (int c = 0; c < dk; ++c) acc += G[(long)a * dk + c] * k[c];
            Gk[a] = acc;
        }
        double db = 0.0;
        for (int a = 0; a < dv; ++a) db += v[a] * Gk[a];
        for (int a = 0; a < dv; ++a) dvv[a] = beta * Gk[a];
        for (int c = 0; c < dk; ++c) {
            double acc = 0.0;
            for (int a = 0; a < dv; ++a) acc += G[(long)a * dk + c] * v[a];
            dkk[c] += beta * acc;
        }
        /* A = P - beta x k^T, with dA = alpha G */
        for (long i = 0; i < SS; ++i) dP[i] = alpha * G[i];
        for (int a = 0; a < dv; ++a) {
            double acc = 0.0;
            for (int c = 0; c < dk; ++c) acc += dP[(long)a * dk + c] * k[c];
            db -= x[a] * acc;
            dx[a] = -beta * acc;
        }
        for (int c = 0; c < dk; ++c) {
            double acc = 0.0;
            for (int a = 0; a < dv; ++a) acc += dP[(long)a * dk + c] * x[a];
            dkk[c] -= beta * acc;
        }
        J->dbeta[row] = db;
        /* x = P k */
        for (int c = 0; c < dk; ++c) {
            double acc = 0.0;
            for (int a = 0; a < dv; ++a) acc += P[(long)a * dk + c] * dx[a];
            dkk[c] += acc;
        }
        for (int a = 0; a < dv; ++a)
            for (int c = 0; c < dk; ++c) dP[(long)a * dk + c] += dx[a] * k[c];
        memcpy(G, dP, sizeof(double) * (size_t)SS);      /* dL/dS_{t-1} */
    }
    if (J->dS0)
        for (int a = 0; a < dv; ++a)
            for (int c = 0; c < dk; ++c)
                J->dS0[st0 + (long)c * dv + a] = G[(long)a * dk + c];
}

static void *bwd_worker(void *arg)
{
    const bwd_job *J = (const bwd_job *)arg;
    const long SS = (long)J->dk_ * J->dv_;
    double *tape = (double *)malloc(sizeof(double) * (size_t)SS * (size_t)(J->T + 1));
    double *G = (double *)malloc(sizeof(double) * (size_t)SS);
    double *dP = (double *)malloc(sizeof(double) * (size_t)SS);
    double *A = (double *)malloc(sizeof(double) * (size_t)SS);
    double *x = (double *)malloc(sizeof(double) * (size_t)J->dv_ * 3);
    if (!tape || !G || !dP || !A || !x) {
        free(tape); free(G); free(dP); free(A); free(x);
        return (void *)1;
    }
    const int G_ = J->Hv / J->Hk;
    const long groups = J->B * J->Hk;
    for (long p = J->tid; p < groups; p += J->nthreads) {
        const long b = p / J->Hk;
        const int hk = (int)(p % J->Hk);
        for (long t = 0; t < J->T; ++t) {           /* this worker owns dq, dk of (b, hk) */
            memset(J->dq + ((b * J->T + t) * J->Hk + hk) * (long)J->dk_, 0, sizeof(double) * J->dk_);
            memset(J->dk + ((b * J->T + t) * J->Hk + hk) * (long)J->dk_, 0, sizeof(double) * J->dk_);
        }
        for (int g = 0; g < G_; ++g)
            bwd_one_head(J, b, hk * G_ + g, tape, G, dP, x, x + J->dv_, x + 2 * J->dv_, A);
    }
    free(tape); free(G); free(dP); free(A); free(x);
    return NULL;
}

/*
 * Gradients of L = sum <dO, o> + <dS_T, S_T> with o, S_T from oracle_gated_delta on the same
 * inputs.  Shapes as there; dO: [B, T, Hv, dv]; dS_T (nullable = zero): [B, Hv, dk, dv] (S^T).
 * Outputs: dq, dk [B, T, Hk, dk] (summed over each key head's value heads), dv [B, T, Hv, dv],
 * dlog_alpha, dbeta [B, T, Hv], dS0 (nullable) [B, Hv, dk, dv] (S^T).  Memory: one tape of T + 1
 * states per host thread.  Returns 0, -1 on bad sizes, -2 if a tape could not be allocated.
 */
int oracle_gated_delta_bwd(const double *q, const double *k, const double *v,
                           const double *log_alpha, const double *beta, const double *S0,
                           const double *dO, const double *dS_T, double *dq, double *dk,
                           double *dv, double *dlog_alpha, double *dbeta, double *dS0, long B,
                           long T, int Hk, int Hv, int dk_, int dv_, double scale, int nthreads)
{
    if (B < 0 || T < 0 || Hk <= 0 || Hv <= 0 || dk_ <= 0 || dv_ <= 0 || Hv % Hk) return -1;
    if (nthreads < 1) nthreads = 1;
    if (nthreads > 1024) nthreads = 1024;
    bwd_job *jobs = (bwd_job *)calloc((size_t)nthreads, sizeof(bwd_job));
    pthread_t *th = (pthread_t *)calloc((size_t)nthreads, sizeof(pthread_t));
    void **ret = (void **)calloc((size_t)nthreads, sizeof(void *));
    for (int i = 0; i < nthreads; ++i) {
        bwd_job J = {q, k, v, log_alpha, beta, S0, dO, dS_T, dq, dk, dv, dlog_alpha, dbeta, dS0,
                     B, T, Hk, Hv, dk_, dv_, scale, nthreads, i};
        jobs[i] = J;
    }
    char *started = (char *)calloc((size_t)nthreads, 1);
    for (int i = 1; i < nthreads; ++i)
        started[i] = pthread_create(&th[i], NULL, bwd_worker, &jobs[i]) == 0;
    ret[0] = bwd_worker(&jobs[0]);
    for (int i = 1; i < nthreads; ++i) {
        if (started[i]) pthread_join(th[i], &ret[i]);
        else ret[i] = bwd_worker(&jobs[i]);
    }
    int rc = 0;
    for (int i = 0; i < nthreads; ++i)
        if (ret[i]) rc = -2;
    free(started); free(jobs); free(th); free(ret);
    return rc;
}

/* ------------------------------------------------------------------------------------------ */
/* Backward of the layer's other pieces: chain rule through each forward definition above      */
/* ------------------------------------------------------------------------------------------ */

/*
 * y = SiLU(conv(x)) as oracle_causal_conv_silu; given dy, with pre the convolution and
 * SiLU'(p) = sigmoid(p) (1 + p (1 - sigmoid(p))):
 *   dpre = dy SiLU'(pre);  dx[s] = sum_j w[j] dpre[s + 3 - j];  dw[c][j] = sum_t dpre[t] x[t - 3 + j]
 * (tokens outside 0 .. T - 1 contribute nothing).  dw is summed over every batch and token.
 */
void oracle_causal_conv_silu_bwd(const double *x, const double *w, const double *dy, double *dx,
                                 double *dw, long B, long T, long C)
{
    for (long i = 0; i < B * T * C; ++i) dx[i] = 0.0;
    for (long i = 0; i < C * 4; ++i) dw[i] = 0.0;
    for (long b = 0; b < B; ++b)
        for (long t = 0; t < T; ++t)
            for (long c = 0; c < C; ++c) {
                double pre = 0.0;
                for (int j = 0; j < 4; ++j) {
                    const long u = t - 3 + j;          /* the tap's token */
                    if (u >= 0) pre += w[c * 4 + j] * x[(b * T + u) * C + c];
                }
                const double sg = sigmoid(pre);
                const double dpre = dy[(b * T + t) * C + c] * sg * (1.0 + pre * (1.0 - sg));
                for (int j = 0; j < 4; ++j) {
                    const long u = t - 3 + j;          /* the tap's token */
                    if (u < 0) continue;
                    dx[(b * T + u) * C + c] += w[c * 4 + j] * dpre;
                    dw[c * 4 + j] += x[(b * T + u) * C + c] * dpre;
                }
            }
}

/* y = x / sqrt(sum x^2 + eps) per row of d:  dx = dy / n - x (x . dy) / n^3,  n = sqrt(ss + eps). */
void oracle_l2_normalize_bwd(const double *x, const double *dy, double *dx, long rows, int d,
                             double eps)
{
    for (long r = 0; r < rows; ++r) {
        double ss = 0.0, xd = 0.0;
        for (int i = 0; i < d; ++i) {
            ss += x[r * d + i] * x[r * d + i];
            xd += x[r * d + i] * dy[r * d + i];
        }
        const double n = sqrt(ss + eps);
        for (int i = 0; i < d; ++i) dx[r * d + i] = dy[r * d + i] / n - x[r * d + i] * xd / (n * n * n);
    }
}

/*
 * y_i = o_i inv w_i SiLU(z_i), inv = 1 / sqrt(mean(o^2) + eps), per row of d; given dy:
 *   dz_i = dy_i o_i inv w_i SiLU'(z_i);  dw_i += dy_i o_i inv SiLU(z_i)  (summed over rows);
 *   with g_i = dy_i w_i SiLU(z_i):  do_i = inv g_i - o_i inv^3 (sum_j g_j o_j) / d.
 */
void oracle_gated_rmsnorm_bwd(const double *o, const double *z, const double *w,
                              const double *dy, double *dout, double *dz, double *dw, long rows,
                              int d, double eps)
{
    for (int i = 0; i < d; ++i) dw[i] = 0.0;
    for (long r = 0; r < rows; ++r) {
        double ss = 0.0, go = 0.0;
        for (int i = 0; i < d; ++i) ss += o[r * d + i] * o[r * d + i];
        const double inv = 1.0 / sqrt(ss / (double)d + eps);   /* 1 / rms */
        for (int i = 0; i < d; ++i) {
            const double zz = z[r * d + i], sg = sigmoid(zz);
            const double g = dy[r * d + i] * w[i] * (zz * sg);
            go += g * o[r * d + i];
            dz[r * d + i] = dy[r * d + i] * o[r * d + i] * inv * w[i] * sg * (1.0 + zz * (1.0 - sg));
            dw[i] += dy[r * d + i] * o[r * d + i] * inv * (zz * sg);
        }
        for (int i = 0; i < d; ++i) {
            const double g = dy[r * d + i] * w[i] * (z[r * d + i] * sigmoid(z[r * d + i]));
            dout[r * d + i] = inv * g - o[r * d + i] * inv * inv * inv * go / d;
        }
    }
}

/* beta = sigmoid(b), log alpha = -softplus(-a):  db = dbeta beta (1 - beta),  da = dlog_alpha
 * sigmoid(-a).  ba, dba: [rows, 2 Hv] (b values then a values). */
void oracle_gates_bwd(const double *ba, const double *dlog_alpha, const double *dbeta, double *dba,
                      long rows, int Hv)
{
    for (long r = 0; r < rows; ++r)
        for (int h = 0; h < Hv; ++h) {
            const double b = ba[r * 2 * Hv + h], a = ba[r * 2 * Hv + Hv + h];
            const double sb = sigmoid(b);
            dba[r * 2 * Hv + h] = dbeta[r * Hv + h] * sb * (1.0 - sb);
            dba[r * 2 * Hv + Hv + h] = dlog_alpha[r * Hv + h] * sigmoid(-a);
        }
}
