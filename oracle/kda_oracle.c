/*
 * KDA (Kimi Delta Attention) forward -- CPU oracle, fp64, one token at a time.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the
 * benchmark's CPU-baseline leg may load this library.  The product path (the
 * CUDA library under kda_linear_attention_fwd_b200/) never calls it, shares no
 * code with it, and must fail loudly when its own extension is missing.
 *
 * What it computes is the plain definition of the layer, written out token by
 * token with no chunking, blocking or reordering:
 *
 *   for each (sequence n, head h), S <- S0 (or 0), then for t = 1..L:
 *     1. forget        S <- Diag(exp(g_t)) S
 *     2. delta write   u  = beta_t (v_t - S^T k_t);   S <- S + k_t u^T
 *     3. read          o_t = S^T (scale * q_t)
 *     4. output gate   y_t = gate_t (.) o_t           (gate == NULL: y_t = o_t)
 *
 * Sources (Kimi K3 report explainer, affta.cn, section "第一关：KDA 解决算得动"):
 *   - the per-token order "control signals -> forget old state -> corrective
 *     write with an update strength -> read the new state -> output gate";
 *   - the channel-wise forget gate: each state direction decays at its own
 *     rate, so the forget step scales row i of S (key channel i) by alpha_t[i];
 *   - the delta rule: read the state with the current key, compare with the
 *     new value, write only the error, scaled by the update strength beta_t;
 *   - the full-rank output gate: one gate value per output channel.
 * Step 2 reads the state after step 1 and step 3 reads it after step 2, as
 * the order above puts them.
 *
 * Optional pieces:
 *   - qk_l2norm: q and k are divided by sqrt(sum x^2 + 1e-6) before use (the
 *     "Query and Key normalisation" of the FlashKDA section; the epsilon is
 *     this library's choice, the pages give none);
 *   - erase = 0 drops the "- S^T k_t" term of step 2 (plain additive write).
 *     It exists only so that tests can reduce the layer to textbook linear
 *     attention; the CUDA library has no such switch.
 *
 * Inputs are fp32 arrays (bf16 values are exactly representable in fp32) and
 * are widened to fp64 exactly.  All arithmetic is fp64.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <unistd.h>

typedef struct {
    int L, dk, dv;
    const float *q, *k, *v, *g, *beta, *gate; /* token 0 of this (n, h) */
    long sqk, sv, sb;                         /* token strides (elements) */
    double scale;
    int qk_l2norm, erase;
    double *S;      /* [dk][dv] state: holds S0 on entry, final S on exit */
    double *y;      /* token 0 of the output for this (n, h), or NULL */
    long sy;        /* token stride of y */
} head_job;

static void run_head(const head_job *J, double *qt, double *kt, double *u)
{
    const int dk = J->dk, dv = J->dv;
    double *S = J->S;
    for (int t = 0; t < J->L; ++t) {
        const float *qs = J->q + (long)t * J->sqk;
        const float *ks = J->k + (long)t * J->sqk;
        const float *gs = J->g + (long)t * J->sqk;
        const float *vs = J->v + (long)t * J->sv;
        const double beta = (double)J->beta[(long)t * J->sb];
        for (int i = 0; i < dk; ++i) { qt[i] = (double)qs[i]; kt[i] = (double)ks[i]; }
        if (J->qk_l2norm) {
            double nq = 0.0, nk = 0.0;
            for (int i = 0; i < dk; ++i) { nq += qt[i] * qt[i]; nk += kt[i] * kt[i]; }
            nq = 1.0 / sqrt(nq + 1e-6);
            nk = 1.0 / sqrt(nk + 1e-6);
            for (int i = 0; i < dk; ++i) { qt[i] *= nq; kt[i] *= nk; }
        }
        for (int i = 0; i < dk; ++i) qt[i] *= J->scale;

        /* 1. forget: row i of S decays by alpha_t[i] = exp(g_t[i]) */
        for (int i = 0; i < dk; ++i) {
            const double a = exp((double)gs[i]);
            double *row = S + (long)i * dv;
            for (int j = 0; j < dv; ++j) row[j] *= a;
        }
        /* 2. delta write: u = beta (v - S^T k), S += k u^T */
        for (int j = 0; j < dv; ++j) u[j] = 0.0;
        if (J->erase) {
            for (int i = 0; i < dk; ++i) {
                const double ki = kt[i];
                const double *row = S + (long)i * dv;
                for (int j = 0; j < dv; ++j) u[j] += row[j] * ki;
            }
        }
        for (int j = 0; j < dv; ++j) u[j] = beta * ((double)vs[j] - u[j]);
        for (int i = 0; i < dk; ++i) {
            const double ki = kt[i];
            double *row = S + (long)i * dv;
            for (int j = 0; j < dv; ++j) row[j] += ki * u[j];
        }
        /* 3. read with the (scaled) query, 4. output gate */
        if (J->y) {
            double *yt = J->y + (long)t * J->sy;
            for (int j = 0; j < dv; ++j) yt[j] = 0.0;
            for (int i = 0; i < dk; ++i) {
                const double qi = qt[i];
                const double *row = S + (long)i * dv;
                for (int j = 0; j < dv; ++j) yt[j] += row[j] * qi;
            }
            if (J->gate) {
                const float *gt = J->gate + (long)t * J->sv;
                for (int j = 0; j < dv; ++j) yt[j] *= (double)gt[j];
            }
        }
    }
}

/* ---- a minimal thread pool over independent (n, h) jobs ---------------- */

typedef struct {
    head_job *jobs;
    int n_jobs;
    int next;
    pthread_mutex_t mu;
    int dk, dv;
} pool;

static void *worker(void *arg)
{
    pool *P = (pool *)arg;
    double *scratch = (double *)malloc(sizeof(double) * (size_t)(2 * P->dk + P->dv));
    if (!scratch) return NULL;
    for (;;) {
        pthread_mutex_lock(&P->mu);
        const int j = P->next++;
        pthread_mutex_unlock(&P->mu);
        if (j >= P->n_jobs) break;
        run_head(&P->jobs[j], scratch, scratch + P->dk, scratch + 2 * P->dk);
    }
    free(scratch);
    return NULL;
}

static int run_pool(head_job *jobs, int n_jobs, int dk, int dv, int n_threads)
{
    if (n_jobs <= 0) return 0;
    if (n_threads <= 0) n_threads = (int)sysconf(_SC_NPROCESSORS_ONLN);
    if (n_threads < 1) n_threads = 1;
    if (n_threads > n_jobs) n_threads = n_jobs;
    pool P;
    P.jobs = jobs; P.n_jobs = n_jobs; P.next = 0; P.dk = dk; P.dv = dv;
    pthread_mutex_init(&P.mu, NULL);
    pthread_t *th = (pthread_t *)malloc(sizeof(pthread_t) * (size_t)n_threads);
    if (!th) return -1;
    int started = 0;
    for (int i = 0; i < n_threads; ++i)
        if (pthread_create(&th[i], NULL, worker, &P) == 0) ++started;
    if (started == 0) worker(&P);
    for (int i = 0; i < started; ++i) pthread_join(th[i], NULL);
    free(th);
    pthread_mutex_destroy(&P.mu);
    return n_threads;
}

/*
 * Packed variable-length layout: q, k, g [T][H][dk]; v, gate, y [T][H][dv];
 * beta [T][H]; sequences delimited by cu_seqlens[0..N].  state [N][H][dk][dv]
 * holds the initial state on entry (zeros for "no initial state") and the
 * final state on exit.  mask [N*H] (may be NULL = all) selects which (n, h)
 * are computed; the others are left untouched in y and state.
 * Returns the number of threads used, or -1.
 */
int kda_oracle_varlen(const float *q, const float *k, const float *v, const float *g,
                      const float *beta, const float *gate, const int32_t *cu_seqlens,
                      int num_seqs, int H, int dk, int dv, double scale, int qk_l2norm,
                      int erase, double *state, double *y, const uint8_t *mask, int n_threads)
{
    head_job *jobs = (head_job *)calloc((size_t)num_seqs * (size_t)H + 1, sizeof(head_job));
    if (!jobs) return -1;
    int n = 0;
    for (int s = 0; s < num_seqs; ++s) {
        const long t0 = cu_seqlens[s];
        const int L = cu_seqlens[s + 1] - cu_seqlens[s];
        for (int h = 0; h < H; ++h) {
            if (mask && !mask[(long)s * H + h]) continue;
            head_job *J = &jobs[n++];
            J->L = L; J->dk = dk; J->dv = dv;
            J->q = q + (t0 * H + h) * dk;
            J->k = k + (t0 * H + h) * dk;
            J->g = g + (t0 * H + h) * dk;
            J->v = v + (t0 * H + h) * dv;
            J->gate = gate ? gate + (t0 * H + h) * dv : NULL;
            J->beta = beta + t0 * H + h;
            J->sqk = (long)H * dk; J->sv = (long)H * dv; J->sb = H;
            J->scale = scale; J->qk_l2norm = qk_l2norm; J->erase = erase;
            J->S = state + ((long)s * H + h) * (long)dk * dv;
            J->y = y ? y + (t0 * H + h) * dv : NULL;
            J->sy = (long)H * dv;
        }
    }
    const int used = run_pool(jobs, n, dk, dv, n_threads);
    free(jobs);
    return used;
}

/*
 * Step-major layout of a run of single-token steps (the decode case): q, k, g
 * [steps][N][H][dk]; v, gate, y [steps][N][H][dv]; beta [steps][N][H].  Each
 * (n, h) is one sequence of `steps` tokens, so this is the same recurrence as
 * above with a different token stride.  state [N][H][dk][dv] in/out.
 */
int kda_oracle_steps(const float *q, const float *k, const float *v, const float *g,
                     const float *beta, const float *gate, int steps, int num_seqs, int H,
                     int dk, int dv, double scale, int qk_l2norm, int erase, double *state,
                     double *y, const uint8_t *mask, int n_threads)
{
    head_job *jobs = (head_job *)calloc((size_t)num_seqs * (size_t)H + 1, sizeof(head_job));
    if (!jobs) return -1;
    int n = 0;
    const long NH = (long)num_seqs * H;
    for (long w = 0; w < NH; ++w) {
        if (mask && !mask[w]) continue;
        head_job *J = &jobs[n++];
        J->L = steps; J->dk = dk; J->dv = dv;
        J->q = q + w * dk; J->k = k + w * dk; J->g = g + w * dk;
        J->v = v + w * dv;
        J->gate = gate ? gate + w * dv : NULL;
        J->beta = beta + w;
        J->sqk = NH * dk; J->sv = NH * dv; J->sb = NH;
        J->scale = scale; J->qk_l2norm = qk_l2norm; J->erase = erase;
        J->S = state + w * (long)dk * dv;
        J->y = y ? y + w * dv : NULL;
        J->sy = NH * dv;
    }
    const int used = run_pool(jobs, n, dk, dv, n_threads);
    free(jobs);
    return used;
}
