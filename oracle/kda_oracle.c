/*
 * KDA / gated-DeltaNet CPU oracle -- TEST INFRASTRUCTURE ONLY.
 *
 * Only the test suite, the smoke check and the benchmark's CPU-baseline leg
 * may load this library.  The CUDA product path never links or calls it, and
 * the two share no code.
 *
 * What it computes: the token-by-token state recurrence of the KDA layer in
 * IEEE fp64, exactly as the pages state it, one (sequence, head) at a time.
 *
 *   "Hybrid Linear Attention Architecture: Making LLM Training and Inference
 *    More Efficient", section 3.3 (KDA update: per-channel decay first, then
 *    the delta rule's erase and write) and section 3.2 (beta -> 0 leaves the
 *    state untouched, beta -> 1 overwrites);
 *   "Hybrid Linear Attention Architecture: Technical Deep Dive ...",
 *    section 3.3 (the KDA formula);
 *   "Linear Attention Architecture Deep Dive ...", section 3.5;
 *   "Demystifying Hybrid LLM Architectures ...", section 2.3 (the inference
 *    loop reads the output from the state AFTER this token's write).
 *
 * Orientation (the pages mix conventions and say so): the state S is
 * d_k x d_v, the transition acts on the d_k side, the write is
 * beta_t * k_t * v_t^T and the read-out is o_t = S_t^T q_t.  Written out:
 *
 *   Shat  = Diag(alpha_t) S_{t-1},           alpha_t = exp(log_alpha_t)
 *   r     = Shat^T k_t                       (value the key currently retrieves)
 *   u     = beta_t (v_t - r)                 (erase on)  |  beta_t v_t  (erase off)
 *   S_t   = Shat + k_t u^T
 *   o_t   = S_t^T q_t
 *
 * which is S_t = (I - beta_t k_t k_t^T) Diag(alpha_t) S_{t-1} + beta_t k_t v_t^T.
 * "erase off" drops the -beta k k^T term (the gated-linear-attention special
 * case, and with alpha = 1 the plain accumulate-only linear attention of
 * section 3.1 of the first page).
 *
 * Sequences are packed token-major: q,k [T_total, H, dk], v [T_total, H, dv],
 * beta [T_total, H], log_alpha [T_total, H, dk], o [T_total, H, dv];
 * sequence n owns tokens cu[n] .. cu[n+1]-1; states are [N, H, dk, dv].
 * A NULL initial state means zeros.  Work is split over (sequence, head)
 * pairs across `nthreads` POSIX threads (each pair is independent).
 *
 * KDA_ORACLE_MUTANT (never defined in a normal build) plants one deliberate
 * mistake per value; the oracle's own tests compile those variants to show
 * that each plausible slip fails at least one independent pin.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

typedef struct {
    const double *q, *k, *v, *beta, *log_alpha, *s0;
    const int64_t *cu;
    int N, H, dk, dv, erase;
    double *o, *sT;
    int next;             /* next (sequence, head) pair to take */
    pthread_mutex_t lock;
} job_t;

static void run_pair(const job_t *J, int n, int h, double *S, double *u)
{
    const int H = J->H, dk = J->dk, dv = J->dv;
    const size_t SS = (size_t)dk * dv;
    if (J->s0)
        memcpy(S, J->s0 + ((size_t)n * H + h) * SS, SS * sizeof(double));
    else
        memset(S, 0, SS * sizeof(double));

    for (int64_t t = J->cu[n]; t < J->cu[n + 1]; ++t) {
        const double *qt = J->q + ((size_t)t * H + h) * dk;
        const double *kt = J->k + ((size_t)t * H + h) * dk;
        const double *vt = J->v + ((size_t)t * H + h) * dv;
        const double *gt = J->log_alpha + ((size_t)t * H + h) * dk;
        const double bt = J->beta[(size_t)t * H + h];

#if defined(KDA_ORACLE_MUTANT) && KDA_ORACLE_MUTANT == 3
        /* planted mistake 3: retrieve from the state before the decay */
        for (int j = 0; j < dv; ++j) u[j] = 0.0;
        for (int i = 0; i < dk; ++i)
            for (int j = 0; j < dv; ++j) u[j] += kt[i] * S[(size_t)i * dv + j];
#endif
#if !(defined(KDA_ORACLE_MUTANT) && KDA_ORACLE_MUTANT == 2)
        /* decay each key channel (row of S) */
        for (int i = 0; i < dk; ++i) {
            const double a = exp(gt[i]);
            double *row = S + (size_t)i * dv;
            for (int j = 0; j < dv; ++j) row[j] *= a;
        }
#endif
#if !(defined(KDA_ORACLE_MUTANT) && KDA_ORACLE_MUTANT == 3)
        /* retrieve r = Shat^T k, form the write vector u */
        for (int j = 0; j < dv; ++j) u[j] = 0.0;
        if (J->erase) {
            for (int i = 0; i < dk; ++i) {
                const double *row = S + (size_t)i * dv;
                for (int j = 0; j < dv; ++j) u[j] += kt[i] * row[j];
            }
        }
#endif
#if defined(KDA_ORACLE_MUTANT) && KDA_ORACLE_MUTANT == 3
        if (!J->erase) for (int j = 0; j < dv; ++j) u[j] = 0.0;
#endif
#if defined(KDA_ORACLE_MUTANT) && KDA_ORACLE_MUTANT == 4
        for (int j = 0; j < dv; ++j) u[j] = bt * (vt[j] + u[j]);   /* planted: wrong sign */
#elif defined(KDA_ORACLE_MUTANT) && KDA_ORACLE_MUTANT == 5
        for (int j = 0; j < dv; ++j) u[j] = (vt[j] - u[j]);        /* planted: beta dropped */
#else
        for (int j = 0; j < dv; ++j) u[j] = bt * (vt[j] - u[j]);
#endif
#if defined(KDA_ORACLE_MUTANT) && KDA_ORACLE_MUTANT == 1
        /* planted mistake 1: read the output before this token's write */
        {
            double *ot1 = J->o + ((size_t)t * H + h) * dv;
            for (int j = 0; j < dv; ++j) ot1[j] = 0.0;
            for (int i = 0; i < dk; ++i)
                for (int j = 0; j < dv; ++j) ot1[j] += qt[i] * S[(size_t)i * dv + j];
        }
#endif
        /* rank-one write along k */
        for (int i = 0; i < dk; ++i) {
            double *row = S + (size_t)i * dv;
            for (int j = 0; j < dv; ++j) row[j] += kt[i] * u[j];
        }
#if defined(KDA_ORACLE_MUTANT) && KDA_ORACLE_MUTANT == 2
        /* planted mistake 2: decay applied after the erase/write */
        for (int i = 0; i < dk; ++i) {
            const double a = exp(gt[i]);
            for (int j = 0; j < dv; ++j) S[(size_t)i * dv + j] *= a;
        }
#endif
#if !(defined(KDA_ORACLE_MUTANT) && KDA_ORACLE_MUTANT == 1)
        /* read-out from the updated state */
        double *ot = J->o + ((size_t)t * H + h) * dv;
        for (int j = 0; j < dv; ++j) ot[j] = 0.0;
        for (int i = 0; i < dk; ++i) {
            const double *row = S + (size_t)i * dv;
            for (int j = 0; j < dv; ++j) ot[j] += qt[i] * row[j];
        }
#endif
    }
    if (J->sT)
        memcpy(J->sT + ((size_t)n * H + h) * SS, S, SS * sizeof(double));
}

static void *worker(void *arg)
{
    job_t *J = (job_t *)arg;
    double *S = (double *)malloc((size_t)J->dk * J->dv * sizeof(double));
    double *u = (double *)malloc((size_t)J->dv * sizeof(double));
    if (!S || !u) { free(S); free(u); return (void *)1; }
    for (;;) {
        pthread_mutex_lock(&J->lock);
        const int p = J->next++;
        pthread_mutex_unlock(&J->lock);
        if (p >= J->N * J->H) break;
        run_pair(J, p / J->H, p % J->H, S, u);
    }
    free(S);
    free(u);
    return NULL;
}

/* Returns 0 on success, -1 on bad arguments, -2 on allocation/thread failure. */
int kda_oracle_fwd(const double *q, const double *k, const double *v,
                   const double *beta, const double *log_alpha,
                   const double *initial_state, const int64_t *cu_seqlens,
                   int N, int H, int dk, int dv, int erase,
                   double *o, double *final_state, int nthreads)
{
    if (!q || !k || !v || !beta || !log_alpha || !cu_seqlens || !o) return -1;
    if (N < 0 || H <= 0 || dk <= 0 || dv <= 0) return -1;
    if (N == 0) return 0;
    if (cu_seqlens[0] != 0) return -1;
    for (int n = 0; n < N; ++n)
        if (cu_seqlens[n + 1] < cu_seqlens[n]) return -1;
    if (nthreads < 1) nthreads = 1;
    if (nthreads > N * H) nthreads = N * H;

    job_t J;
    J.q = q; J.k = k; J.v = v; J.beta = beta; J.log_alpha = log_alpha;
    J.s0 = initial_state; J.cu = cu_seqlens;
    J.N = N; J.H = H; J.dk = dk; J.dv = dv; J.erase = erase ? 1 : 0;
    J.o = o; J.sT = final_state; J.next = 0;
    pthread_mutex_init(&J.lock, NULL);

    int rc = 0;
    pthread_t *th = (pthread_t *)malloc(sizeof(pthread_t) * (size_t)nthreads);
    if (!th) { pthread_mutex_destroy(&J.lock); return -2; }
    int started = 0;
    for (; started < nthreads; ++started)
        if (pthread_create(&th[started], NULL, worker, &J) != 0) { rc = -2; break; }
    for (int i = 0; i < started; ++i) {
        void *ret = NULL;
        pthread_join(th[i], &ret);
        if (ret) rc = -2;
    }
    if (started == 0) rc = -2;
    free(th);
    pthread_mutex_destroy(&J.lock);
    return rc;
}
