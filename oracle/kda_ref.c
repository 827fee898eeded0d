/*
 * kda_ref.c -- float64 CPU oracle for the KDA (Kimi Delta Attention) recurrence.
 *
 * TEST INFRASTRUCTURE ONLY. Nothing in the product path may call, link or run
 * this file: only the test suite, the smoke check and the benchmark's CPU
 * baseline leg use it. It shares no code, header or constant with the CUDA
 * library.
 *
 * What it computes (plain definition, token by token, no chunking):
 *
 *   for every sequence n and head h, starting from S = S0[n,h] (d_k x d_v):
 *     for each token t of the sequence, in order:
 *       S   <- (I - beta_t k_t k_t^T) . Diag(alpha_t) . S  +  beta_t k_t v_t^T
 *       o_t <- S^T q_t                      (reads the updated state)
 *     S_final[n,h] <- S
 *
 *   with alpha_t = exp(log_alpha_t), one decay per key channel.
 *
 * Sources: the channel-wise ("fine-grained") forget gate of KDA as a refined
 * Gated DeltaNet -- "Kimi Linear" news article (jdon.com), the passage on
 * KDA's fine-grained gating; the fixed-size per-head state and channel-level
 * gating -- KimiLinear KDA/MLA tutorial (icman.com.cn), sec. 2; the delta
 * erase term (I - beta k k^T) and its unit-norm key precondition -- same
 * tutorial, sec. 5. The pages print no formula; the order "decay, then erase
 * and write, then read" is the plainest reading of that delta-rule update.
 *
 * The product (I - beta k k^T)(Diag(alpha) S) is expanded as
 *   S' = Diag(alpha) S;  S <- S' - beta k (k^T S') + beta k v^T,
 * which is the same matrix product written without forming the d_k x d_k
 * matrix. All arithmetic is double; inputs arrive as float32 (every bf16
 * value is exactly representable in float32) and S0 as double.
 *
 * Layouts (row-major, last index fastest):
 *   q, k, log_alpha : [B, T, H, dk]      v : [B, T, H, dv]      beta : [B, T, H]
 *   S0, S_final     : [N, H, dk, dv]     out : [B, T, H, dv]
 *   cu_seqlens      : NULL (N = B, each batch row is one sequence of T tokens)
 *                     or int32 [N+1] offsets into the packed token axis (B = 1).
 *   S0 may be NULL (zero initial state); S_final and out may be NULL.
 *
 * Threads: (n, h) pairs are independent and are shared out over `nthreads`
 * POSIX threads (<= 0 means one per online core).
 *
 * Return value: 0 on success, -1 on an invalid argument.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <unistd.h>

typedef struct {
    const float *q, *k, *v, *log_alpha, *beta;
    const double *S0;
    const int32_t *cu_seqlens;
    int B, T, H, N, dk, dv;
    double *out, *S_final;
    int next;                 /* next (n, h) work item */
    pthread_mutex_t lock;
} job_t;

static void run_pair(job_t *J, int n, int h, double *S, double *w)
{
    const int H = J->H, dk = J->dk, dv = J->dv;
    int64_t t0, t1;
    if (J->cu_seqlens) {
        t0 = J->cu_seqlens[n];
        t1 = J->cu_seqlens[n + 1];
    } else {
        t0 = (int64_t)n * J->T;
        t1 = t0 + J->T;
    }
    const size_t sidx = ((size_t)n * H + h) * (size_t)dk * dv;
    if (J->S0)
        memcpy(S, J->S0 + sidx, sizeof(double) * (size_t)dk * dv);
    else
        memset(S, 0, sizeof(double) * (size_t)dk * dv);

    for (int64_t t = t0; t < t1; ++t) {
        const size_t row = (size_t)t * H + h;         /* flat (b, t) token index times H plus h */
        const float *qt = J->q + row * dk;
        const float *kt = J->k + row * dk;
        const float *vt = J->v + row * dv;
        const float *lat = J->log_alpha + row * dk;
        const double bt = (double)J->beta[row];

        /* S' = Diag(alpha_t) S : channel i of the key axis decays by exp(log_alpha_t[i]) */
        for (int i = 0; i < dk; ++i) {
            const double a = exp((double)lat[i]);
            double *Si = S + (size_t)i * dv;
            for (int j = 0; j < dv; ++j) Si[j] *= a;
        }
        /* w = S'^T k_t */
        for (int j = 0; j < dv; ++j) w[j] = 0.0;
        for (int i = 0; i < dk; ++i) {
            const double ki = (double)kt[i];
            const double *Si = S + (size_t)i * dv;
            for (int j = 0; j < dv; ++j) w[j] += ki * Si[j];
        }
        /* S = S' - beta k (k^T S') + beta k v^T = S' + beta k (v - w)^T */
        for (int i = 0; i < dk; ++i) {
            const double bki = bt * (double)kt[i];
            double *Si = S + (size_t)i * dv;
            for (int j = 0; j < dv; ++j) Si[j] += bki * ((double)vt[j] - w[j]);
        }
        /* o_t = S^T q_t */
        if (J->out) {
            double *ot = J->out + row * dv;
            for (int j = 0; j < dv; ++j) ot[j] = 0.0;
            for (int i = 0; i < dk; ++i) {
                const double qi = (double)qt[i];
                const double *Si = S + (size_t)i * dv;
                for (int j = 0; j < dv; ++j) ot[j] += qi * Si[j];
            }
        }
    }
    if (J->S_final)
        memcpy(J->S_final + sidx, S, sizeof(double) * (size_t)dk * dv);
}

static void *worker(void *arg)
{
    job_t *J = (job_t *)arg;
    double *S = (double *)malloc(sizeof(double) * (size_t)J->dk * J->dv);
    double *w = (double *)malloc(sizeof(double) * (size_t)J->dv);
    if (!S || !w) { free(S); free(w); return (void *)1; }
    for (;;) {
        pthread_mutex_lock(&J->lock);
        int item = J->next++;
        pthread_mutex_unlock(&J->lock);
        if (item >= J->N * J->H) break;
        run_pair(J, item / J->H, item % J->H, S, w);
    }
    free(S);
    free(w);
    return NULL;
}

int kda_oracle_forward(const float *q, const float *k, const float *v,
                       const float *log_alpha, const float *beta,
                       const double *S0, const int32_t *cu_seqlens,
                       int B, int T, int H, int N, int dk, int dv,
                       double *out, double *S_final, int nthreads)
{
    if (!q || !k || !v || !log_alpha || !beta) return -1;
    if (B < 0 || T < 0 || H <= 0 || dk <= 0 || dv <= 0) return -1;
    if (cu_seqlens) {
        if (B != 1 || N < 0) return -1;
        if (cu_seqlens[0] != 0 || cu_seqlens[N] != T) return -1;
        for (int n = 0; n < N; ++n)
            if (cu_seqlens[n + 1] < cu_seqlens[n]) return -1;
    } else {
        N = B;
    }
    job_t J;
    J.q = q; J.k = k; J.v = v; J.log_alpha = log_alpha; J.beta = beta;
    J.S0 = S0; J.cu_seqlens = cu_seqlens;
    J.B = B; J.T = T; J.H = H; J.N = N; J.dk = dk; J.dv = dv;
    J.out = out; J.S_final = S_final; J.next = 0;
    pthread_mutex_init(&J.lock, NULL);

    int items = N * H;
    if (nthreads <= 0) nthreads = (int)sysconf(_SC_NPROCESSORS_ONLN);
    if (nthreads < 1) nthreads = 1;
    if (nthreads > items) nthreads = items > 0 ? items : 1;
    int rc = 0;
    if (nthreads == 1) {
        if (worker(&J) != NULL) rc = -1;
    } else {
        pthread_t *th = (pthread_t *)malloc(sizeof(pthread_t) * (size_t)nthreads);
        if (!th) { pthread_mutex_destroy(&J.lock); return -1; }
        int started = 0;
        for (; started < nthreads; ++started)
            if (pthread_create(&th[started], NULL, worker, &J) != 0) break;
        if (started == 0 && worker(&J) != NULL) rc = -1;
        for (int i = 0; i < started; ++i) {
            void *r = NULL;
            pthread_join(th[i], &r);
            if (r != NULL) rc = -1;
        }
        free(th);
    }
    pthread_mutex_destroy(&J.lock);
    return rc;
}

int kda_oracle_online_cores(void)
{
    return (int)sysconf(_SC_NPROCESSORS_ONLN);
}
