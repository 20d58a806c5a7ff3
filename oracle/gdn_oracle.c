/*
 * gdn_oracle.c -- TEST INFRASTRUCTURE ONLY.
 *
 * Plain, slow, obviously correct fp64 CPU reference of the Gated DeltaNet
 * token mixer used by InfiniteVL.  Only the tests, the smoke check and the
 * benchmark's CPU-baseline leg may load this file's library.  It shares no
 * code, header or constant with the CUDA path.
 *
 * What it computes (InfiniteVL explainer page, "Gated DeltaNet" concept box
 * and "Building Blocks": a fixed-size memory matrix per head; a gate decides
 * how much old memory is kept; an erase step along the key direction; a
 * write of the new value; a read with the current query).  The pages give no
 * equation; the recurrence is the standard gated delta rule, per sequence n
 * and head h, token by token:
 *
 *     a   = exp(g_t)                      (g_t = log alpha_t, per token/head)
 *     sk  = S k_t                         (d_v vector)
 *     u   = beta_t (v_t - a sk)           (delta residual vs the decayed state)
 *     S   = a S + u k_t^T                 (== a S (I - beta k k^T) + beta v k^T)
 *     o_t = S q_t                         (read-out uses the UPDATED state)
 *
 * S is d_v x d_k, row-major (S[i*dk + j]), fp64.  No 1/sqrt(d_k) scale and no
 * normalisation is applied here: the caller passes q, k, v, g, beta as they
 * are (already rounded to their storage precision and widened to double).
 *
 * Layouts (all row-major, contiguous):
 *   q, k   [T_total, H, dk]      v, out [T_total, H, dv]
 *   g, beta [T_total, H]         state  [N, H, dv, dk]
 *   cu_seqlens [N+1] (int64, non-decreasing, cu_seqlens[0] = 0)
 *
 * Parallelism: independent (sequence, head) units are spread over POSIX
 * threads.  Each unit runs the loop above exactly in token order; threading
 * changes no arithmetic.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* One token of the recurrence for one head.  sk is caller scratch (dv). */
static void gdn_oracle_token(double *S, int dk, int dv,
                             const double *q, const double *k, const double *v,
                             double g, double beta, double *sk, double *o)
{
    const double a = exp(g);
    /* sk = S k */
    for (int i = 0; i < dv; ++i) {
        double acc = 0.0;
        for (int j = 0; j < dk; ++j) acc += S[(size_t)i * dk + j] * k[j];
        sk[i] = acc;
    }
    /* S = a S + u k^T with u = beta (v - a sk) */
    for (int i = 0; i < dv; ++i) {
        const double u = beta * (v[i] - a * sk[i]);
        for (int j = 0; j < dk; ++j)
            S[(size_t)i * dk + j] = a * S[(size_t)i * dk + j] + u * k[j];
    }
    /* o = S q */
    for (int i = 0; i < dv; ++i) {
        double acc = 0.0;
        for (int j = 0; j < dk; ++j) acc += S[(size_t)i * dk + j] * q[j];
        o[i] = acc;
    }
}

typedef struct {
    const double *q, *k, *v, *g, *beta, *state_in;
    double *out, *state_out;
    const int64_t *cu_seqlens;
    int num_seqs, H, dk, dv;
    int next_unit;              /* work counter, guarded by mu */
    pthread_mutex_t mu;
    int failed;
} gdn_oracle_job;

static void gdn_oracle_unit(gdn_oracle_job *J, int unit, double *S, double *sk)
{
    const int n = unit / J->H, h = unit % J->H;
    const int H = J->H, dk = J->dk, dv = J->dv;
    const size_t ssz = (size_t)dv * dk;
    const size_t soff = ((size_t)n * H + h) * ssz;
    if (J->state_in) memcpy(S, J->state_in + soff, ssz * sizeof(double));
    else memset(S, 0, ssz * sizeof(double));
    for (int64_t t = J->cu_seqlens[n]; t < J->cu_seqlens[n + 1]; ++t) {
        const size_t th = (size_t)t * H + h;
        gdn_oracle_token(S, dk, dv, J->q + th * dk, J->k + th * dk,
                         J->v + th * dv, J->g[th], J->beta[th], sk,
                         J->out + th * dv);
    }
    if (J->state_out) memcpy(J->state_out + soff, S, ssz * sizeof(double));
}

static void *gdn_oracle_worker(void *arg)
{
    gdn_oracle_job *J = (gdn_oracle_job *)arg;
    const size_t ssz = (size_t)J->dv * J->dk;
    double *S = (double *)malloc(ssz * sizeof(double));
    double *sk = (double *)malloc((size_t)J->dv * sizeof(double));
    if (!S || !sk) {
        pthread_mutex_lock(&J->mu);
        J->failed = 1;
        pthread_mutex_unlock(&J->mu);
        free(S);
        free(sk);
        return NULL;
    }
    const int units = J->num_seqs * J->H;
    for (;;) {
        pthread_mutex_lock(&J->mu);
        const int u = J->next_unit++;
        pthread_mutex_unlock(&J->mu);
        if (u >= units) break;
        gdn_oracle_unit(J, u, S, sk);
    }
    free(S);
    free(sk);
    return NULL;
}

/*
 * Prefill over a packed batch.  state_in may be NULL (zero initial state);
 * state_out may be NULL (not written).  Returns 0 on success, -1 on bad
 * arguments, -2 if memory or threads could not be obtained.
 */
int gdn_oracle_prefill(const double *q, const double *k, const double *v,
                       const double *g, const double *beta,
                       const double *state_in, double *out, double *state_out,
                       const int64_t *cu_seqlens, int num_seqs, int H, int dk,
                       int dv, int nthreads)
{
    if (!q || !k || !v || !g || !beta || !out || !cu_seqlens) return -1;
    if (num_seqs < 0 || H <= 0 || dk <= 0 || dv <= 0) return -1;
    if (cu_seqlens[0] != 0) return -1;
    for (int n = 0; n < num_seqs; ++n)
        if (cu_seqlens[n + 1] < cu_seqlens[n]) return -1;
    gdn_oracle_job J;
    J.q = q; J.k = k; J.v = v; J.g = g; J.beta = beta;
    J.state_in = state_in; J.out = out; J.state_out = state_out;
    J.cu_seqlens = cu_seqlens;
    J.num_seqs = num_seqs; J.H = H; J.dk = dk; J.dv = dv;
    J.next_unit = 0;
    J.failed = 0;
    pthread_mutex_init(&J.mu, NULL);
    const int units = num_seqs * H;
    if (nthreads < 1) nthreads = 1;
    if (nthreads > units) nthreads = units > 0 ? units : 1;
    pthread_t *th = (pthread_t *)malloc((size_t)nthreads * sizeof(pthread_t));
    if (!th) { pthread_mutex_destroy(&J.mu); return -2; }
    int started = 0;
    for (int i = 0; i < nthreads; ++i) {
        if (pthread_create(&th[i], NULL, gdn_oracle_worker, &J) != 0) break;
        ++started;
    }
    if (started == 0) gdn_oracle_worker(&J);  /* run inline */
    for (int i = 0; i < started; ++i) pthread_join(th[i], NULL);
    free(th);
    pthread_mutex_destroy(&J.mu);
    return J.failed ? -2 : 0;
}

/*
 * One decode step for B independent sequences: each sequence receives one
 * token.  The same recurrence as above with T = 1 per sequence.
 * q, k [B, H, dk]; v, out [B, H, dv]; g, beta [B, H]; state [B, H, dv, dk]
 * (updated in place).
 */
int gdn_oracle_decode(const double *q, const double *k, const double *v,
                      const double *g, const double *beta, double *state,
                      double *out, int B, int H, int dk, int dv)
{
    if (!q || !k || !v || !g || !beta || !state || !out) return -1;
    if (B < 0 || H <= 0 || dk <= 0 || dv <= 0) return -1;
    double *sk = (double *)malloc((size_t)dv * sizeof(double));
    if (!sk) return -2;
    for (int b = 0; b < B; ++b)
        for (int h = 0; h < H; ++h) {
            const size_t bh = (size_t)b * H + h;
            gdn_oracle_token(state + bh * dv * dk, dk, dv, q + bh * dk,
                             k + bh * dk, v + bh * dv, g[bh], beta[bh], sk,
                             out + bh * dv);
        }
    free(sk);
    return 0;
}
