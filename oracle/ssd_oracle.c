/*
 * ssd_oracle.c -- float64 CPU oracle for the selective state-space (SSD) scan.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the checker, not the product: only
 * the tests, the smoke check and the bench's CPU-baseline leg load it.  It
 * shares no code, header or constant with the CUDA library, and the library
 * never calls it.
 *
 * What it computes (plain definition, no blocking, no reordering):
 *
 *   The scan is the Mamba-2 selective state-space recurrence.  The DiffuMamba
 *   page ("DiffuMamba: High-Throughput Diffusion LMs with Mamba Backbone",
 *   technical summary, section 2 Methodology) names a bidirectional Mamba-2
 *   mixer; the Bifocal dLLM / R2LM page ("Bifocal Diffusion Language Models",
 *   section 2 Methodology, mechanism) names the selective scan that the
 *   right-to-left stream applies.  Neither page prints the recurrence; the
 *   standard Mamba-2 form with a scalar decay per head is taken:
 *
 *     for every batch b and head h (group g = h / (H/G)), state S in R^{P x N},
 *     S = 0 before the first token, and for each token t in scan order:
 *       S      <- exp(dt[b,t,h] * A[h]) * S + dt[b,t,h] * x[b,t,h,:] (outer) B[b,t,g,:]
 *       y[b,t,h,p] = sum_n C[b,t,g,n] * S[p,n] + D[h] * x[b,t,h,p]
 *
 *   direction = +1 visits t = 0 .. L-1; direction = -1 visits t = L-1 .. 0,
 *   which is the R2LM "flip the sequence, scan, flip back" (section 2,
 *   mechanism) written as a reversed loop.
 *
 *   ssd_oracle_scan_state also takes the state before the first scanned token
 *   and returns the state after the last one.  That is what block-wise
 *   decoding needs: the DiffuMamba page (technical summary, section 2,
 *   training and inference; section 4, block caching) runs block diffusion
 *   with cache reuse, and for a Mamba layer the reusable cache of everything
 *   before a block is this state.
 *
 * Layouts (row-major, contiguous): x, y [B][L][H][P]; dt [B][L][H];
 * B, C [B][L][G][N]; A, D [H]; states [B][H][P][N].  D may be NULL (no skip
 * term).
 * Work is split over (b, h) pairs across POSIX threads; each pair is computed
 * by one thread in the order above, so the result does not depend on the
 * thread count.
 */
#include <math.h>
#include <pthread.h>
#include <stdlib.h>
#include <string.h>

typedef struct {
    int batch, seqlen, nheads, headdim, dstate, ngroups, direction;
    const double *x, *dt, *A, *B, *C, *D;
    double *y;
    const double *s_in;    /* state before the first scanned token, [B][H][P][N], or NULL = 0 */
    double *s_out;         /* state after the last scanned token, [B][H][P][N], or NULL */
    int next;              /* next (b,h) pair to take */
    pthread_mutex_t lock;
} job_t;

static void scan_pair(const job_t *j, int b, int h, double *S)
{
    const int L = j->seqlen, H = j->nheads, P = j->headdim, N = j->dstate;
    const int g = h / (H / j->ngroups);
    const double a_h = j->A[h];
    const double d_h = j->D ? j->D[h] : 0.0;
    const size_t soff = ((size_t)b * H + h) * (size_t)P * N;
    if (j->s_in)
        memcpy(S, j->s_in + soff, sizeof(double) * (size_t)P * N);
    else
        memset(S, 0, sizeof(double) * (size_t)P * N);
    for (int k = 0; k < L; ++k) {
        const int t = j->direction > 0 ? k : L - 1 - k;
        const double dt = j->dt[((size_t)b * L + t) * H + h];
        const double decay = exp(dt * a_h);
        const double *xt = j->x + (((size_t)b * L + t) * H + h) * P;
        const double *Bt = j->B + (((size_t)b * L + t) * j->ngroups + g) * N;
        const double *Ct = j->C + (((size_t)b * L + t) * j->ngroups + g) * N;
        double *yt = j->y + (((size_t)b * L + t) * H + h) * P;
        for (int p = 0; p < P; ++p) {
            double *Sp = S + (size_t)p * N;
            const double u = dt * xt[p];
            double acc = 0.0;
            for (int n = 0; n < N; ++n) {
                Sp[n] = decay * Sp[n] + u * Bt[n];
                acc += Ct[n] * Sp[n];
            }
            yt[p] = acc + d_h * xt[p];
        }
    }
    if (j->s_out) memcpy(j->s_out + soff, S, sizeof(double) * (size_t)P * N);
}

static void *worker(void *arg)
{
    job_t *j = (job_t *)arg;
    double *S = (double *)malloc(sizeof(double) * (size_t)j->headdim * j->dstate);
    if (!S) return (void *)1;
    for (;;) {
        pthread_mutex_lock(&j->lock);
        int w = j->next++;
        pthread_mutex_unlock(&j->lock);
        if (w >= j->batch * j->nheads) break;
        scan_pair(j, w / j->nheads, w % j->nheads, S);
    }
    free(S);
    return NULL;
}

/* The scan with the state carried across the call boundary: s_in (may be NULL
 * = zero) is the state before the first token in scan order, s_out (may be
 * NULL) receives the state after the last one.  Both are [B][H][P][N].  Scanning
 * a sequence in two pieces, the second starting from the first's s_out, gives
 * the same y and final state as scanning it whole (the recurrence only looks at
 * S and the current token).  Returns 0, -1 on bad arguments, -2 on allocation
 * failure. */
int ssd_oracle_scan_state(int batch, int seqlen, int nheads, int headdim, int dstate, int ngroups,
                          const double *x, const double *dt, const double *A, const double *B,
                          const double *C, const double *D, int direction, const double *s_in,
                          double *y, double *s_out, int nthreads)
{
    if (batch < 0 || seqlen < 0 || nheads <= 0 || headdim <= 0 || dstate <= 0 || ngroups <= 0)
        return -1;
    if (nheads % ngroups != 0 || (direction != 1 && direction != -1)) return -1;
    if (batch == 0) return 0;
    if (seqlen == 0) {
        /* no token: the state passes through unchanged */
        if (s_out) {
            const size_t n = (size_t)batch * nheads * headdim * dstate;
            if (s_in) memcpy(s_out, s_in, sizeof(double) * n);
            else memset(s_out, 0, sizeof(double) * n);
        }
        return 0;
    }
    if (!x || !dt || !A || !B || !C || !y) return -1;
    job_t j = {batch, seqlen, nheads, headdim, dstate, ngroups, direction,
               x, dt, A, B, C, D, y, s_in, s_out, 0};
    pthread_mutex_init(&j.lock, NULL);
    int pairs = batch * nheads;
    if (nthreads < 1) nthreads = 1;
    if (nthreads > pairs) nthreads = pairs;
    pthread_t *th = (pthread_t *)malloc(sizeof(pthread_t) * (size_t)nthreads);
    if (!th) return -2;
    int rc = 0;
    for (int i = 0; i < nthreads; ++i) pthread_create(&th[i], NULL, worker, &j);
    for (int i = 0; i < nthreads; ++i) {
        void *r = NULL;
        pthread_join(th[i], &r);
        if (r) rc = -2;
    }
    free(th);
    pthread_mutex_destroy(&j.lock);
    return rc;
}

/* The scan from a zero state.  Returns 0 on success, -1 on bad arguments, -2 on
 * allocation failure. */
int ssd_oracle_scan(int batch, int seqlen, int nheads, int headdim, int dstate, int ngroups,
                    const double *x, const double *dt, const double *A, const double *B,
                    const double *C, const double *D, int direction, double *y, int nthreads)
{
    return ssd_oracle_scan_state(batch, seqlen, nheads, headdim, dstate, ngroups, x, dt, A, B, C, D,
                                 direction, NULL, y, NULL, nthreads);
}
