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

/* ------------------------------------------------------------------ gradients
 *
 * Reverse-mode derivative of the scan above (for training the layers that run
 * it; the DiffuMamba page, technical summary, section 2, trains the Mamba
 * backbone with the masked-diffusion objective).  Given gy = dL/dy it returns
 * dL/dx, dL/ddt, dL/dA, dL/dB, dL/dC and dL/dD, from the zero starting state.
 *
 * With k the scan position and t its token, S_k = a_k S_{k-1} + dt_t x_t B_t^T,
 * a_k = exp(dt_t A), y_t = S_k C_t + D x_t.  The total derivative of L with
 * respect to S_k is  G_k = gy_t C_t^T + a_{k+1} G_{k+1}  (G after the last
 * position is 0), and then, term by term,
 *   dC_t   = S_k^T gy_t
 *   dx_t   = dt_t G_k B_t + D gy_t
 *   dB_t   = dt_t G_k^T x_t
 *   ddt_t  = <G_k, x_t B_t^T> + A a_k <G_k, S_{k-1}>
 *   dA     = sum_k dt_t a_k <G_k, S_{k-1}>
 *   dD     = sum_t <gy_t, x_t>
 * B and C of a group collect the contributions of every head in the group.
 * The states S_{k-1} are recomputed segment by segment from checkpoints taken
 * every BWD_SEG positions, so memory stays O(P N (L/BWD_SEG + BWD_SEG)).
 */
#define BWD_SEG 64

typedef struct {
    int batch, seqlen, nheads, headdim, dstate, ngroups, direction;
    const double *x, *dt, *A, *B, *C, *D, *gy;
    double *gx, *gdt, *gB, *gC;
    double *gA_part, *gD_part;   /* [B][H] partial sums, added up by the caller */
    int next;                    /* next (b, g) unit to take */
    int err;
    pthread_mutex_t lock;
} bjob_t;

static void bwd_head(const bjob_t *j, int b, int h, double *ck, double *seg, double *G)
{
    const int L = j->seqlen, H = j->nheads, P = j->headdim, N = j->dstate, GR = j->ngroups;
    const int g = h / (H / GR);
    const size_t PN = (size_t)P * N;
    const int nseg = (L + BWD_SEG - 1) / BWD_SEG;
    const double a_h = j->A[h], d_h = j->D ? j->D[h] : 0.0;
    double gA = 0.0, gD = 0.0;
#define TOK(k) (j->direction > 0 ? (k) : L - 1 - (k))
#define XP(t) (j->x + (((size_t)b * L + (t)) * H + h) * P)
#define GYP(t) (j->gy + (((size_t)b * L + (t)) * H + h) * P)
#define BP(t) (j->B + (((size_t)b * L + (t)) * GR + g) * N)
#define CP(t) (j->C + (((size_t)b * L + (t)) * GR + g) * N)
#define DT(t) (j->dt[((size_t)b * L + (t)) * H + h])
    /* forward: checkpoint the state before every segment */
    double *S = seg; /* scratch for the running state during the checkpoint pass */
    memset(S, 0, sizeof(double) * PN);
    for (int k = 0; k < L; ++k) {
        if (k % BWD_SEG == 0) memcpy(ck + (size_t)(k / BWD_SEG) * PN, S, sizeof(double) * PN);
        const int t = TOK(k);
        const double dt = DT(t), a = exp(dt * a_h);
        const double *xt = XP(t), *Bt = BP(t);
        for (int p = 0; p < P; ++p)
            for (int n = 0; n < N; ++n) S[(size_t)p * N + n] = a * S[(size_t)p * N + n] + dt * xt[p] * Bt[n];
    }
    /* backward, segment by segment from the end */
    memset(G, 0, sizeof(double) * PN);
    for (int sgi = nseg - 1; sgi >= 0; --sgi) {
        const int k0 = sgi * BWD_SEG, k1 = (k0 + BWD_SEG < L) ? k0 + BWD_SEG : L;
        /* seg[i] = S after position k0 + i; ck[sgi] = S before position k0 */
        const double *prev = ck + (size_t)sgi * PN;
        for (int k = k0; k < k1; ++k) {
            const int t = TOK(k);
            const double dt = DT(t), a = exp(dt * a_h);
            const double *xt = XP(t), *Bt = BP(t);
            double *Sk = seg + (size_t)(k - k0) * PN;
            for (int p = 0; p < P; ++p)
                for (int n = 0; n < N; ++n)
                    Sk[(size_t)p * N + n] = a * prev[(size_t)p * N + n] + dt * xt[p] * Bt[n];
            prev = Sk;
        }
        for (int k = k1 - 1; k >= k0; --k) {
            const int t = TOK(k);
            const double dt = DT(t), a = exp(dt * a_h);
            const double *xt = XP(t), *Bt = BP(t), *Ct = CP(t), *gyt = GYP(t);
            const double *Sk = seg + (size_t)(k - k0) * PN;
            const double *Sprev = (k == k0) ? ck + (size_t)sgi * PN : seg + (size_t)(k - 1 - k0) * PN;
            double *gxt = j->gx + (((size_t)b * L + t) * H + h) * P;
            double *gBt = j->gB + (((size_t)b * L + t) * GR + g) * N;
            double *gCt = j->gC + (((size_t)b * L + t) * GR + g) * N;
            /* G_k = gy_t C_t^T + (a_{k+1} G_{k+1}, already in G) */
            for (int p = 0; p < P; ++p)
                for (int n = 0; n < N; ++n) G[(size_t)p * N + n] += gyt[p] * Ct[n];
            for (int n = 0; n < N; ++n) {
                double acc = 0.0;
                for (int p = 0; p < P; ++p) acc += gyt[p] * Sk[(size_t)p * N + n];
                gCt[n] += acc;
            }
            double gxb = 0.0, q = 0.0;
            for (int p = 0; p < P; ++p) {
                double acc = 0.0;
                for (int n = 0; n < N; ++n) {
                    acc += G[(size_t)p * N + n] * Bt[n];
                    q += G[(size_t)p * N + n] * Sprev[(size_t)p * N + n];
                }
                gxt[p] = dt * acc + d_h * gyt[p];
                gxb += acc * xt[p];               /* <G_k, x_t B_t^T> */
            }
            for (int n = 0; n < N; ++n) {
                double acc = 0.0;
                for (int p = 0; p < P; ++p) acc += G[(size_t)p * N + n] * xt[p];
                gBt[n] += dt * acc;
            }
            j->gdt[((size_t)b * L + t) * H + h] = gxb + a_h * a * q;
            gA += dt * a * q;
            for (int p = 0; p < P; ++p) gD += gyt[p] * xt[p];
            for (size_t i = 0; i < PN; ++i) G[i] *= a;      /* becomes a_k G_k for position k - 1 */
        }
    }
    j->gA_part[(size_t)b * H + h] = gA;
    j->gD_part[(size_t)b * H + h] = gD;
#undef TOK
#undef XP
#undef GYP
#undef BP
#undef CP
#undef DT
}

static void *bwd_worker(void *arg)
{
    bjob_t *j = (bjob_t *)arg;
    const size_t PN = (size_t)j->headdim * j->dstate;
    const int nseg = (j->seqlen + BWD_SEG - 1) / BWD_SEG;
    double *ck = (double *)malloc(sizeof(double) * PN * (size_t)nseg);
    double *seg = (double *)malloc(sizeof(double) * PN * BWD_SEG);
    double *G = (double *)malloc(sizeof(double) * PN);
    if (!ck || !seg || !G) {
        free(ck); free(seg); free(G);
        return (void *)1;
    }
    const int per_group = j->nheads / j->ngroups;
    for (;;) {
        pthread_mutex_lock(&j->lock);
        int w = j->next++;
        pthread_mutex_unlock(&j->lock);
        if (w >= j->batch * j->ngroups) break;
        const int b = w / j->ngroups, g = w % j->ngroups;
        /* every head of the group in this thread: their B and C gradients add up without races */
        for (int h = g * per_group; h < (g + 1) * per_group; ++h) bwd_head(j, b, h, ck, seg, G);
    }
    free(ck); free(seg); free(G);
    return NULL;
}

/* Gradients of the scan (zero starting state).  gx, gdt, gB, gC are written
 * (gB, gC summed over the heads of each group); gA [H] and, when D is not
 * NULL, gD [H] are summed over the batch.  Returns 0, -1 on bad arguments, -2
 * on allocation failure. */
int ssd_oracle_scan_bwd(int batch, int seqlen, int nheads, int headdim, int dstate, int ngroups,
                        const double *x, const double *dt, const double *A, const double *B,
                        const double *C, const double *D, int direction, const double *gy,
                        double *gx, double *gdt, double *gA, double *gB, double *gC, double *gD,
                        int nthreads)
{
    if (batch < 0 || seqlen < 0 || nheads <= 0 || headdim <= 0 || dstate <= 0 || ngroups <= 0)
        return -1;
    if (nheads % ngroups != 0 || (direction != 1 && direction != -1)) return -1;
    if (!gA) return -1;
    memset(gA, 0, sizeof(double) * nheads);
    if (gD) memset(gD, 0, sizeof(double) * nheads);
    if (batch == 0 || seqlen == 0) return 0;
    if (!x || !dt || !A || !B || !C || !gy || !gx || !gdt || !gB || !gC) return -1;
    const size_t nbc = (size_t)batch * seqlen * ngroups * dstate;
    memset(gB, 0, sizeof(double) * nbc);
    memset(gC, 0, sizeof(double) * nbc);
    double *gA_part = (double *)calloc((size_t)batch * nheads, sizeof(double));
    double *gD_part = (double *)calloc((size_t)batch * nheads, sizeof(double));
    if (!gA_part || !gD_part) {
        free(gA_part); free(gD_part);
        return -2;
    }
    bjob_t j = {batch, seqlen, nheads, headdim, dstate, ngroups, direction,
                x, dt, A, B, C, D, gy, gx, gdt, gB, gC, gA_part, gD_part, 0, 0};
    pthread_mutex_init(&j.lock, NULL);
    int units = batch * ngroups;
    if (nthreads < 1) nthreads = 1;
    if (nthreads > units) nthreads = units;
    pthread_t *th = (pthread_t *)malloc(sizeof(pthread_t) * (size_t)nthreads);
    int rc = 0;
    if (!th) {
        rc = -2;
    } else {
        for (int i = 0; i < nthreads; ++i) pthread_create(&th[i], NULL, bwd_worker, &j);
        for (int i = 0; i < nthreads; ++i) {
            void *r = NULL;
            pthread_join(th[i], &r);
            if (r) rc = -2;
        }
        free(th);
    }
    pthread_mutex_destroy(&j.lock);
    for (int b = 0; b < batch; ++b)
        for (int h = 0; h < nheads; ++h) {
            gA[h] += gA_part[(size_t)b * nheads + h];
            if (gD) gD[h] += gD_part[(size_t)b * nheads + h];
        }
    free(gA_part); free(gD_part);
    return rc;
}
