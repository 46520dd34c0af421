/*
 * gen.c -- bulk generation for the seeded input streams (see __init__.py).
 *
 * Element i of stream (seed, tensor_id) is a pure function of (seed,
 * tensor_id, i): SplitMix64 mixing (Steele, Lea & Flood, OOPSLA 2014) of
 * counter values, two 53-bit uniforms in (0,1), Box-Muller for normals.
 * This file draws random numbers only; it holds none of the scan's arithmetic.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>

#define GOLDEN 0x9E3779B97F4A7C15ULL

static inline uint64_t mix64(uint64_t z) {
    z ^= z >> 30; z *= 0xBF58476D1CE4E5B9ULL;
    z ^= z >> 27; z *= 0x94D049BB133111EBULL;
    return z ^ (z >> 31);
}

uint64_t stream_key(uint64_t seed, uint64_t tensor_id) {
    return mix64(((seed << 32) | tensor_id) + GOLDEN);
}

static inline void uniform_pair(uint64_t key, uint64_t i, double *u1, double *u2) {
    const double scale = 1.0 / 9007199254740992.0; /* 2^-53 */
    uint64_t w1 = mix64(key + (2 * i + 1) * GOLDEN);
    uint64_t w2 = mix64(key + (2 * i + 2) * GOLDEN);
    *u1 = ((double)(w1 >> 11) + 0.5) * scale;
    *u2 = ((double)(w2 >> 11) + 0.5) * scale;
}

typedef struct {
    uint64_t key; const int64_t *idx; int64_t start, n; double *out; int normal;
} job_t;

static void *run(void *arg) {
    job_t *j = (job_t *)arg;
    const double two_pi = 6.283185307179586476925286766559;
    for (int64_t k = 0; k < j->n; ++k) {
        uint64_t i = j->idx ? (uint64_t)j->idx[k] : (uint64_t)(j->start + k);
        double u1, u2;
        uniform_pair(j->key, i, &u1, &u2);
        j->out[k] = j->normal ? sqrt(-2.0 * log(u1)) * cos(two_pi * u2) : u1;
    }
    return NULL;
}

/* out[k] = element (idx ? idx[k] : start + k) of the stream, for k < n. */
int gen_stream(uint64_t seed, uint64_t tensor_id, int normal, int64_t start, const int64_t *idx,
               int64_t n, double *out, int nthreads) {
    if (n <= 0) return 0;
    if (nthreads < 1) nthreads = 1;
    if (n < 65536) nthreads = 1;
    job_t *jobs = (job_t *)malloc(sizeof(job_t) * nthreads);
    pthread_t *th = (pthread_t *)malloc(sizeof(pthread_t) * nthreads);
    if (!jobs || !th) { free(jobs); free(th); return -1; }
    uint64_t key = stream_key(seed, tensor_id);
    int64_t per = (n + nthreads - 1) / nthreads;
    for (int t = 0; t < nthreads; ++t) {
        int64_t s = t * per, e = s + per < n ? s + per : n;
        jobs[t].key = key; jobs[t].normal = normal; jobs[t].n = e > s ? e - s : 0;
        jobs[t].idx = idx ? idx + s : NULL; jobs[t].start = start + s; jobs[t].out = out + s;
        pthread_create(&th[t], NULL, run, &jobs[t]);
    }
    for (int t = 0; t < nthreads; ++t) pthread_join(th[t], NULL);
    free(jobs); free(th);
    return 0;
}
