/*
 * synth_host.c -- host (CPU) fill routines of the seeded input generator
 * defined in synth.h.  Built with -ffp-contract=off so that every operation
 * of the definition is rounded exactly as written.
 *
 * All fill routines write a row/column block of a logical 2-D tensor whose
 * flat element index is row * ncols + col (the counter of synth.h), so a
 * caller can regenerate any sub-block of a huge tensor without producing the
 * rest.  Work is split over POSIX threads (SYNTH_THREADS, default: all
 * online cores).
 */
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <unistd.h>

#include "synth.h"

enum { KIND_BF16_NORMAL = 0, KIND_F32_NORMAL = 1, KIND_F32_UNIFORM = 2 };

typedef struct {
    int kind;
    uint64_t key;
    int64_t ncols, r0, c0, nr, nc;
    double scale;
    void* out;
    int64_t lo, hi; /* range of output elements [lo, hi) for this worker */
} job_t;

static void* worker(void* p) {
    job_t* j = (job_t*)p;
    for (int64_t e = j->lo; e < j->hi; ++e) {
        int64_t r = j->r0 + e / j->nc;
        int64_t c = j->c0 + e % j->nc;
        uint64_t i = (uint64_t)(r * j->ncols + c);
        switch (j->kind) {
        case KIND_BF16_NORMAL:
            ((uint16_t*)j->out)[e] = synth_bf16(j->scale * synth_normal(j->key, i));
            break;
        case KIND_F32_NORMAL:
            ((float*)j->out)[e] = synth_f32(j->scale * synth_normal(j->key, i));
            break;
        default:
            ((float*)j->out)[e] = synth_f32(j->scale * synth_uniform(j->key, i));
            break;
        }
    }
    return NULL;
}

static int num_threads(int64_t n) {
    const char* env = getenv("SYNTH_THREADS");
    long t = env ? atol(env) : sysconf(_SC_NPROCESSORS_ONLN);
    if (t < 1) t = 1;
    if (t > 256) t = 256;
    int64_t by_size = n / 65536 + 1;
    return (int)(t < by_size ? t : by_size);
}

static int run(int kind, uint64_t seed, int tensor, int64_t seq, int64_t ncols, int64_t r0, int64_t r1,
               int64_t c0, int64_t c1, double scale, void* out) {
    if (!out || ncols <= 0 || r1 < r0 || c1 < c0 || c0 < 0 || c1 > ncols || r0 < 0) return -1;
    int64_t nr = r1 - r0, nc = c1 - c0, n = nr * nc;
    if (n == 0) return 0;
    int nt = num_threads(n);
    pthread_t th[256];
    job_t jobs[256];
    for (int t = 0; t < nt; ++t) {
        jobs[t].kind = kind;
        jobs[t].key = synth_key(seed, (uint64_t)tensor, (uint64_t)seq);
        jobs[t].ncols = ncols;
        jobs[t].r0 = r0;
        jobs[t].c0 = c0;
        jobs[t].nr = nr;
        jobs[t].nc = nc;
        jobs[t].scale = scale;
        jobs[t].out = out;
        jobs[t].lo = n * t / nt;
        jobs[t].hi = n * (t + 1) / nt;
    }
    int started = 0;
    for (int t = 1; t < nt; ++t) {
        if (pthread_create(&th[t], NULL, worker, &jobs[t]) != 0) break;
        started = t;
    }
    worker(&jobs[0]);
    for (int t = started + 1; t < nt; ++t) worker(&jobs[t]); /* threads that failed to start */
    for (int t = 1; t <= started; ++t) pthread_join(th[t], NULL);
    return 0;
}

/* bf16( scale * normal(i) ) for rows [r0,r1) x cols [c0,c1); out is dense [(r1-r0), (c1-c0)]. */
int synth_fill_bf16_normal(uint64_t seed, int tensor, int64_t seq, int64_t ncols, int64_t r0, int64_t r1,
                           int64_t c0, int64_t c1, double scale, uint16_t* out) {
    return run(KIND_BF16_NORMAL, seed, tensor, seq, ncols, r0, r1, c0, c1, scale, out);
}

/* float( scale * normal(i) ). */
int synth_fill_f32_normal(uint64_t seed, int tensor, int64_t seq, int64_t ncols, int64_t r0, int64_t r1,
                          int64_t c0, int64_t c1, double scale, float* out) {
    return run(KIND_F32_NORMAL, seed, tensor, seq, ncols, r0, r1, c0, c1, scale, out);
}

/* float( scale * uniform(i) ). */
int synth_fill_f32_uniform(uint64_t seed, int tensor, int64_t seq, int64_t ncols, int64_t r0, int64_t r1,
                           int64_t c0, int64_t c1, double scale, float* out) {
    return run(KIND_F32_UNIFORM, seed, tensor, seq, ncols, r0, r1, c0, c1, scale, out);
}

/* Integer lengths lo + floor(uniform(b) * (hi - lo + 1)) for b in [0, n): uniform on [lo, hi]. */
int synth_lengths(uint64_t seed, int64_t n, int64_t lo, int64_t hi, int64_t* out) {
    if (!out || n < 0 || hi < lo) return -1;
    uint64_t key = synth_key(seed, SYNTH_LEN, 0);
    for (int64_t b = 0; b < n; ++b) {
        double u = synth_uniform(key, (uint64_t)b);
        out[b] = lo + (int64_t)(u * (double)(hi - lo + 1));
    }
    return 0;
}

/* Raw 64-bit draws, for tests of the generator itself. */
int synth_raw_bits(uint64_t seed, int tensor, int64_t seq, int64_t i0, int64_t n, uint64_t* out) {
    if (!out || n < 0) return -1;
    uint64_t key = synth_key(seed, (uint64_t)tensor, (uint64_t)seq);
    for (int64_t i = 0; i < n; ++i) out[i] = synth_bits(key, (uint64_t)(i0 + i));
    return 0;
}

/* The generator's own log, cos and bf16 rounding, exposed so that tests can
 * check them against a math library and against exhaustive rounding cases. */
double synth_log_host(double u) { return synth_log(u); }
double synth_cos2pi_host(double t) { return synth_cos2pi(t); }
uint16_t synth_bf16_host(double v) { return synth_bf16(v); }
