/*
 * kda_synth.c -- seeded, counter-based synthetic inputs for the KDA workloads.
 *
 * This module holds only input generation (random numbers, their
 * distributions, L2 normalisation of q/k rows, round-to-nearest-even bf16
 * encoding).  It contains none of the recurrence's arithmetic and is used by
 * both the CUDA path's tests/benchmark and the CPU oracle's tests, so the two
 * sides see bit-identical inputs.
 *
 * Generator: SplitMix64 (Steele, Lea, Flood, "Fast splittable pseudorandom
 * number generators", OOPSLA 2014) used in counter mode: element `i` of a
 * stream with key `K` is the (i+1)-th output of a SplitMix64 seeded with K,
 * i.e. mix(K + (i+1)*gamma).  Any block of any tensor can therefore be
 * generated on its own and equals the same block of the whole tensor.
 * Standard normals use the Box-Muller transform on two consecutive uniforms.
 */
#define _GNU_SOURCE
#include <math.h>
#include <pthread.h>
#include <sched.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define SY_API __attribute__((visibility("default")))

static const uint64_t SM_GAMMA = 0x9E3779B97F4A7C15ULL;

static inline uint64_t sm_mix(uint64_t z) {
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
    return z ^ (z >> 31);
}

/* Stream key for (seed, tag). */
static inline uint64_t sy_key(uint64_t seed, uint64_t tag) {
    return sm_mix(sm_mix(seed + SM_GAMMA) ^ (tag * 0xD1B54A32D192ED03ULL));
}

/* uniform in [0,1) with 53 random bits */
static inline double sy_uniform(uint64_t key, uint64_t ctr) {
    return (double)(sm_mix(key + (ctr + 1) * SM_GAMMA) >> 11) * (1.0 / 9007199254740992.0);
}

static inline double sy_normal(uint64_t key, uint64_t i) {
    const double u1 = sy_uniform(key, 2 * i);
    const double u2 = sy_uniform(key, 2 * i + 1);
    const double r = sqrt(-2.0 * log(1.0 - u1)); /* 1-u1 in (0,1] */
    return r * cos(6.283185307179586 * u2);
}

/* float -> bf16 bits, round to nearest even (NaN kept quiet) */
static inline uint16_t sy_bf16_bits(float f) {
    uint32_t x;
    memcpy(&x, &f, 4);
    if ((x & 0x7F800000u) == 0x7F800000u && (x & 0x007FFFFFu)) return (uint16_t)((x >> 16) | 0x40);
    const uint32_t lsb = (x >> 16) & 1u;
    x += 0x7FFFu + lsb;
    return (uint16_t)(x >> 16);
}

static inline float sy_bf16_round(float f) {
    uint32_t x = (uint32_t)sy_bf16_bits(f) << 16;
    float r;
    memcpy(&r, &x, 4);
    return r;
}

/* ---------------- threading ---------------- */

typedef void (*sy_range_fn)(void* ctx, int64_t begin, int64_t end);
typedef struct { sy_range_fn fn; void* ctx; int64_t b, e; } sy_job;

static void* sy_worker(void* a) {
    sy_job* j = (sy_job*)a;
    j->fn(j->ctx, j->b, j->e);
    return NULL;
}

static int sy_cores(void) {
    cpu_set_t set;
    CPU_ZERO(&set);
    if (sched_getaffinity(0, sizeof(set), &set) == 0 && CPU_COUNT(&set) > 0) return CPU_COUNT(&set);
    return 1;
}

/* splits [0, n) into contiguous ranges over the available cores */
static void sy_parallel(sy_range_fn fn, void* ctx, int64_t n) {
    int nt = sy_cores();
    if (nt > 64) nt = 64;
    if (n < 65536 || nt <= 1) { fn(ctx, 0, n); return; }
    pthread_t th[64];
    sy_job jobs[64];
    for (int i = 0; i < nt; ++i) {
        jobs[i].fn = fn; jobs[i].ctx = ctx;
        jobs[i].b = n * i / nt; jobs[i].e = n * (i + 1) / nt;
        pthread_create(&th[i], NULL, sy_worker, &jobs[i]);
    }
    for (int i = 0; i < nt; ++i) pthread_join(th[i], NULL);
}

/* ---------------- element-wise distributions ---------------- */

enum { SY_NORMAL = 0, SY_SIGMOID_NORMAL = 1, SY_NEG_SOFTPLUS_NORMAL = 2 };

typedef struct {
    uint64_t key;
    int64_t idx0;
    int kind;
    double std, floor_;
    int round_bf16;
    float* out;
} sy_elem_ctx;

static void sy_elem_range(void* vc, int64_t b, int64_t e) {
    const sy_elem_ctx* c = (const sy_elem_ctx*)vc;
    for (int64_t i = b; i < e; ++i) {
        const double z = sy_normal(c->key, (uint64_t)(c->idx0 + i));
        double x;
        if (c->kind == SY_NORMAL) {
            x = c->std * z;
        } else if (c->kind == SY_SIGMOID_NORMAL) {
            x = 1.0 / (1.0 + exp(-z));
        } else { /* -softplus(z), bounded below */
            const double sp = (z > 30.0) ? z : log1p(exp(z));
            x = -sp;
            if (x < c->floor_) x = c->floor_;
        }
        float f = (float)x;
        c->out[i] = c->round_bf16 ? sy_bf16_round(f) : f;
    }
}

/* Elements [idx0, idx0+n) of a flat tensor whose entries are N(0, std^2). */
SY_API void synth_normal(uint64_t seed, uint64_t tag, int64_t idx0, int64_t n, double std,
                         int round_bf16, float* out) {
    sy_elem_ctx c = {sy_key(seed, tag), idx0, SY_NORMAL, std, 0.0, round_bf16, out};
    sy_parallel(sy_elem_range, &c, n);
}

/* Elements of a tensor whose entries are sigmoid(N(0,1)). */
SY_API void synth_sigmoid_normal(uint64_t seed, uint64_t tag, int64_t idx0, int64_t n,
                                 int round_bf16, float* out) {
    sy_elem_ctx c = {sy_key(seed, tag), idx0, SY_SIGMOID_NORMAL, 1.0, 0.0, round_bf16, out};
    sy_parallel(sy_elem_range, &c, n);
}

/* Elements of a tensor whose entries are max(floor, -softplus(N(0,1))). */
SY_API void synth_neg_softplus_normal(uint64_t seed, uint64_t tag, int64_t idx0, int64_t n,
                                      double floor_, int round_bf16, float* out) {
    sy_elem_ctx c = {sy_key(seed, tag), idx0, SY_NEG_SOFTPLUS_NORMAL, 1.0, floor_, round_bf16, out};
    sy_parallel(sy_elem_range, &c, n);
}

/* ---------------- unit rows (q, k) ---------------- */

typedef struct {
    uint64_t key;
    int64_t row0;
    int d;
    int round_bf16;
    float* out;
} sy_rows_ctx;

static void sy_rows_range(void* vc, int64_t b, int64_t e) {
    const sy_rows_ctx* c = (const sy_rows_ctx*)vc;
    double buf[1024];
    for (int64_t r = b; r < e; ++r) {
        const uint64_t base = (uint64_t)(c->row0 + r) * (uint64_t)c->d;
        double ss = 0.0;
        for (int i = 0; i < c->d; ++i) {
            buf[i] = sy_normal(c->key, base + (uint64_t)i);
            ss += buf[i] * buf[i];
        }
        const double inv = 1.0 / sqrt(ss);
        for (int i = 0; i < c->d; ++i) {
            float f = (float)(buf[i] * inv);
            c->out[(size_t)r * c->d + i] = c->round_bf16 ? sy_bf16_round(f) : f;
        }
    }
}

/* Rows [row0, row0+nrows) of a [rows, d] tensor of N(0,1) vectors divided by
 * their L2 norm (one row = one token of one head).  d <= 1024. */
SY_API int synth_unit_rows(uint64_t seed, uint64_t tag, int64_t row0, int64_t nrows, int d,
                           int round_bf16, float* out) {
    if (d <= 0 || d > 1024) return -1;
    sy_rows_ctx c = {sy_key(seed, tag), row0, d, round_bf16, out};
    sy_parallel(sy_rows_range, &c, nrows);
    return 0;
}

/* n integers drawn uniformly from [lo, hi] (inclusive). */
SY_API void synth_uniform_int(uint64_t seed, uint64_t tag, int64_t n, int64_t lo, int64_t hi,
                              int64_t* out) {
    const uint64_t key = sy_key(seed, tag);
    const uint64_t span = (uint64_t)(hi - lo + 1);
    for (int64_t i = 0; i < n; ++i) {
        const double u = sy_uniform(key, (uint64_t)i);
        uint64_t off = (uint64_t)(u * (double)span);
        if (off >= span) off = span - 1;
        out[i] = lo + (int64_t)off;
    }
}

/* ---------------- encoding ---------------- */

typedef struct { const float* in; uint16_t* out; } sy_enc_ctx;

static void sy_enc_range(void* vc, int64_t b, int64_t e) {
    const sy_enc_ctx* c = (const sy_enc_ctx*)vc;
    for (int64_t i = b; i < e; ++i) c->out[i] = sy_bf16_bits(c->in[i]);
}

/* float32 -> bf16 bit patterns, round to nearest even. */
SY_API void synth_to_bf16_bits(const float* in, int64_t n, uint16_t* out) {
    sy_enc_ctx c = {in, out};
    sy_parallel(sy_enc_range, &c, n);
}
