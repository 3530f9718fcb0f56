/*
 * Seeded synthetic inputs for the ExpertsInt8 mixture-of-experts layer.
 *
 * This module is shared by the fp64 CPU oracle and by the CUDA path, and by
 * nothing else.  It holds none of the layer's arithmetic: it only draws normal
 * variates, so that both sides see exactly the same bf16 / fp32 inputs.
 *
 * Generator (counter based, so any slice of any tensor can be drawn alone):
 *   - SplitMix64 (Steele, Lea and Flood, "Fast splittable pseudorandom number
 *     generators", OOPSLA 2014): the n-th output of a stream whose state
 *     starts at `key` is mix(key + (n + 1) * GAMMA), GAMMA = 0x9E3779B97F4A7C15,
 *     mix = the variant-13 64-bit finalizer given there.
 *   - Stream key for (seed, stream, attempt):
 *       key = out0(out0(out0(seed) ^ stream) ^ attempt), out0(s) = mix(s + GAMMA).
 *   - Element i of a stream uses the outputs 2*(i/2) and 2*(i/2)+1 as two
 *     uniforms u1 = ((b1 >> 11) + 1) * 2^-53 in (0, 1], u2 = (b2 >> 11) * 2^-53
 *     in [0, 1), and the Box-Muller transform (Box and Muller, Ann. Math.
 *     Statist. 1958): r = sqrt(-2 ln u1), z = r cos(2 pi u2) for even i,
 *     z = r sin(2 pi u2) for odd i, all in IEEE double with the C library's
 *     log / sqrt / cos / sin.
 *   - The value is stddev * z in double, rounded to nearest-even once, either
 *     to bf16 (returned as its 16-bit pattern) or to fp32.
 *
 * Build: gcc -O2 -shared -fPIC -pthread synth.c -lm (no -ffast-math).
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <string.h>
#include <unistd.h>

#define GAMMA 0x9E3779B97F4A7C15ULL

static inline uint64_t mix64(uint64_t z) {
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
    return z ^ (z >> 31);
}

static inline uint64_t out_n(uint64_t key, uint64_t n) { return mix64(key + (n + 1) * GAMMA); }

uint64_t synth_stream_key(uint64_t seed, uint64_t stream, uint64_t attempt) {
    uint64_t k = out_n(seed, 0);
    k = out_n(k ^ stream, 0);
    k = out_n(k ^ attempt, 0);
    return k;
}

/* The raw 64-bit output n of a stream (exported so tests can pin the mixer). */
uint64_t synth_raw(uint64_t key, uint64_t n) { return out_n(key, n); }

static inline double normal_at(uint64_t key, uint64_t i) {
    const uint64_t j = i >> 1;
    const uint64_t b1 = out_n(key, 2 * j), b2 = out_n(key, 2 * j + 1);
    const double u1 = (double)((b1 >> 11) + 1) * 0x1.0p-53;
    const double u2 = (double)(b2 >> 11) * 0x1.0p-53;
    const double r = sqrt(-2.0 * log(u1));
    const double th = 6.283185307179586476925286766559 * u2;
    return (i & 1) ? r * sin(th) : r * cos(th);
}

/* Round a finite double to the nearest bf16 (ties to even), returned as bits. */
static inline uint16_t bf16_rne_from_double(double v) {
    uint64_t b;
    memcpy(&b, &v, 8);
    const uint64_t sign = b >> 63;
    int64_t e = (int64_t)((b >> 52) & 0x7FF);
    const uint64_t mant = b & ((1ULL << 52) - 1);
    if (e == 0) return (uint16_t)(sign << 15); /* zero or double subnormal */
    uint64_t m7 = mant >> 45, rem = mant & ((1ULL << 45) - 1);
    const uint64_t half = 1ULL << 44;
    if (rem > half || (rem == half && (m7 & 1))) m7++;
    if (m7 == 128) { m7 = 0; e++; }
    int64_t eb = e - 1023 + 127;
    if (eb <= 0) return (uint16_t)(sign << 15); /* below bf16's normal range: flush */
    if (eb >= 255) return (uint16_t)((sign << 15) | 0x7F80); /* overflow to inf */
    return (uint16_t)((sign << 15) | ((uint64_t)eb << 7) | m7);
}

typedef struct {
    uint64_t key, start, count;
    double stddev;
    void* out;
    int is_bf16;
} job_t;

static void* run_job(void* p) {
    job_t* j = (job_t*)p;
    if (j->is_bf16) {
        uint16_t* o = (uint16_t*)j->out;
        for (uint64_t t = 0; t < j->count; ++t) o[t] = bf16_rne_from_double(j->stddev * normal_at(j->key, j->start + t));
    } else {
        float* o = (float*)j->out;
        for (uint64_t t = 0; t < j->count; ++t) o[t] = (float)(j->stddev * normal_at(j->key, j->start + t));
    }
    return NULL;
}

static void run(uint64_t key, uint64_t start, uint64_t count, double stddev, void* out, int is_bf16, int threads) {
    if (threads <= 0) {
        long n = sysconf(_SC_NPROCESSORS_ONLN);
        threads = n > 0 ? (int)n : 1;
    }
    if (threads > 256) threads = 256;
    if ((uint64_t)threads > count / 65536 + 1) threads = (int)(count / 65536 + 1);
    job_t jobs[256];
    pthread_t tids[256];
    const size_t esz = is_bf16 ? 2 : 4;
    uint64_t per = (count + threads - 1) / threads;
    for (int t = 0; t < threads; ++t) {
        uint64_t b = per * t, e = b + per;
        if (b > count) b = count;
        if (e > count) e = count;
        jobs[t] = (job_t){key, start + b, e - b, stddev, (char*)out + b * esz, is_bf16};
    }
    for (int t = 1; t < threads; ++t) pthread_create(&tids[t], NULL, run_job, &jobs[t]);
    run_job(&jobs[0]);
    for (int t = 1; t < threads; ++t) pthread_join(tids[t], NULL);
}

void synth_normal_bf16(uint64_t seed, uint64_t stream, uint64_t attempt, uint64_t start, uint64_t count,
                       double stddev, uint16_t* out, int threads) {
    run(synth_stream_key(seed, stream, attempt), start, count, stddev, out, 1, threads);
}

void synth_normal_f32(uint64_t seed, uint64_t stream, uint64_t attempt, uint64_t start, uint64_t count,
                      double stddev, float* out, int threads) {
    run(synth_stream_key(seed, stream, attempt), start, count, stddev, out, 0, threads);
}
