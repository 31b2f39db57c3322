/*
 * Seeded synthetic inputs for the Wan full self-attention workloads.
 *
 * This file holds no arithmetic of the attention method.  It only turns
 * (seed, stream, index) into numbers, so that the CUDA path and the CPU
 * oracle read the very same bytes.
 *
 * Generator (counter based, no state carried between calls):
 *   mix(z)            = SplitMix64 finaliser (Steele, Lea, Flood,
 *                       "Fast splittable pseudorandom number generators",
 *                       OOPSLA 2014): z ^= z>>30; z *= 0xBF58476D1CE4E5B9;
 *                       z ^= z>>27; z *= 0x94D049BB133111EB; z ^= z>>31.
 *   key(seed, stream) = mix(mix(seed + G) ^ (stream * 0xD1B54A32D192ED03 + G)),
 *                       G = 0x9E3779B97F4A7C15.
 *   draw(key, n)      = mix(key + (n + 1) * G)       (SplitMix64's n-th output)
 *   uniform01(x)      = (x >> 11) * 2^-53            in [0, 1)
 *   normal(i)         = sqrt(-2 ln u1) * cos(2 pi u2) (Box-Muller, fp64) with
 *                       u1 = 1 - uniform01(draw(key, 2i))   in (0, 1]
 *                       u2 = uniform01(draw(key, 2i + 1))
 *   bf16(i)           = fp64 -> fp32 (round to nearest even) -> bf16 (round
 *                       to nearest even), stored as its 16 bit pattern.
 *
 * Build: gcc -O2 -fPIC -shared -pthread synth.c -o libsynth.so -lm
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <string.h>

#define SYN_G 0x9E3779B97F4A7C15ULL

static inline uint64_t syn_mix(uint64_t z) {
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
    return z ^ (z >> 31);
}

uint64_t synth_key(uint64_t seed, uint64_t stream) {
    return syn_mix(syn_mix(seed + SYN_G) ^ (stream * 0xD1B54A32D192ED03ULL + SYN_G));
}

static inline uint64_t syn_draw(uint64_t key, uint64_t n) {
    return syn_mix(key + (n + 1) * SYN_G);
}

static inline double syn_u01(uint64_t x) {
    return (double)(x >> 11) * (1.0 / 9007199254740992.0);
}

static inline double syn_normal(uint64_t key, uint64_t i) {
    const double two_pi = 6.283185307179586476925286766559;
    double u1 = 1.0 - syn_u01(syn_draw(key, 2 * i));
    double u2 = syn_u01(syn_draw(key, 2 * i + 1));
    return sqrt(-2.0 * log(u1)) * cos(two_pi * u2);
}

static inline uint16_t syn_bf16_bits(double x) {
    float f = (float)x;                 /* round to nearest even */
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    u += 0x7FFFu + ((u >> 16) & 1u);    /* round to nearest even; no NaN reaches here */
    return (uint16_t)(u >> 16);
}

typedef struct {
    uint64_t key, first, count;
    double mul;
    uint16_t *out_bf16;
    double *out_f64;
} syn_job;

static void *syn_worker(void *arg) {
    syn_job *j = (syn_job *)arg;
    for (uint64_t t = 0; t < j->count; ++t) {
        double z = syn_normal(j->key, j->first + t) * j->mul;
        if (j->out_bf16) j->out_bf16[t] = syn_bf16_bits(z);
        if (j->out_f64) j->out_f64[t] = z;
    }
    return 0;
}

static void syn_run(uint64_t key, uint64_t first, uint64_t n, double mul,
                    uint16_t *out_bf16, double *out_f64, int nthreads) {
    if (nthreads < 1) nthreads = 1;
    if (nthreads > 256) nthreads = 256;
    if ((uint64_t)nthreads > n / 4096 + 1) nthreads = (int)(n / 4096 + 1);
    pthread_t th[256];
    syn_job jobs[256];
    uint64_t per = (n + (uint64_t)nthreads - 1) / (uint64_t)nthreads;
    int started = 0;
    for (int t = 0; t < nthreads; ++t) {
        uint64_t lo = (uint64_t)t * per;
        if (lo >= n) break;
        uint64_t hi = lo + per < n ? lo + per : n;
        jobs[t].key = key;
        jobs[t].first = first + lo;
        jobs[t].count = hi - lo;
        jobs[t].mul = mul;
        jobs[t].out_bf16 = out_bf16 ? out_bf16 + lo : 0;
        jobs[t].out_f64 = out_f64 ? out_f64 + lo : 0;
        if (pthread_create(&th[t], 0, syn_worker, &jobs[t]) != 0) {
            syn_worker(&jobs[t]);   /* run inline if a thread cannot start */
            th[t] = 0;
        }
        started = t + 1;
    }
    for (int t = 0; t < started; ++t)
        if (th[t]) pthread_join(th[t], 0);
}

/* n standard normals (elements first .. first+n-1 of the stream), as bf16 bits. */
void synth_normal_bf16(uint64_t seed, uint64_t stream, uint64_t first, uint64_t n,
                       uint16_t *out, int nthreads) {
    syn_run(synth_key(seed, stream), first, n, 1.0, out, 0, nthreads);
}

/* The same normals before any rounding (fp64), for testing the generator. */
void synth_normal_f64(uint64_t seed, uint64_t stream, uint64_t first, uint64_t n,
                      double *out, int nthreads) {
    syn_run(synth_key(seed, stream), first, n, 1.0, 0, out, nthreads);
}

/* n uniforms in [0,1): uniform01(draw(key, first + t)). */
void synth_uniform_f64(uint64_t seed, uint64_t stream, uint64_t first, uint64_t n,
                       double *out) {
    uint64_t key = synth_key(seed, stream);
    for (uint64_t t = 0; t < n; ++t) out[t] = syn_u01(syn_draw(key, first + t));
}
