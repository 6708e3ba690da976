/*
 * synth.c -- seeded synthetic inputs shared by the tests, the benchmark and the
 * oracle checks.  It holds none of the attention arithmetic: it only turns
 * (seed, tensor id, element index) into an N(0,1) sample rounded to bf16.
 *
 * Generator: SplitMix64 (Steele, Lea and Flood, "Fast splittable pseudorandom
 * number generators", OOPSLA 2014), in its usual form: the state advances by the
 * odd constant 0x9E3779B97F4A7C15 and each output is the state passed through
 * the variant-13 mix (xor-shift 30, multiply, xor-shift 27, multiply,
 * xor-shift 31).  Because output n is mix(state0 + (n + 1) * gamma), any element
 * can be generated on its own, so threads fill disjoint ranges and the result
 * does not depend on the thread count.
 *
 * Stream for one tensor: state0 = seed XOR tensor_id.
 * Normal samples: Box-Muller on consecutive output pairs (2p, 2p+1):
 *   u1 = (x >> 11 + 1) * 2^-53 in (0, 1],  u2 = (y >> 11) * 2^-53 in [0, 1)
 *   r = sqrt(-2 ln u1), z0 = r cos(2 pi u2) -> element 2p, z1 = r sin(2 pi u2) -> 2p+1
 * computed in double, rounded to float, then to bf16 with round-to-nearest-even.
 */
#define _GNU_SOURCE
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <unistd.h>

static const uint64_t kGamma = 0x9E3779B97F4A7C15ull;

static inline uint64_t mix64(uint64_t z)
{
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
    return z ^ (z >> 31);
}

/* n-th output (n = 0, 1, ...) of the stream that starts at state0 */
uint64_t synth_splitmix64_at(uint64_t state0, uint64_t n)
{
    return mix64(state0 + (n + 1) * kGamma);
}

static inline uint16_t float_to_bf16_rne(float f)
{
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    uint32_t lsb = (u >> 16) & 1u;
    u += 0x7FFFu + lsb;
    return (uint16_t)(u >> 16);
}

static void normal_pair(uint64_t state0, uint64_t pair, double* z0, double* z1)
{
    uint64_t x = synth_splitmix64_at(state0, 2 * pair);
    uint64_t y = synth_splitmix64_at(state0, 2 * pair + 1);
    double u1 = (double)((x >> 11) + 1) * 0x1.0p-53;
    double u2 = (double)(y >> 11) * 0x1.0p-53;
    double r = sqrt(-2.0 * log(u1));
    double th = 6.283185307179586476925286766559 * u2;
    *z0 = r * cos(th);
    *z1 = r * sin(th);
}

typedef struct {
    uint64_t state0;
    uint16_t* out16;
    float* out32;
    int64_t n;
    int64_t begin, end; /* element range */
} job_t;

static void* fill(void* arg)
{
    job_t* j = (job_t*)arg;
    int64_t e = j->begin;
    while (e < j->end) {
        uint64_t pair = (uint64_t)e >> 1;
        double z[2];
        normal_pair(j->state0, pair, &z[0], &z[1]);
        for (int t = (int)(e & 1); t < 2 && e < j->end; ++t, ++e) {
            float f = (float)z[t];
            if (j->out16)
                j->out16[e] = float_to_bf16_rne(f);
            if (j->out32)
                j->out32[e] = f;
        }
    }
    return NULL;
}

static void run(uint64_t seed, uint64_t tensor_id, uint16_t* out16, float* out32, int64_t n,
                int nthreads)
{
    if (nthreads <= 0) {
        long c = sysconf(_SC_NPROCESSORS_ONLN);
        nthreads = c > 0 ? (int)c : 1;
    }
    if ((int64_t)nthreads > n / 65536 + 1)
        nthreads = (int)(n / 65536 + 1);
    job_t* jobs = (job_t*)malloc(sizeof(job_t) * nthreads);
    pthread_t* th = (pthread_t*)malloc(sizeof(pthread_t) * nthreads);
    for (int t = 0; t < nthreads; ++t) {
        jobs[t].state0 = seed ^ tensor_id;
        jobs[t].out16 = out16;
        jobs[t].out32 = out32;
        jobs[t].n = n;
        jobs[t].begin = n * t / nthreads;
        jobs[t].end = n * (t + 1) / nthreads;
        if (nthreads == 1)
            fill(&jobs[t]);
        else
            pthread_create(&th[t], NULL, fill, &jobs[t]);
    }
    if (nthreads > 1)
        for (int t = 0; t < nthreads; ++t)
            pthread_join(th[t], NULL);
    free(jobs);
    free(th);
}

/* n bf16 samples (bit patterns) of the stream (seed, tensor_id) */
void synth_normal_bf16(uint64_t seed, uint64_t tensor_id, uint16_t* out, int64_t n, int nthreads)
{
    run(seed, tensor_id, out, NULL, n, nthreads);
}

/* the same samples before the bf16 rounding (float) */
void synth_normal_f32(uint64_t seed, uint64_t tensor_id, float* out, int64_t n, int nthreads)
{
    run(seed, tensor_id, NULL, out, n, nthreads);
}
