/*
 * Seeded synthetic inputs for the MoE-layer forward path.
 *
 * This file holds random-number generation only: no routing, no expert
 * arithmetic, nothing of the method itself.  Both the CPU oracle and the CUDA
 * path receive the buffers written here, so neither side ever generates its
 * own inputs.
 *
 * Generator: a counter-based form of SplitMix64 (Steele, Lea and Flood,
 * "Fast splittable pseudorandom number generators", OOPSLA 2014).  Draw i of a
 * stream with key K is mix(K + (i + 1) * GAMMA), which is exactly the i-th
 * output of the sequential SplitMix64 generator seeded with K.  Because every
 * draw depends only on its counter, a buffer can be filled by any number of
 * threads and still come out bit-identical.
 *
 * Normal deviates use the Box-Muller transform (Box and Muller, 1958): draws
 * 2p and 2p+1 give the pair (u1, u2); element 2p takes the cosine branch and
 * element 2p+1 the sine branch.
 *
 * Rounding: a deviate is scaled in double, rounded to fp32 (round to nearest
 * even, by the C cast), then, for bf16 outputs, rounded to bf16 (round to
 * nearest even on the fp32 bit pattern).
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <string.h>
#include <unistd.h>

#define GAMMA 0x9E3779B97F4A7C15ULL

static uint64_t mix64(uint64_t z) {
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
    return z ^ (z >> 31);
}

/* Key of stream `stream` under `seed`: the seed and stream id are mixed so
 * that nearby (seed, stream) pairs give unrelated keys. */
uint64_t synth_stream_key(uint64_t seed, uint64_t stream) {
    return mix64(seed * GAMMA + 0x632BE59BD9B4E019ULL) ^ mix64((stream + 1) * 0xD1B54A32D192ED03ULL);
}

uint64_t synth_draw(uint64_t key, uint64_t i) { return mix64(key + (i + 1) * GAMMA); }

static double normal_at(uint64_t key, uint64_t i) {
    const uint64_t p = i >> 1;
    const uint64_t r1 = synth_draw(key, 2 * p), r2 = synth_draw(key, 2 * p + 1);
    const double u1 = (double)((r1 >> 11) + 1) * 0x1.0p-53; /* (0, 1] */
    const double u2 = (double)(r2 >> 11) * 0x1.0p-53;       /* [0, 1) */
    const double rad = sqrt(-2.0 * log(u1));
    const double ang = 6.283185307179586476925286766559 * u2;
    return (i & 1) ? rad * sin(ang) : rad * cos(ang);
}

static uint16_t f32_to_bf16_rne(float f) {
    uint32_t u;
    memcpy(&u, &f, 4);
    if ((u & 0x7F800000u) == 0x7F800000u && (u & 0x007FFFFFu)) return (uint16_t)((u >> 16) | 0x40u);
    u += 0x7FFFu + ((u >> 16) & 1u);
    return (uint16_t)(u >> 16);
}

typedef struct {
    void *out;
    uint64_t begin, end, key;
    double scale;
    int is_bf16;
} fill_job;

static void *fill_worker(void *arg) {
    fill_job *j = (fill_job *)arg;
    if (j->is_bf16) {
        uint16_t *o = (uint16_t *)j->out;
        for (uint64_t i = j->begin; i < j->end; ++i) o[i] = f32_to_bf16_rne((float)(j->scale * normal_at(j->key, i)));
    } else {
        float *o = (float *)j->out;
        for (uint64_t i = j->begin; i < j->end; ++i) o[i] = (float)(j->scale * normal_at(j->key, i));
    }
    return 0;
}

static void fill_parallel(void *out, uint64_t n, uint64_t key, double scale, int is_bf16, int nthreads) {
    enum { MAXT = 64 };
    if (nthreads <= 0) {
        long c = sysconf(_SC_NPROCESSORS_ONLN);
        nthreads = c > 0 ? (int)c : 1;
    }
    if (nthreads > MAXT) nthreads = MAXT;
    if (n < (1u << 16)) nthreads = 1;
    pthread_t th[MAXT];
    fill_job jobs[MAXT];
    for (int t = 0; t < nthreads; ++t) {
        jobs[t].out = out;
        jobs[t].begin = n * (uint64_t)t / (uint64_t)nthreads;
        jobs[t].end = n * (uint64_t)(t + 1) / (uint64_t)nthreads;
        jobs[t].key = key;
        jobs[t].scale = scale;
        jobs[t].is_bf16 = is_bf16;
    }
    int started = 0;
    for (int t = 1; t < nthreads; ++t) {
        if (pthread_create(&th[t], 0, fill_worker, &jobs[t]) != 0) break;
        started = t;
    }
    fill_worker(&jobs[0]);
    for (int t = 1; t <= started; ++t) pthread_join(th[t], 0);
    for (int t = started + 1; t < nthreads; ++t) fill_worker(&jobs[t]); /* threads that failed to start */
}

/* out[i] = bf16(fp32(scale * N_i(0,1))), i in [0, n). */
void synth_fill_bf16_normal(uint16_t *out, uint64_t n, uint64_t seed, uint64_t stream, double scale, int nthreads) {
    fill_parallel(out, n, synth_stream_key(seed, stream), scale, 1, nthreads);
}

/* out[i] = fp32(scale * N_i(0,1)), i in [0, n). */
void synth_fill_f32_normal(float *out, uint64_t n, uint64_t seed, uint64_t stream, double scale, int nthreads) {
    fill_parallel(out, n, synth_stream_key(seed, stream), scale, 0, nthreads);
}

/* A uniformly random permutation of 1..n written to rank[0..n), by the
 * Fisher-Yates shuffle driven by the stream's draws (draw d picks the swap
 * partner of position n-1-d by reduction modulo the remaining length). */
void synth_rank_permutation(int32_t *rank, int32_t n, uint64_t seed, uint64_t stream) {
    const uint64_t key = synth_stream_key(seed, stream);
    for (int32_t i = 0; i < n; ++i) rank[i] = i + 1;
    for (int32_t i = n - 1, d = 0; i > 0; --i, ++d) {
        const int32_t j = (int32_t)(synth_draw(key, (uint64_t)d) % (uint64_t)(i + 1));
        const int32_t t = rank[i];
        rank[i] = rank[j];
        rank[j] = t;
    }
}
