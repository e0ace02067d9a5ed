/*
 * Seeded synthetic inputs for the Ulysses attention path.
 *
 * This module only draws numbers; it holds none of the attention, pack or
 * unpack arithmetic.  Both the CUDA path and the fp64 oracle consume the
 * arrays it writes.
 *
 * Generator: element e of tensor `tid` under `seed` takes outputs 2e and 2e+1
 * of a SplitMix64 stream (Steele, Lea & Flood, "Fast splittable pseudorandom
 * number generators", OOPSLA 2014: state advances by the golden-gamma
 * constant, each output is the state passed through the mix64 finaliser).
 * The two outputs become uniforms u1 in (0,1] and u2 in [0,1) with 53-bit
 * resolution, and the Box-Muller transform (Box & Muller 1958) turns them
 * into one standard normal z = sqrt(-2 ln u1) cos(2 pi u2).  z is computed in
 * double, multiplied by `mul` in double, narrowed to fp32 and then rounded to
 * bf16 with round-to-nearest-even.
 *
 * The value of a logical element depends only on (seed, tid, e), with
 * e = ((b*N + t)*H + h)*D + c, so every sharding of the same logical tensor
 * holds the same numbers.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <string.h>

#define GOLDEN_GAMMA 0x9E3779B97F4A7C15ULL

static inline uint64_t mix64(uint64_t z) {
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
    return z ^ (z >> 31);
}

/* Stream seed for (seed, tid): the finaliser of a value that mixes both. */
static inline uint64_t stream_key(uint64_t seed, uint64_t tid) {
    return mix64(seed * GOLDEN_GAMMA + (tid << 1) + 1ULL);
}

/* i-th output (i >= 0) of the SplitMix64 stream that starts at `key`. */
static inline uint64_t stream_out(uint64_t key, uint64_t i) {
    return mix64(key + (i + 1ULL) * GOLDEN_GAMMA);
}

static inline uint16_t f32_to_bf16_rne(float f) {
    uint32_t u;
    memcpy(&u, &f, 4);
    u += 0x7FFFu + ((u >> 16) & 1u);
    return (uint16_t)(u >> 16);
}

static inline double normal_at(uint64_t key, uint64_t e) {
    const double two_pi = 6.283185307179586476925286766559;
    uint64_t a = stream_out(key, 2 * e);
    uint64_t b = stream_out(key, 2 * e + 1);
    double u1 = ((double)(a >> 11) + 1.0) * (1.0 / 9007199254740992.0);
    double u2 = (double)(b >> 11) * (1.0 / 9007199254740992.0);
    return sqrt(-2.0 * log(u1)) * cos(two_pi * u2);
}

uint64_t synth_stream_out(uint64_t seed, uint64_t tid, uint64_t i) {
    return stream_out(stream_key(seed, tid), i);
}

typedef struct {
    uint64_t key;
    uint64_t e0;
    int64_t count;
    double mul;
    uint16_t *out;
} job_t;

static void *normal_worker(void *arg) {
    job_t *j = (job_t *)arg;
    for (int64_t i = 0; i < j->count; ++i) {
        double z = normal_at(j->key, j->e0 + (uint64_t)i) * j->mul;
        j->out[i] = f32_to_bf16_rne((float)z);
    }
    return NULL;
}

/* Writes count bf16 normals (times mul) for logical elements e0 .. e0+count-1
 * into out[0 .. count-1], using up to nthreads threads. */
void synth_normal_bf16(uint64_t seed, uint64_t tid, uint64_t e0, int64_t count,
                       double mul, uint16_t *out, int nthreads) {
    if (count <= 0) return;
    if (nthreads < 1) nthreads = 1;
    if (nthreads > 256) nthreads = 256;
    if (count < (int64_t)1 << 16) nthreads = 1;
    uint64_t key = stream_key(seed, tid);
    pthread_t th[256];
    job_t jobs[256];
    int64_t per = (count + nthreads - 1) / nthreads;
    int started = 0;
    for (int t = 0; t < nthreads; ++t) {
        int64_t lo = (int64_t)t * per;
        int64_t hi = lo + per < count ? lo + per : count;
        if (lo >= hi) break;
        jobs[t].key = key;
        jobs[t].e0 = e0 + (uint64_t)lo;
        jobs[t].count = hi - lo;
        jobs[t].mul = mul;
        jobs[t].out = out + lo;
        if (t == 0) continue;
        if (pthread_create(&th[t], NULL, normal_worker, &jobs[t]) != 0) {
            normal_worker(&jobs[t]);
            th[t] = 0;
        }
        started = t + 1;
    }
    normal_worker(&jobs[0]);
    for (int t = 1; t < started; ++t)
        if (th[t]) pthread_join(th[t], NULL);
}

/* Double-precision normal for element e (no bf16 rounding); for tests of the
 * generator itself. */
double synth_normal_f64(uint64_t seed, uint64_t tid, uint64_t e) {
    return normal_at(stream_key(seed, tid), e);
}
