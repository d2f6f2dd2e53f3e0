/*
 * Seeded synthetic-input generator shared by the CUDA path's tests/bench and
 * by the CPU oracle's tests.  It draws random numbers and rounds them to bf16;
 * it holds none of the attention layer's arithmetic.
 *
 * Generator: SplitMix64 (Steele, Lea & Flood, "Fast splittable pseudorandom
 * number generators", OOPSLA 2014) seeds xoshiro256** (Blackman & Vigna,
 * "Scrambled linear pseudorandom number generators", 2018); normals come from
 * the Box-Muller transform (Box & Muller, 1958).  All three are written here
 * from their published definitions.
 *
 * Every tensor is a "stream" of values in token-major order.  A stream is cut
 * into chunks of GEN_CHUNK values; chunk c of stream s of seed S draws from a
 * xoshiro256** state that SplitMix64 derives from (S, s, c).  The output is
 * therefore the same for any thread count.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>
#include <pthread.h>

#define GEN_CHUNK 65536u

static uint64_t splitmix64_next(uint64_t *x) {
    uint64_t z = (*x += 0x9E3779B97F4A7C15ull);
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
    return z ^ (z >> 31);
}

static inline uint64_t rotl64(uint64_t v, int k) { return (v << k) | (v >> (64 - k)); }

typedef struct { uint64_t s[4]; } xoshiro256;

static uint64_t xoshiro_next(xoshiro256 *g) {
    uint64_t *s = g->s;
    const uint64_t out = rotl64(s[1] * 5u, 7) * 9u;
    const uint64_t t = s[1] << 17;
    s[2] ^= s[0];
    s[3] ^= s[1];
    s[1] ^= s[2];
    s[0] ^= s[3];
    s[2] ^= t;
    s[3] = rotl64(s[3], 45);
    return out;
}

static void xoshiro_seed(xoshiro256 *g, uint64_t seed, uint64_t stream, uint64_t chunk) {
    uint64_t x = seed;
    /* fold stream and chunk ids into the SplitMix64 seed, each through its own
       SplitMix64 step so that nearby ids land far apart */
    uint64_t a = stream + 0x1234567ull;
    uint64_t b = chunk + 0x89ABCDEFull;
    x ^= splitmix64_next(&a);
    x ^= rotl64(splitmix64_next(&b), 17);
    for (int i = 0; i < 4; ++i) g->s[i] = splitmix64_next(&x);
}

/* uniform in (0, 1]: 53 random bits, never 0 so that log() is finite */
static inline double uniform01(xoshiro256 *g) {
    return ((double)(xoshiro_next(g) >> 11) + 1.0) * (1.0 / 9007199254740992.0);
}

/* float -> bf16 bits, round to nearest even (NaN -> quiet NaN) */
static inline uint16_t f32_to_bf16_rne(float f) {
    uint32_t u;
    memcpy(&u, &f, 4);
    if ((u & 0x7F800000u) == 0x7F800000u && (u & 0x007FFFFFu)) return (uint16_t)((u >> 16) | 0x40u);
    u += 0x7FFFu + ((u >> 16) & 1u);
    return (uint16_t)(u >> 16);
}

/* kind: 0 = scale * N(0,1); 1 = 1/(1+exp(-N(0,1))) (a value in (0,1));
         2 = scale * N(0,1) as double (no rounding) */
typedef struct {
    uint64_t seed, stream, count;
    double scale;
    int kind;
    void *out;
    uint64_t c0, c1; /* chunk range */
} job_t;

static void fill_chunk(const job_t *j, uint64_t chunk) {
    xoshiro256 g;
    xoshiro_seed(&g, j->seed, j->stream, chunk);
    uint64_t i0 = chunk * GEN_CHUNK;
    uint64_t i1 = i0 + GEN_CHUNK;
    if (i1 > j->count) i1 = j->count;
    const double two_pi = 6.283185307179586476925286766559;
    for (uint64_t i = i0; i < i1; i += 2) {
        double u1 = uniform01(&g), u2 = uniform01(&g);
        double rad = sqrt(-2.0 * log(u1));
        double z[2] = {rad * cos(two_pi * u2), rad * sin(two_pi * u2)};
        for (int h = 0; h < 2 && i + h < i1; ++h) {
            double val = z[h];
            if (j->kind == 1) val = 1.0 / (1.0 + exp(-val));
            else val *= j->scale;
            if (j->kind == 2) ((double *)j->out)[i + h] = val;
            else ((uint16_t *)j->out)[i + h] = f32_to_bf16_rne((float)val);
        }
    }
}

static void *worker(void *arg) {
    const job_t *j = (const job_t *)arg;
    for (uint64_t c = j->c0; c < j->c1; ++c) fill_chunk(j, c);
    return 0;
}

static int run(uint64_t seed, uint64_t stream, uint64_t count, double scale, int kind, void *out, int nthreads) {
    uint64_t nchunks = (count + GEN_CHUNK - 1) / GEN_CHUNK;
    if (nthreads < 1) nthreads = 1;
    if (nthreads > 256) nthreads = 256;
    if ((uint64_t)nthreads > nchunks) nthreads = (int)(nchunks ? nchunks : 1);
    pthread_t th[256];
    job_t jobs[256];
    for (int t = 0; t < nthreads; ++t) {
        jobs[t].seed = seed; jobs[t].stream = stream; jobs[t].count = count;
        jobs[t].scale = scale; jobs[t].kind = kind; jobs[t].out = out;
        jobs[t].c0 = nchunks * (uint64_t)t / (uint64_t)nthreads;
        jobs[t].c1 = nchunks * (uint64_t)(t + 1) / (uint64_t)nthreads;
    }
    int started = 0;
    for (int t = 1; t < nthreads; ++t) {
        if (pthread_create(&th[t], 0, worker, &jobs[t]) != 0) break;
        started = t;
    }
    worker(&jobs[0]);
    for (int t = 1; t <= started; ++t) pthread_join(th[t], 0);
    /* any job whose thread failed to start runs here */
    for (int t = started + 1; t < nthreads; ++t) worker(&jobs[t]);
    return 0;
}

/* count values of scale*N(0,1), rounded to bf16, into out (uint16 bits). */
int nsa_gen_normal_bf16(uint64_t seed, uint64_t stream, uint64_t count, double scale, uint16_t *out, int nthreads) {
    return run(seed, stream, count, scale, 0, out, nthreads);
}

/* count values of sigmoid(N(0,1)) rounded to bf16: gate values in (0,1). */
int nsa_gen_sigmoid_normal_bf16(uint64_t seed, uint64_t stream, uint64_t count, uint16_t *out, int nthreads) {
    return run(seed, stream, count, 1.0, 1, out, nthreads);
}

/* count values of scale*N(0,1) as doubles (used for geometric noise). */
int nsa_gen_normal_f64(uint64_t seed, uint64_t stream, uint64_t count, double scale, double *out, int nthreads) {
    return run(seed, stream, count, scale, 2, out, nthreads);
}

/* raw xoshiro256** outputs of (seed, stream), for the generator's own tests */
int nsa_gen_raw_u64(uint64_t seed, uint64_t stream, uint64_t chunk, uint64_t count, uint64_t *out) {
    xoshiro256 g;
    xoshiro_seed(&g, seed, stream, chunk);
    for (uint64_t i = 0; i < count; ++i) out[i] = xoshiro_next(&g);
    return 0;
}

/* first outputs of SplitMix64 from a given state (generator self-test) */
int nsa_gen_splitmix64(uint64_t state, uint64_t count, uint64_t *out) {
    for (uint64_t i = 0; i < count; ++i) out[i] = splitmix64_next(&state);
    return 0;
}

/* xoshiro256** from an explicit state (generator self-test) */
int nsa_gen_xoshiro_from_state(const uint64_t *state4, uint64_t count, uint64_t *out) {
    xoshiro256 g;
    memcpy(g.s, state4, sizeof g.s);
    for (uint64_t i = 0; i < count; ++i) out[i] = xoshiro_next(&g);
    return 0;
}
