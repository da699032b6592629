/*
 * Seeded synthetic inputs shared by the CUDA path's tests/bench and by the
 * oracle.  This file holds no attention arithmetic: it only turns a seed and
 * an element index into a standard-normal sample.
 *
 * Generator: counter-based SplitMix64 (Steele, Lea & Flood, "Fast splittable
 * pseudorandom number generators", OOPSLA 2014; finaliser constants as
 * published there and in Vigna's public-domain splitmix64.c).  Element n of
 * stream `seed` uses the 64-bit outputs number 2n and 2n+1 of a SplitMix64
 * sequence started at `seed`, mapped to two uniforms in (0,1), and one
 * Box-Muller transform (Box & Muller 1958): z = sqrt(-2 ln u1) cos(2 pi u2).
 * Because every element is a pure function of (seed, n), the array can be
 * filled by any number of threads in any order with identical results.
 *
 * Outputs: float32 (round-to-nearest from the double sample), bfloat16
 * bit patterns (round-to-nearest-even from that float32), or OFP8 E4M3 bit
 * patterns (round-to-nearest-even from that float32, saturating at +-448).
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>

#define GOLDEN 0x9e3779b97f4a7c15ULL

static inline uint64_t mix64(uint64_t z) {
    z = (z ^ (z >> 30)) * 0xbf58476d1ce4e5b9ULL;
    z = (z ^ (z >> 27)) * 0x94d049bb133111ebULL;
    return z ^ (z >> 31);
}

/* k-th output (k >= 0) of a SplitMix64 generator whose state starts at seed. */
static inline uint64_t splitmix_at(uint64_t seed, uint64_t k) {
    return mix64(seed + (k + 1) * GOLDEN);
}

static inline double to_unit_open(uint64_t x) {
    /* 53 high bits, centred in their cell: strictly inside (0, 1). */
    return ((double)(x >> 11) + 0.5) * (1.0 / 9007199254740992.0);
}

static inline double normal_at(uint64_t seed, uint64_t n) {
    const double two_pi = 6.283185307179586476925286766559;
    double u1 = to_unit_open(splitmix_at(seed, 2 * n));
    double u2 = to_unit_open(splitmix_at(seed, 2 * n + 1));
    return sqrt(-2.0 * log(u1)) * cos(two_pi * u2);
}

static inline uint16_t f32_to_bf16_rne(float f) {
    union { float f; uint32_t u; } b;
    b.f = f;
    uint32_t u = b.u;
    if ((u & 0x7f800000u) == 0x7f800000u && (u & 0x007fffffu)) /* NaN: keep quiet NaN */
        return (uint16_t)((u >> 16) | 0x40u);
    uint32_t lsb = (u >> 16) & 1u;
    u += 0x7fffu + lsb;
    return (uint16_t)(u >> 16);
}

/* OFP8 E4M3 (1 sign, 4 exponent bits with bias 7, 3 mantissa bits; no
 * infinities; largest finite 448 = 1.75 * 2^8; subnormals m * 2^-9) from a
 * float32, rounding to nearest even and saturating out-of-range values. */
static inline uint8_t f32_to_e4m3_rne(float f) {
    const uint8_t sign = signbit(f) ? 0x80u : 0u;
    const double a = fabs((double)f);
    if (a != a) return 0x7fu;                 /* NaN */
    if (a >= 448.0) return sign | 0x7eu;      /* saturate */
    if (a < 0.015625) {                       /* below 2^-6: subnormal grid of 2^-9 */
        const double q = rint(a * 512.0);     /* 0..8; 8 is the smallest normal */
        return sign | (uint8_t)q;
    }
    int e;
    const double m = frexp(a, &e);           /* a = m * 2^e, m in [0.5, 1) */
    int ex = e - 1;                          /* a = (2m) * 2^ex, 2m in [1, 2) */
    double q = rint((2.0 * m - 1.0) * 8.0);  /* 0..8 */
    if (q == 8.0) { q = 0.0; ++ex; }
    const int code = ((ex + 7) << 3) | (int)q;
    return sign | (uint8_t)(code > 0x7e ? 0x7e : code);
}

typedef struct {
    uint64_t seed;
    uint64_t begin, end;
    float scale;
    int kind;      /* 0 = float32, 1 = bf16 bits, 2 = E4M3 bits */
    void* out;
} job_t;

static void* run_job(void* p) {
    job_t* j = (job_t*)p;
    if (j->kind == 0) {
        float* o = (float*)j->out;
        for (uint64_t n = j->begin; n < j->end; ++n)
            o[n] = (float)(normal_at(j->seed, n) * j->scale);
    } else if (j->kind == 1) {
        uint16_t* o = (uint16_t*)j->out;
        for (uint64_t n = j->begin; n < j->end; ++n)
            o[n] = f32_to_bf16_rne((float)(normal_at(j->seed, n) * j->scale));
    } else {
        uint8_t* o = (uint8_t*)j->out;
        for (uint64_t n = j->begin; n < j->end; ++n)
            o[n] = f32_to_e4m3_rne((float)(normal_at(j->seed, n) * j->scale));
    }
    return NULL;
}

static int fill(uint64_t seed, uint64_t count, float scale, int kind, void* out, int nthreads) {
    if (!out && count) return -1;
    if (nthreads < 1) nthreads = 1;
    if (nthreads > 256) nthreads = 256;
    if ((uint64_t)nthreads > count / 65536 + 1) nthreads = (int)(count / 65536 + 1);
    pthread_t th[256];
    job_t jobs[256];
    uint64_t per = (count + (uint64_t)nthreads - 1) / (uint64_t)nthreads;
    for (int t = 0; t < nthreads; ++t) {
        jobs[t].seed = seed;
        jobs[t].begin = per * (uint64_t)t < count ? per * (uint64_t)t : count;
        jobs[t].end = per * (uint64_t)(t + 1) < count ? per * (uint64_t)(t + 1) : count;
        jobs[t].scale = scale;
        jobs[t].kind = kind;
        jobs[t].out = out;
    }
    for (int t = 1; t < nthreads; ++t) {
        if (pthread_create(&th[t], NULL, run_job, &jobs[t]) != 0) {
            run_job(&jobs[t]); /* could not start a thread: do the slice here */
            th[t] = 0;
        }
    }
    run_job(&jobs[0]);
    for (int t = 1; t < nthreads; ++t)
        if (th[t]) pthread_join(th[t], NULL);
    return 0;
}

/* Fill out[0..count) with N(0, scale^2) samples as float32. Returns 0 on success. */
int na_gen_normal_f32(uint64_t seed, uint64_t count, float scale, float* out, int nthreads) {
    return fill(seed, count, scale, 0, out, nthreads);
}

/* Same samples, rounded to bfloat16 (RNE), written as raw 16-bit patterns. */
int na_gen_normal_bf16(uint64_t seed, uint64_t count, float scale, uint16_t* out, int nthreads) {
    return fill(seed, count, scale, 1, out, nthreads);
}

/* Same samples, rounded to OFP8 E4M3 (RNE, saturating at +-448), raw bytes. */
int na_gen_normal_e4m3(uint64_t seed, uint64_t count, float scale, uint8_t* out, int nthreads) {
    return fill(seed, count, scale, 2, out, nthreads);
}

/* E4M3 rounding of arbitrary float32 values (the same routine), for tests. */
void na_gen_round_e4m3(const float* in, uint64_t count, uint8_t* out) {
    for (uint64_t n = 0; n < count; ++n) out[n] = f32_to_e4m3_rne(in[n]);
}

/* Single raw SplitMix64 output, exposed so tests can check the published sequence. */
uint64_t na_gen_splitmix64_at(uint64_t seed, uint64_t k) { return splitmix_at(seed, k); }
