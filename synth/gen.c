/*
 * Seeded synthetic inputs for the TTT-E2E prefill loop: token streams and
 * initial weights.  This file holds no arithmetic of the method itself; it is
 * the one module that both the CUDA path and the CPU oracle draw inputs from.
 *
 * Random numbers come from SplitMix64 used as a counter-based generator:
 * value(key, i) = mix64(key + (i + 1) * GOLDEN), with mix64 the SplitMix64
 * finaliser (Steele, Lea, Flood, "Fast splittable pseudorandom number
 * generators", OOPSLA 2014).  Every tensor has its own key, so any element can
 * be regenerated on its own and the result does not depend on thread count.
 *
 * Build: gcc -O2 -fopenmp -shared -fPIC gen.c -o _gen.so -lm
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define GOLDEN 0x9E3779B97F4A7C15ULL

static inline uint64_t mix64(uint64_t z) {
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
    return z ^ (z >> 31);
}

static inline uint64_t draw(uint64_t key, uint64_t i) { return mix64(key + (i + 1) * GOLDEN); }

/* uniform double in [0, 1) with 53 random bits */
static inline double unit(uint64_t key, uint64_t i) { return (double)(draw(key, i) >> 11) * 0x1.0p-53; }

uint64_t synth_stream_key(uint64_t seed, uint64_t stream) { return mix64(seed ^ mix64(stream * GOLDEN + 0x51ED2701ULL)); }

uint64_t synth_u64(uint64_t key, uint64_t i) { return draw(key, i); }

/* n samples of N(0, std^2): Box-Muller on pairs (2j, 2j+1) of uniforms. */
void synth_normal_f32(uint64_t key, int64_t n, double std, float* out) {
    const double two_pi = 6.283185307179586476925286766559;
#pragma omp parallel for schedule(static)
    for (int64_t j = 0; j < (n + 1) / 2; ++j) {
        double u1 = unit(key, 2 * (uint64_t)j);
        double u2 = unit(key, 2 * (uint64_t)j + 1);
        double r = sqrt(-2.0 * log(1.0 - u1)); /* 1-u1 in (0, 1] */
        double z0 = r * cos(two_pi * u2), z1 = r * sin(two_pi * u2);
        out[2 * j] = (float)(std * z0);
        if (2 * j + 1 < n) out[2 * j + 1] = (float)(std * z1);
    }
}

/* Round-to-nearest-even of fp32 to bfloat16.  Writes the 16-bit pattern and,
 * optionally, the rounded value widened back to fp32.  NaN inputs are not
 * expected (generated weights are finite). */
void synth_round_bf16(const float* in, int64_t n, uint16_t* bits, float* widened) {
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) {
        uint32_t u;
        memcpy(&u, &in[i], 4);
        uint32_t lsb = (u >> 16) & 1u;
        uint32_t r = u + 0x7FFFu + lsb;
        uint16_t h = (uint16_t)(r >> 16);
        if (bits) bits[i] = h;
        if (widened) {
            uint32_t w = ((uint32_t)h) << 16;
            memcpy(&widened[i], &w, 4);
        }
    }
}

/* Token stream: iid Zipf(alpha) over ranks 1..V (rank r -> id r-1) by inverse
 * CDF, then `span`-token spans copied from earlier in the stream at random
 * distances, so that a model which adapts to the document has something to
 * recall.  Span placement: cursor p starts at `span`; before each copy it
 * advances by a gap uniform in [gap_lo, gap_hi); the copy source lies D tokens
 * back with D log-uniform in [span, p].  Returns 0, or -1 on bad arguments. */
int synth_tokens(uint64_t seed, int64_t T, int32_t V, double alpha, int32_t span, int32_t gap_lo,
                 int32_t gap_hi, int32_t* out) {
    if (T < 0 || V < 1 || span < 1 || gap_lo < 0 || gap_hi <= gap_lo) return -1;
    double* cdf = (double*)malloc(sizeof(double) * (size_t)V);
    if (!cdf) return -1;
    double acc = 0.0;
    for (int32_t r = 1; r <= V; ++r) {
        acc += pow((double)r, -alpha);
        cdf[r - 1] = acc;
    }
    for (int32_t r = 0; r < V; ++r) cdf[r] /= acc;
    const uint64_t key_tok = synth_stream_key(seed, 1);
    const uint64_t key_span = synth_stream_key(seed, 2);
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < T; ++t) {
        double u = unit(key_tok, (uint64_t)t);
        int32_t lo = 0, hi = V - 1; /* smallest r with cdf[r] > u */
        while (lo < hi) {
            int32_t mid = lo + (hi - lo) / 2;
            if (cdf[mid] > u) hi = mid; else lo = mid + 1;
        }
        out[t] = lo;
    }
    free(cdf);
    uint64_t c = 0;
    int64_t p = span;
    for (;;) {
        p += gap_lo + (int64_t)(unit(key_span, c++) * (double)(gap_hi - gap_lo));
        if (p + span > T) break;
        double lmin = log((double)span), lmax = log((double)p);
        int64_t D = (int64_t)floor(exp(lmin + unit(key_span, c++) * (lmax - lmin)));
        if (D < span) D = span;
        if (D > p) D = p;
        for (int32_t j = 0; j < span; ++j) out[p + j] = out[p - D + j];
        p += span;
    }
    return 0;
}
