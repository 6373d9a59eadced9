/*
 * Seeded synthetic inputs for the indirect expert matmul workloads.
 *
 * This file produces INPUTS only: Q8_0 weight blocks, activations and routing
 * ids.  It contains none of the arithmetic of the operator itself (no row-id
 * pass, no dequantisation, no dot product), so that both the CPU oracle and the
 * GPU library can be fed the very same bytes without sharing any method code.
 *
 * Random numbers come from a counter-based generator: the i-th output of a
 * splitmix64 stream (Steele, Lea, Flood, "Fast splittable pseudorandom number
 * generators", OOPSLA 2014) whose seed is derived from (seed, tensor id).
 * Every element is a pure function of (seed, tensor id, element index), so the
 * result does not depend on the thread count or on how a batch is sharded.
 *
 * Q8_0 block layout (the de-facto GGUF layout; the pages name the type but do
 * not print it): 34 bytes per 32 weights along a row, an IEEE fp16 scale d
 * first (little endian), then 32 signed int8 values q; the weight is d*q.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

#define GOLDEN_GAMMA 0x9E3779B97F4A7C15ULL

static inline uint64_t mix64(uint64_t z) {
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
    return z ^ (z >> 31);
}

/* Stream key of a tensor: a splitmix64 output of the seed, salted by the id. */
static inline uint64_t stream_key(uint64_t seed, uint64_t tensor) {
    return mix64(mix64(seed + GOLDEN_GAMMA) ^ (tensor * 0xD1B54A32D192ED03ULL));
}

/* i-th output of the splitmix64 stream started at `key`. */
static inline uint64_t draw(uint64_t key, uint64_t i) {
    return mix64(key + (i + 1) * GOLDEN_GAMMA);
}

/* Uniform double in [0, 1) with 53 random bits. */
static inline double unif01(uint64_t r) { return (double)(r >> 11) * 0x1.0p-53; }

/* Uniform double in (0, 1): never 0, never 1. */
static inline double unif_open(uint64_t r) { return ((double)(r >> 11) + 0.5) * 0x1.0p-53; }

/* Standard normal by Box-Muller (cosine branch) from draws 2i and 2i+1. */
static inline double normal(uint64_t key, uint64_t i) {
    double u1 = ((double)(draw(key, 2 * i) >> 11) + 1.0) * 0x1.0p-53; /* (0,1] */
    double u2 = unif01(draw(key, 2 * i + 1));
    return sqrt(-2.0 * log(u1)) * cos(6.283185307179586476925286766559 * u2);
}

/* IEEE binary16 of a double, round to nearest even (finite inputs). */
static uint16_t f64_to_f16(double v) {
    uint16_t sign = signbit(v) ? 0x8000 : 0;
    double a = fabs(v);
    if (isnan(a)) return 0x7e00;
    if (a >= 65520.0) return sign | 0x7c00;
    if (a < 0x1.0p-14) { /* subnormal: integer multiples of 2^-24 */
        double r = nearbyint(a * 0x1.0p24);
        return sign | (uint16_t)r; /* r == 1024 is the smallest normal */
    }
    int e;
    double f = frexp(a, &e);               /* a = f * 2^e, f in [0.5, 1) */
    double r = nearbyint(f * 2048.0);      /* 11 significant bits */
    int ex = e - 1;
    if (r == 2048.0) { r = 1024.0; ex += 1; }
    if (ex > 15) return sign | 0x7c00;
    return sign | (uint16_t)((ex + 15) << 10) | (uint16_t)((int)r - 1024);
}

/* bfloat16 of a float, round to nearest even. */
static uint16_t f32_to_bf16(float f) {
    uint32_t u;
    memcpy(&u, &f, 4);
    if ((u & 0x7fffffffu) > 0x7f800000u) return 0x7fc0;
    u += 0x7fffu + ((u >> 16) & 1u);
    return (uint16_t)(u >> 16);
}

/*
 * Q8_0 weights of a stacked matrix [n_rows][n_in], n_rows = n_experts*n_out.
 * Rows [row0, row0 + n_rows_here) are written to `blocks` (34 bytes per
 * 32 weights).  q ~ U{-127..127}, d = fp16(U[d_lo, d_hi)).
 */
void wl_fill_q8_0(uint8_t *blocks, int64_t row0, int64_t n_rows_here, int64_t n_in,
                  uint64_t seed, uint64_t tensor, double d_lo, double d_hi) {
    const uint64_t kq = stream_key(seed, 2 * tensor);
    const uint64_t kd = stream_key(seed, 2 * tensor + 1);
    const int64_t nb = n_in / 32;
#pragma omp parallel for schedule(static)
    for (int64_t rr = 0; rr < n_rows_here; ++rr) {
        const int64_t row = row0 + rr;
        uint8_t *dst = blocks + rr * nb * 34;
        for (int64_t b = 0; b < nb; ++b) {
            double u = unif01(draw(kd, (uint64_t)(row * nb + b)));
            uint16_t d = f64_to_f16(d_lo + (d_hi - d_lo) * u);
            dst[b * 34 + 0] = (uint8_t)(d & 0xff);
            dst[b * 34 + 1] = (uint8_t)(d >> 8);
            for (int j = 0; j < 32; ++j) {
                uint64_t g = (uint64_t)(row * n_in + b * 32 + j);
                int q = (int)((draw(kq, g) >> 32) % 255u) - 127;
                dst[b * 34 + 2 + j] = (uint8_t)(int8_t)q;
            }
        }
    }
}

/*
 * MXFP4 blocks (the OCP microscaling FP4 type, E2M1 elements sharing one E8M0
 * scale per 32; the pages name "MXFP4" among the weight types of their
 * benchmarks but do not print its bytes): 17 bytes per 32 weights along a
 * row, the scale byte first, then 16 bytes of 4-bit element codes.  Only
 * random bytes are drawn here: the scale byte uniform in [x_lo, x_hi], each
 * 4-bit code uniform in [0, 15].  How a code and a scale give a weight is the
 * consumer's business.
 */
void wl_fill_mxfp4(uint8_t *blocks, int64_t row0, int64_t n_rows_here, int64_t n_in,
                   uint64_t seed, uint64_t tensor, int x_lo, int x_hi) {
    const uint64_t kq = stream_key(seed, 2 * tensor);
    const uint64_t kx = stream_key(seed, 2 * tensor + 1);
    const int64_t nb = n_in / 32;
    const uint64_t span = (uint64_t)(x_hi - x_lo + 1);
#pragma omp parallel for schedule(static)
    for (int64_t rr = 0; rr < n_rows_here; ++rr) {
        const int64_t row = row0 + rr;
        uint8_t *dst = blocks + rr * nb * 17;
        for (int64_t b = 0; b < nb; ++b) {
            dst[b * 17] = (uint8_t)(x_lo + (int)((draw(kx, (uint64_t)(row * nb + b)) >> 32) % span));
            for (int j = 0; j < 16; ++j) {
                uint64_t g = (uint64_t)(row * (n_in / 2) + b * 16 + j);
                dst[b * 17 + 1 + j] = (uint8_t)(draw(kq, g) >> 56);
            }
        }
    }
}

/* N(0,1) samples i0 .. i0+n-1 of a tensor, stored as float. */
void wl_fill_normal_f32(float *out, int64_t i0, int64_t n, uint64_t seed, uint64_t tensor) {
    const uint64_t key = stream_key(seed, tensor);
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) out[i] = (float)normal(key, (uint64_t)(i0 + i));
}

/* N(0,1) samples i0 .. i0+n-1 of a tensor, stored as bf16 of the float value. */
void wl_fill_normal_bf16(uint16_t *out, int64_t i0, int64_t n, uint64_t seed, uint64_t tensor) {
    const uint64_t key = stream_key(seed, tensor);
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) out[i] = f32_to_bf16((float)normal(key, (uint64_t)(i0 + i)));
}

/* U[lo, hi) samples i0 .. i0+n-1 of a tensor, stored as float. */
void wl_fill_uniform_f32(float *out, int64_t i0, int64_t n, double lo, double hi, uint64_t seed, uint64_t tensor) {
    const uint64_t key = stream_key(seed, tensor);
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) out[i] = (float)(lo + (hi - lo) * unif01(draw(key, (uint64_t)(i0 + i))));
}

/* N(0,1) samples stored as fp16 (for fp16-activation cases). */
void wl_fill_normal_f16(uint16_t *out, int64_t i0, int64_t n, uint64_t seed, uint64_t tensor) {
    const uint64_t key = stream_key(seed, tensor);
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) out[i] = f64_to_f16((double)(float)normal(key, (uint64_t)(i0 + i)));
}

/* Top-k of one token's keys, descending; ties go to the lower expert index.
 * Keys equal to -INFINITY are never chosen (caller guarantees k finite keys). */
static void topk_desc(const double *key, int n_experts, int k, int32_t *out) {
    for (int s = 0; s < k; ++s) {
        int best = -1;
        double bv = -INFINITY;
        for (int e = 0; e < n_experts; ++e) {
            int taken = 0;
            for (int r = 0; r < s; ++r) taken |= (out[r] == e);
            if (taken) continue;
            if (best < 0 ? key[e] > -INFINITY : key[e] > bv) { best = e; bv = key[e]; }
        }
        out[s] = best;
    }
}

/*
 * Routing: top-k distinct experts of logits z[t][e] + b[e],
 * z ~ N(0,1) per (token, expert), b ~ N(0, bias_sigma) per expert.
 * Top-k of softmax(logits) equals top-k of the logits.  Tokens are numbered
 * globally from t0 so that a shard of a batch draws the same ids.
 */
void wl_route_topk_normal(int32_t *ids, int64_t t0, int64_t n_tokens, int n_experts, int k,
                          double bias_sigma, uint64_t seed, uint64_t tensor) {
    const uint64_t kz = stream_key(seed, tensor);
    const uint64_t kb = stream_key(seed, tensor + 1);
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < n_tokens; ++t) {
        double key[n_experts];
        for (int e = 0; e < n_experts; ++e)
            key[e] = normal(kz, (uint64_t)((t0 + t) * n_experts + e)) +
                     bias_sigma * normal(kb, (uint64_t)e);
        topk_desc(key, n_experts, k, ids + t * k);
    }
}

/* Uniform routing: a uniformly random k-subset per token (top-k of i.i.d.
 * uniform keys), listed in descending key order. */
void wl_route_uniform(int32_t *ids, int64_t t0, int64_t n_tokens, int n_experts, int k,
                      uint64_t seed, uint64_t tensor) {
    const uint64_t ku = stream_key(seed, tensor);
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < n_tokens; ++t) {
        double key[n_experts];
        for (int e = 0; e < n_experts; ++e) key[e] = unif01(draw(ku, (uint64_t)((t0 + t) * n_experts + e)));
        topk_desc(key, n_experts, k, ids + t * k);
    }
}

/*
 * Zipf-skewed routing.  A seeded permutation ranks the experts 1..E; expert
 * of rank r has popularity p ~ r^(-s), except that the n_zero lowest-ranked
 * experts get p = 0 (they never receive a token).  Each token takes k distinct
 * experts by Gumbel-top-k: key = log p + G, G = -log(-log U).
 */
void wl_route_zipf(int32_t *ids, int64_t t0, int64_t n_tokens, int n_experts, int k, double s,
                   int n_zero, uint64_t seed, uint64_t tensor) {
    const uint64_t kp = stream_key(seed, tensor + 1);
    const uint64_t kg = stream_key(seed, tensor);
    double logp[n_experts];
    /* rank of e = 1 + number of experts whose permutation key is smaller
     * (ties broken by index) */
    for (int e = 0; e < n_experts; ++e) {
        uint64_t ke = draw(kp, (uint64_t)e);
        int rank = 1;
        for (int f = 0; f < n_experts; ++f) {
            uint64_t kf = draw(kp, (uint64_t)f);
            if (kf < ke || (kf == ke && f < e)) ++rank;
        }
        logp[e] = (rank > n_experts - n_zero) ? -INFINITY : -s * log((double)rank);
    }
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < n_tokens; ++t) {
        double key[n_experts];
        for (int e = 0; e < n_experts; ++e) {
            double u = unif_open(draw(kg, (uint64_t)((t0 + t) * n_experts + e)));
            key[e] = logp[e] + (-log(-log(u)));
        }
        topk_desc(key, n_experts, k, ids + t * k);
    }
}
