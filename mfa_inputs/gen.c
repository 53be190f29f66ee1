/*
 * Seeded synthetic inputs shared by the parity tests, the bench and the oracle driver.
 *
 * This file holds no attention arithmetic. It only turns (seed, stream, counter) into
 * numbers:
 *   - SplitMix64 (Steele, Lea and Flood, "Fast splittable pseudorandom number generators",
 *     OOPSLA 2014) used as a counter-based generator: draw n of stream s is
 *     mix(key(seed, s) + (n + 1) * gamma), so any slice can be produced independently.
 *   - Box-Muller (Box and Muller, 1958) turns draw pairs (2p, 2p+1) into two N(0,1) values.
 *   - The fp64 normal, times a caller factor, is rounded to the storage type:
 *       fp16: one round-to-nearest-even step from fp64 (C's _Float16 conversion);
 *       bf16: fp64 -> fp32 (RNE), then fp32 -> bf16 (RNE on the bit pattern).
 *     The stored 16-bit patterns ARE the inputs; both the CUDA path and the oracle read them.
 */
#include <stdint.h>
#include <math.h>
#include <string.h>

#define GAMMA 0x9E3779B97F4A7C15ULL

static inline uint64_t mix64(uint64_t z) {
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
    return z ^ (z >> 31);
}

/* Stream key: one SplitMix64 step from a seed/stream combination. */
static inline uint64_t stream_key(uint64_t seed, uint64_t stream) {
    return mix64(seed * GAMMA + stream * 0xD1B54A32D192ED03ULL + GAMMA);
}

uint64_t mfa_gen_draw(uint64_t seed, uint64_t stream, uint64_t n) {
    return mix64(stream_key(seed, stream) + (n + 1) * GAMMA);
}

/* Raw 64-bit draws [offset, offset + n). */
void mfa_gen_u64(uint64_t seed, uint64_t stream, uint64_t offset, int64_t n, uint64_t* out) {
    uint64_t key = stream_key(seed, stream);
    #pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) out[i] = mix64(key + (offset + (uint64_t)i + 1) * GAMMA);
}

static inline uint16_t f32_to_bf16_rne(float f) {
    uint32_t u;
    memcpy(&u, &f, 4);
    if ((u & 0x7F800000u) == 0x7F800000u && (u & 0x007FFFFFu)) return (uint16_t)((u >> 16) | 0x40u);
    uint32_t lsb = (u >> 16) & 1u;
    u += 0x7FFFu + lsb;
    return (uint16_t)(u >> 16);
}

static inline uint16_t f64_to_f16_bits(double x) {
    _Float16 h = (_Float16)x;
    uint16_t b;
    memcpy(&b, &h, 2);
    return b;
}

/*
 * Normal values number [offset, offset + n) of one stream, times `mul`, rounded to
 * dtype (0 = fp16, 1 = bf16, 2 = fp64 written as raw doubles into out64).
 * Value 2p and 2p+1 come from the Box-Muller pair built on draws 2p and 2p+1.
 */
static inline void normal_pair(uint64_t key, uint64_t p, double* z0, double* z1) {
    uint64_t r0 = mix64(key + (2 * p + 1) * GAMMA);
    uint64_t r1 = mix64(key + (2 * p + 2) * GAMMA);
    double u1 = ((double)(r0 >> 11) + 1.0) * 0x1.0p-53;   /* (0, 1] */
    double u2 = (double)(r1 >> 11) * 0x1.0p-53;           /* [0, 1) */
    double rad = sqrt(-2.0 * log(u1));
    double th = 6.283185307179586476925286766559 * u2;
    *z0 = rad * cos(th);
    *z1 = rad * sin(th);
}

void mfa_gen_normal(uint64_t seed, uint64_t stream, uint64_t offset, int64_t n, double mul,
                    int dtype, uint16_t* out16, double* out64) {
    uint64_t key = stream_key(seed, stream);
    #pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) {
        uint64_t idx = offset + (uint64_t)i;
        double z0, z1;
        normal_pair(key, idx >> 1, &z0, &z1);
        double z = ((idx & 1) ? z1 : z0) * mul;
        if (dtype == 0) out16[i] = f64_to_f16_bits(z);
        else if (dtype == 1) out16[i] = f32_to_bf16_rne((float)z);
        else out64[i] = z;
    }
}

/* 16-bit float patterns -> exact fp64 values (the oracle's view of the stored inputs). */
void mfa_gen_widen(const uint16_t* in, int64_t n, int dtype, double* out) {
    #pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) {
        if (dtype == 0) {
            _Float16 h;
            memcpy(&h, &in[i], 2);
            out[i] = (double)h;
        } else {
            uint32_t u = (uint32_t)in[i] << 16;
            float f;
            memcpy(&f, &u, 4);
            out[i] = (double)f;
        }
    }
}
