/*
 * Host side of the seeded input generator (test and benchmark inputs only).
 *
 * This file holds no arithmetic of the attention method. It turns
 * (seed, tensor id, flat element index) into a reproducible pseudo-normal
 * value, so that the fp64 oracle on the host and the CUDA path on the
 * device see bit-identical inputs without ever copying one from the other.
 * The device twin is rng_device.cu; both follow the same published
 * definitions, written out below.
 *
 * Definition (all arithmetic modulo 2^64 on uint64):
 *   mix64(z)      : SplitMix64 output function (Steele, Lea and Flood,
 *                   "Fast splittable pseudorandom number generators",
 *                   OOPSLA 2014; constants as in Vigna's public-domain
 *                   splitmix64.c):
 *                     z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9
 *                     z = (z ^ (z >> 27)) * 0x94D049BB133111EB
 *                     z =  z ^ (z >> 31)
 *   base(s, t)    = mix64(s + G * (t + 1)),      G = 0x9E3779B97F4A7C15
 *   draw(s, t, i) = mix64(base(s, t) + G * (i + 1))
 *                   (the (i+1)-th SplitMix64 output of a stream whose
 *                   state starts at base(s, t))
 *   normal        : Irwin-Hall sum of the four 16-bit fields u0..u3 of
 *                   draw:  s = u0+u1+u2+u3 (integer, exact),
 *                   z = fp32(s - 131070) * 2^-16      (exact)
 *                   z = z * fp32(sqrt(3))             (one RNE rounding)
 *                   giving mean 0, variance 1 (up to the 16-bit grid),
 *                   support [-2*sqrt(3), 2*sqrt(3)].
 *   scaled        : v = z * sigma  (fp32, one RNE rounding)
 *   bf16 storage  : round-to-nearest-even of the fp32 value.
 *
 * Built with -ffp-contract=off so no product is fused with anything.
 */
#include <stdint.h>
#include <string.h>

#define MSA_RNG_G 0x9E3779B97F4A7C15ULL

static inline uint64_t mix64(uint64_t z) {
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
    return z ^ (z >> 31);
}

static inline uint64_t stream_base(uint64_t seed, uint64_t tensor_id) {
    return mix64(seed + MSA_RNG_G * (tensor_id + 1ULL));
}

static inline float irwin_hall4(uint64_t h) {
    int32_t s = (int32_t)(h & 0xFFFFULL) + (int32_t)((h >> 16) & 0xFFFFULL) +
                (int32_t)((h >> 32) & 0xFFFFULL) + (int32_t)(h >> 48);
    float t = (float)(s - 131070) * (1.0f / 65536.0f);
    return t * 1.7320508075688772f;
}

static inline uint16_t f32_to_bf16_rne(float f) {
    uint32_t u;
    memcpy(&u, &f, 4);
    u += 0x7FFFu + ((u >> 16) & 1u);
    return (uint16_t)(u >> 16);
}

/* Raw 64-bit draws: out[j] = draw(seed, tid, start + j). */
void rng_draw_u64(uint64_t seed, uint64_t tid, uint64_t start, int64_t n, uint64_t* out) {
    const uint64_t b = stream_base(seed, tid);
#pragma omp parallel for schedule(static)
    for (int64_t j = 0; j < n; ++j) out[j] = mix64(b + MSA_RNG_G * (start + (uint64_t)j + 1ULL));
}

/* out[j] = fp32 normal of element (start + j), times sigma. */
void rng_normal_f32(uint64_t seed, uint64_t tid, uint64_t start, int64_t n, float sigma, float* out) {
    const uint64_t b = stream_base(seed, tid);
#pragma omp parallel for schedule(static)
    for (int64_t j = 0; j < n; ++j) {
        float z = irwin_hall4(mix64(b + MSA_RNG_G * (start + (uint64_t)j + 1ULL)));
        out[j] = z * sigma;
    }
}

/* Same values, stored as bf16 bit patterns. */
void rng_normal_bf16(uint64_t seed, uint64_t tid, uint64_t start, int64_t n, float sigma, uint16_t* out) {
    const uint64_t b = stream_base(seed, tid);
#pragma omp parallel for schedule(static)
    for (int64_t j = 0; j < n; ++j) {
        float z = irwin_hall4(mix64(b + MSA_RNG_G * (start + (uint64_t)j + 1ULL)));
        out[j] = f32_to_bf16_rne(z * sigma);
    }
}

/* Rows of a [rows][row_len] tensor picked by an index list: out[r][:] = tensor[rows[r]][:]. */
void rng_normal_rows_f32(uint64_t seed, uint64_t tid, int64_t row_len, const int64_t* rows, int64_t n_rows,
                         float sigma, float* out) {
    const uint64_t b = stream_base(seed, tid);
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < n_rows; ++r) {
        const uint64_t s0 = (uint64_t)rows[r] * (uint64_t)row_len;
        for (int64_t j = 0; j < row_len; ++j) {
            float z = irwin_hall4(mix64(b + MSA_RNG_G * (s0 + (uint64_t)j + 1ULL)));
            out[r * row_len + j] = z * sigma;
        }
    }
}

void rng_normal_rows_bf16(uint64_t seed, uint64_t tid, int64_t row_len, const int64_t* rows, int64_t n_rows,
                          float sigma, uint16_t* out) {
    const uint64_t b = stream_base(seed, tid);
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < n_rows; ++r) {
        const uint64_t s0 = (uint64_t)rows[r] * (uint64_t)row_len;
        for (int64_t j = 0; j < row_len; ++j) {
            float z = irwin_hall4(mix64(b + MSA_RNG_G * (s0 + (uint64_t)j + 1ULL)));
            out[r * row_len + j] = f32_to_bf16_rne(z * sigma);
        }
    }
}

/* Plain SplitMix64 stream from an explicit state: out[j] = mix64(state + G*(j+1)).
 * Exposed only so a test can compare it with the generator's published reference outputs. */
void rng_splitmix64_from_state(uint64_t state, int64_t n, uint64_t* out) {
    for (int64_t j = 0; j < n; ++j) out[j] = mix64(state + MSA_RNG_G * ((uint64_t)j + 1ULL));
}
