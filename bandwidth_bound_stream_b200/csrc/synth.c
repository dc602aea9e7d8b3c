/*
 * Seeded synthetic inputs for the decode engine and for its test oracle.
 *
 * This module only draws numbers: weights ~ N(0, std) rounded to fp16/bf16, constant
 * norm gains, uniform token ids and per-session prompt lengths. It holds none of the
 * forward-pass arithmetic, and both the CUDA engine's harness and the CPU oracle's
 * harness consume exactly the bytes it writes.
 *
 * Generator: splitmix64 (Steele, Lea & Flood, "Fast splittable pseudorandom number
 * generators", OOPSLA 2014; constants of Vigna's public-domain splitmix64.c). The
 * i-th output of a splitmix64 stream whose state starts at s is mix(s + (i+1)*golden),
 * so any word can be drawn directly from (seed, stream, i): the generator is
 * counter-based and the result does not depend on thread count or call order.
 *
 * Normals: the Box-Muller transform (Box & Muller 1958) on two words per pair;
 * element 2j takes r*cos(t), element 2j+1 takes r*sin(t).
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

#define GOLDEN 0x9E3779B97F4A7C15ULL

static inline uint64_t mix64(uint64_t z) {
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
    return z ^ (z >> 31);
}

/* One step of the sequential splitmix64 generator (for cross-checking the counter form). */
uint64_t synth_splitmix64_next(uint64_t *state) {
    *state += GOLDEN;
    return mix64(*state);
}

/* Starting state of stream `stream` under `seed`. */
uint64_t synth_stream_key(uint64_t seed, uint64_t stream) {
    return mix64(seed ^ mix64(stream * GOLDEN + 0x632BE59BD9B4E019ULL));
}

/* Word i (0-based) of stream `stream`: the (i+1)-th output of splitmix64 started at the key. */
uint64_t synth_word(uint64_t seed, uint64_t stream, uint64_t i) {
    return mix64(synth_stream_key(seed, stream) + (i + 1) * GOLDEN);
}

/* float -> IEEE binary16, round to nearest even. */
static uint16_t f32_to_f16(float f) {
    uint32_t x;
    memcpy(&x, &f, 4);
    uint32_t sign = (x >> 16) & 0x8000u;
    uint32_t ax = x & 0x7FFFFFFFu;
    if (ax >= 0x7F800000u) return (uint16_t)(sign | (ax > 0x7F800000u ? 0x7E00u : 0x7C00u));
    if (ax >= 0x477FF000u) return (uint16_t)(sign | 0x7C00u); /* >= 65520 -> inf */
    if (ax < 0x38800000u) {                                   /* below 2^-14: subnormal */
        uint32_t e = ax >> 23;
        if (e < 102) return (uint16_t)sign;
        uint32_t m = (ax & 0x7FFFFFu) | 0x800000u;
        uint32_t shift = 126 - e;
        uint32_t q = m >> shift, rem = m & ((1u << shift) - 1u), half = 1u << (shift - 1);
        if (rem > half || (rem == half && (q & 1u))) q++;
        return (uint16_t)(sign | q);
    }
    uint32_t r = ax + 0xFFFu + ((ax >> 13) & 1u);
    r -= 0x38000000u;
    return (uint16_t)(sign | (r >> 13));
}

/* float -> bfloat16, round to nearest even (inputs here are finite). */
static uint16_t f32_to_bf16(float f) {
    uint32_t x;
    memcpy(&x, &f, 4);
    return (uint16_t)((x + 0x7FFFu + ((x >> 16) & 1u)) >> 16);
}

uint16_t synth_round_f32(float f, int32_t dtype) { return dtype == 0 ? f32_to_f16(f) : f32_to_bf16(f); }

static inline double u01(uint64_t w) { return (double)((w >> 11) + 1) * 0x1.0p-53; } /* (0, 1] */

/*
 * Elements [offset, offset + n) of a N(0, std^2) tensor drawn from stream `stream`,
 * rounded double -> float -> storage dtype (0 = fp16, 1 = bf16).
 */
void synth_normal_u16(uint64_t seed, uint64_t stream, int64_t offset, int64_t n, double std,
                      int32_t dtype, uint16_t *out) {
    const uint64_t key = synth_stream_key(seed, stream);
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; i++) {
        uint64_t e = (uint64_t)(offset + i);
        uint64_t j = e >> 1;
        double u1 = u01(mix64(key + (2 * j + 1) * GOLDEN));
        double u2 = u01(mix64(key + (2 * j + 2) * GOLDEN));
        double r = sqrt(-2.0 * log(u1));
        double t = 6.283185307179586476925 * u2;
        double z = (e & 1) ? r * sin(t) : r * cos(t);
        out[i] = synth_round_f32((float)(std * z), dtype);
    }
}

/* n copies of one storage value (norm gains). */
void synth_fill_u16(int64_t n, uint16_t value, uint16_t *out) {
    for (int64_t i = 0; i < n; i++) out[i] = value;
}

/* Token ids: word j of the stream, reduced modulo the vocabulary. */
void synth_tokens(uint64_t seed, uint64_t stream, int64_t n, int32_t vocab, int32_t *out) {
    const uint64_t key = synth_stream_key(seed, stream);
    for (int64_t j = 0; j < n; j++) out[j] = (int32_t)(mix64(key + (uint64_t)(j + 1) * GOLDEN) % (uint64_t)vocab);
}

/* Integer uniform on [lo, hi] from word i of a stream. */
int32_t synth_uniform_int(uint64_t seed, uint64_t stream, uint64_t i, int32_t lo, int32_t hi) {
    return lo + (int32_t)(synth_word(seed, stream, i) % (uint64_t)(hi - lo + 1));
}
