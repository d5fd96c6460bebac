/*
 * Seeded synthetic-input generator, host side.
 *
 * This module only makes test inputs.  It holds none of the MoE layer's
 * arithmetic: it turns (seed, stream, counter) into 64-bit words, and maps
 * words onto raw bytes, integer codes in a range and uniform scales.  Both
 * the CPU oracle's inputs and the GPU path's inputs come from here (the GPU
 * twin in synth_gpu.cu produces the same words for the large resident
 * weight sets).
 *
 * Word generator: Vigna's splitmix64 output mixer used as a counter-based
 * hash (published with xoroshiro, "Further scramblings of Marsaglia's
 * xorshift generators", and in java.util.SplittableRandom):
 *   mix(z):  z += 0x9E3779B97F4A7C15
 *            z  = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9
 *            z  = (z ^ (z >> 27)) * 0x94D049BB133111EB
 *            return z ^ (z >> 31)
 *   key(seed, stream) = mix(mix(seed) ^ stream)
 *   word(seed, stream, i) = mix(key + i)
 */
#include <stdint.h>
#include <stddef.h>

static inline uint64_t synth_mix(uint64_t z) {
    z += 0x9E3779B97F4A7C15ull;
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
    return z ^ (z >> 31);
}

uint64_t synth_key(uint64_t seed, uint64_t stream) {
    return synth_mix(synth_mix(seed) ^ stream);
}

/* out[j] = word(seed, stream, start + j) for j in [0, n). */
void synth_words(uint64_t seed, uint64_t stream, uint64_t start, size_t n, uint64_t* out) {
    const uint64_t k = synth_key(seed, stream);
    for (size_t j = 0; j < n; ++j) out[j] = synth_mix(k + start + (uint64_t)j);
}

/* Raw bytes: byte b is bits 8*(b%8).. of word b/8 (little-endian unpacking of
 * consecutive words).  Covers bytes [start_byte, start_byte + n).  Used for
 * packed int4 / int2 weights, where every nibble / 2-bit field of a uniform
 * random byte is itself uniform over its code range. */
void synth_bytes(uint64_t seed, uint64_t stream, uint64_t start_byte, size_t n, uint8_t* out) {
    const uint64_t k = synth_key(seed, stream);
    for (size_t j = 0; j < n; ++j) {
        const uint64_t b = start_byte + (uint64_t)j;
        out[j] = (uint8_t)(synth_mix(k + (b >> 3)) >> (8u * (unsigned)(b & 7u)));
    }
}

/* Integer codes uniform on [-127, 127]: code c uses the 32-bit half
 * (c & 1) of word c/2, r, and maps it to ((r * 255) >> 32) - 127. */
void synth_codes_i8(uint64_t seed, uint64_t stream, uint64_t start_code, size_t n, int8_t* out) {
    const uint64_t k = synth_key(seed, stream);
    for (size_t j = 0; j < n; ++j) {
        const uint64_t c = start_code + (uint64_t)j;
        const uint64_t r = (synth_mix(k + (c >> 1)) >> (32u * (unsigned)(c & 1u))) & 0xFFFFFFFFull;
        out[j] = (int8_t)((int)((r * 255ull) >> 32) - 127);
    }
}

/* Scales uniform on [lo, lo + span): u = top 24 bits of word r,
 * scale = lo + span * (u * 2^-24), each step one fp32 rounding
 * (mul by 2^-24 is exact). */
void synth_scales(uint64_t seed, uint64_t stream, uint64_t start, size_t n,
                  float lo, float span, float* out) {
    const uint64_t k = synth_key(seed, stream);
    volatile float two_m24 = 5.9604644775390625e-08f;
    for (size_t j = 0; j < n; ++j) {
        const uint32_t u = (uint32_t)(synth_mix(k + start + (uint64_t)j) >> 40);
        volatile float a = (float)u * two_m24;
        volatile float b = a * span;
        out[j] = b + lo;
    }
}
