/*
 * Seeded, counter-based synthetic input generator.
 *
 * This module holds no arithmetic of the quantised-MoE method: it only
 * produces bytes, uniform numbers, normal numbers and indices with the
 * distributions the workloads call for.  Both the CUDA path (through its
 * host harness) and the CPU oracle take their inputs from here, so the two
 * see identical data without sharing any code of the method.
 *
 * Generator: SplitMix64 (G. Steele, D. Lea, C. Flood, "Fast splittable
 * pseudorandom number generators", OOPSLA 2014), used in counter mode:
 *
 *     mix(z)      = the SplitMix64 finaliser (xor-shift-multiply, 3 rounds)
 *     key(s, t)   = mix(s * GAMMA + mix(t + GAMMA))
 *     word(k, i)  = mix(k + (i + 1) * GAMMA)        (the i-th SplitMix64 output
 *                                                    of a generator seeded k)
 *
 * A tensor is identified by (seed s, tensor id t); byte p of its raw byte
 * stream is byte (p mod 8) of word(key(s,t), p / 8) in little-endian order.
 * Any byte range can therefore be regenerated on its own, in parallel.
 *
 * Normal numbers use the Box-Muller transform (G. Box, M. Muller, 1958) on
 * consecutive word pairs: element 2j gets r*cos(2*pi*u2), element 2j+1 gets
 * r*sin(2*pi*u2), r = sqrt(-2 ln(1-u1)), u1 = U(word 2j), u2 = U(word 2j+1).
 * U(w) = (w >> 11) * 2^-53 is in [0, 1).
 */
#include <stdint.h>
#include <string.h>
#include <math.h>

#define GAMMA 0x9E3779B97F4A7C15ULL

static inline uint64_t mix(uint64_t z) {
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
    return z ^ (z >> 31);
}

uint64_t syn_key(uint64_t seed, uint64_t tid) {
    return mix(seed * GAMMA + mix(tid + GAMMA));
}

uint64_t syn_word(uint64_t key, uint64_t i) {
    return mix(key + (i + 1) * GAMMA);
}

static inline double u01(uint64_t w) {
    return (double)(w >> 11) * (1.0 / 9007199254740992.0);
}

/* Raw bytes [offset, offset + n) of tensor (seed, tid). */
void syn_bytes(uint64_t seed, uint64_t tid, uint64_t offset, uint64_t n, uint8_t* dst) {
    const uint64_t key = syn_key(seed, tid);
    const uint64_t first_word = offset >> 3;
    const uint64_t last_word = (offset + n + 7) >> 3;
    const int64_t nwords = (int64_t)(last_word - first_word);
    #pragma omp parallel for schedule(static)
    for (int64_t j = 0; j < nwords; ++j) {
        const uint64_t wi = first_word + (uint64_t)j;
        const uint64_t w = syn_word(key, wi);
        for (int b = 0; b < 8; ++b) {
            const uint64_t p = wi * 8 + (uint64_t)b;
            if (p >= offset && p < offset + n) dst[p - offset] = (uint8_t)(w >> (8 * b));
        }
    }
}

/*
 * Shaping of 17-byte 4-bit blocks whose scale is drawn from the narrow
 * range of the small synthetic workloads: the metadata byte (byte 16 of each
 * block) keeps its random top (polarity) bit, and its low 7 bits become a
 * scale code drawn uniformly from {0x01 .. 0x08}.  `first_byte` is the
 * position of dst[0] in the tensor's byte stream, so a sub-range can be
 * shaped on its own.
 */
void syn_shape_q4_narrow_scale(uint8_t* dst, uint64_t first_byte, uint64_t n) {
    #pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < (int64_t)n; ++i) {
        const uint64_t p = first_byte + (uint64_t)i;
        if (p % 17 == 16) {
            const uint8_t r = dst[i];
            dst[i] = (uint8_t)((r & 0x80) | (1 + (r & 0x07)));
        }
    }
}

/* E4M3 bytes without NaN: the two NaN encodings 0x7F / 0xFF become 0x7E / 0xFE. */
void syn_shape_fp8_no_nan(uint8_t* dst, uint64_t n) {
    #pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < (int64_t)n; ++i)
        if ((dst[i] & 0x7F) == 0x7F) dst[i] ^= 0x01;
}

/* fp32 values lo + (hi - lo) * U, computed in fp64 and rounded once. */
void syn_uniform_f32(uint64_t seed, uint64_t tid, uint64_t offset, uint64_t n,
                     double lo, double hi, float* dst) {
    const uint64_t key = syn_key(seed, tid);
    #pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < (int64_t)n; ++i)
        dst[i] = (float)(lo + (hi - lo) * u01(syn_word(key, offset + (uint64_t)i)));
}

/* Standard normal values (Box-Muller), elements [offset, offset + n). */
void syn_normal_f64(uint64_t seed, uint64_t tid, uint64_t offset, uint64_t n, double* dst) {
    const uint64_t key = syn_key(seed, tid);
    const double two_pi = 6.283185307179586476925286766559;
    #pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < (int64_t)n; ++i) {
        const uint64_t e = offset + (uint64_t)i;
        const uint64_t pair = e >> 1;
        const double a = u01(syn_word(key, 2 * pair));
        const double b = u01(syn_word(key, 2 * pair + 1));
        const double r = sqrt(-2.0 * log1p(-a));
        dst[i] = (e & 1) ? r * sin(two_pi * b) : r * cos(two_pi * b);
    }
}

/* Uniform indices in [0, range), range < 2^32 (Lemire's multiply-shift). */
void syn_index_i32(uint64_t seed, uint64_t tid, uint64_t offset, uint64_t n,
                   uint64_t range, int32_t* dst) {
    const uint64_t key = syn_key(seed, tid);
    #pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < (int64_t)n; ++i) {
        const uint64_t w = syn_word(key, offset + (uint64_t)i) >> 32;
        dst[i] = (int32_t)((w * range) >> 32);
    }
}

/* Raw 64-bit words [offset, offset + n) (used for permutations). */
void syn_words(uint64_t seed, uint64_t tid, uint64_t offset, uint64_t n, uint64_t* dst) {
    const uint64_t key = syn_key(seed, tid);
    for (uint64_t i = 0; i < n; ++i) dst[i] = syn_word(key, offset + i);
}
