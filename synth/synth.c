/*
 * Seeded synthetic inputs for decoupled-head attention (shared by the
 * float64 oracle, the tests and the bench).  This file holds none of the
 * attention arithmetic: it only turns (seed, tensor id, element index) into a
 * bf16 bit pattern.
 *
 * Recipe (all integer steps are exact, so every machine gets the same bits):
 *   key   = mix64(seed * 0x100 + tensor_id)
 *   u1,u2 = 53-bit uniforms in (0,1] from mix64(key + 2e + 1), mix64(key + 2e + 2)
 *   z     = sqrt(-2 ln u1) * cos(2 pi u2)          (Box-Muller, one normal per pair)
 *   value = z * factor                             (factor 1, 0.5 or 0.02)
 *   bits  = round-to-nearest-even of value to bfloat16, taken once from the double
 *
 * mix64 is the SplitMix64 output function (Steele, Lea & Flood, "Fast
 * splittable pseudorandom number generators", OOPSLA 2014): add the golden
 * gamma 0x9E3779B97F4A7C15, then xor-shift-multiply by 0xBF58476D1CE4E5B9 and
 * 0x94D049BB133111EB with shifts 30, 27, 31.
 *
 * Build: gcc -O2 -fopenmp -shared -fPIC synth.c -o libsynth.so -lm
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

static inline uint64_t mix64(uint64_t x)
{
    uint64_t z = x + 0x9E3779B97F4A7C15ull;
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
    return z ^ (z >> 31);
}

/* 53 random bits -> uniform in (0, 1]; never 0, so log() is finite. */
static inline double unit53(uint64_t r)
{
    return (double)((r >> 11) + 1ull) * (1.0 / 9007199254740992.0);
}

/* Round a double to bfloat16 bits, nearest-even, in one step from the double.
 * Values below the bf16 normal range (|x| < 2^-126) keep the same rule on the
 * subnormal grid; overflow goes to infinity. NaN maps to the canonical NaN. */
uint16_t synth_double_to_bf16(double x)
{
    if (x != x) return 0x7FC0u;
    uint64_t b;
    memcpy(&b, &x, sizeof b);
    uint16_t sign = (uint16_t)((b >> 48) & 0x8000u);
    double ax = fabs(x);
    if (ax == 0.0) return sign;
    if (ax >= 0x1.0p-126) {
        /* normal bf16 range: keep 7 of the 52 fraction bits */
        uint64_t mag = b & 0x7FFFFFFFFFFFFFFFull;
        uint64_t lsb = (mag >> 45) & 1ull;
        mag += 0x00000FFFFFFFFFFFull + lsb;      /* 2^44 - 1 + lsb */
        mag &= ~0x00001FFFFFFFFFFFull;           /* clear low 45 bits */
        int e = (int)(mag >> 52) - 1023;
        if (e > 127) return (uint16_t)(sign | 0x7F80u);
        uint16_t frac = (uint16_t)((mag >> 45) & 0x7Fu);
        return (uint16_t)(sign | (uint16_t)((e + 127) << 7) | frac);
    }
    /* subnormal bf16: quantum 2^-133; rint() rounds half to even */
    double q = rint(ax * 0x1.0p133);
    if (q >= 128.0) return (uint16_t)(sign | 0x0080u); /* rounds up to min normal */
    return (uint16_t)(sign | (uint16_t)q);
}

/* Fill out[0..n) with the bf16 bits of element offset+i of tensor `tensor_id`. */
void synth_fill_bf16(uint16_t *out, int64_t n, int64_t offset,
                     uint64_t seed, uint32_t tensor_id, double factor)
{
    const uint64_t key = mix64(seed * 0x100ull + (uint64_t)tensor_id);
    const double two_pi = 6.283185307179586476925286766559;
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) {
        uint64_t e = (uint64_t)(offset + i);
        double u1 = unit53(mix64(key + 2ull * e + 1ull));
        double u2 = unit53(mix64(key + 2ull * e + 2ull));
        double z = sqrt(-2.0 * log(u1)) * cos(two_pi * u2);
        out[i] = synth_double_to_bf16(z * factor);
    }
}

/* Same stream as float64 (before the bf16 rounding); used by the generator's tests. */
void synth_fill_f64(double *out, int64_t n, int64_t offset,
                    uint64_t seed, uint32_t tensor_id, double factor)
{
    const uint64_t key = mix64(seed * 0x100ull + (uint64_t)tensor_id);
    const double two_pi = 6.283185307179586476925286766559;
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) {
        uint64_t e = (uint64_t)(offset + i);
        double u1 = unit53(mix64(key + 2ull * e + 1ull));
        double u2 = unit53(mix64(key + 2ull * e + 2ull));
        out[i] = sqrt(-2.0 * log(u1)) * cos(two_pi * u2) * factor;
    }
}

/* Seeded sample of n distinct-ish row indices in [0, limit): used to pick the
 * query positions checked at long sequence lengths. Plain counter hashing;
 * duplicates are removed by the caller. */
void synth_sample_indices(int64_t *out, int64_t n, int64_t limit, uint64_t seed)
{
    const uint64_t key = mix64(seed ^ 0x5A17ull);
    for (int64_t i = 0; i < n; ++i)
        out[i] = (int64_t)(mix64(key + (uint64_t)i) % (uint64_t)limit);
}

uint64_t synth_mix64(uint64_t x) { return mix64(x); }
