/*
 * seeded_inputs/philox.h -- the seeded synthetic-input generator.
 *
 * This header is the ONLY code shared by the CPU oracle and the CUDA path, and it
 * holds none of the optimizer-step arithmetic: it only turns (seed, stream, index)
 * into input values (fp32 master weights and moments, fp16 gradients) so that both
 * sides see bit-identical inputs without copying multi-GB buffers between them.
 *
 * Generator: Philox4x32-10, the counter-based generator published by Salmon, Moraes,
 * Dror and Shaw ("Parallel random numbers: as easy as 1, 2, 3", SC'11, section 4.2):
 * 10 rounds of two 32x32->64 multiplies per round, with the key bumped by the Weyl
 * constants between rounds.  Written here from that definition; checked against the
 * published known-answer vectors in the tests.
 *
 * Normal variates: Irwin-Hall with 12 terms.  Twelve 24-bit uniform integers are
 * summed exactly in uint32; subtracting 6*2^24 gives an integer with mean ~0 and
 * variance 2^48 (i.e. 1 in units of 2^24).  The integer is converted to double
 * (exact), multiplied by (sigma * 2^-24) in double (one IEEE multiply), and rounded
 * once to fp32.  Every step is an integer op or a single correctly rounded IEEE
 * operation, so host and device produce the same bits without any libm call.
 *
 * fp16 values are produced from that fp32 value by round-to-nearest-even, using an
 * integer-only conversion below (no hardware intrinsic), so again host == device.
 *
 * Usable from C (gcc) and from CUDA device code (nvcc).
 */
#ifndef SEEDED_INPUTS_PHILOX_H
#define SEEDED_INPUTS_PHILOX_H

#include <stdint.h>
#include <string.h>

#if defined(__CUDACC__)
#define SI_FN __host__ __device__ __forceinline__
#else
#define SI_FN static inline
#endif

/* Stream ids: each input array draws from its own Philox key (seed, stream). */
enum {
    SI_STREAM_MASTER = 1,   /* fp32 master weights            */
    SI_STREAM_M      = 2,   /* fp32 first moment (warm state)  */
    SI_STREAM_V      = 3,   /* fp32 second moment (warm state) */
    SI_STREAM_SIZES  = 4,   /* tensor sizes of the ragged list */
    SI_STREAM_GRAD0  = 1024 /* rank r's fp16 gradient: GRAD0 + r */
};

typedef struct { uint32_t w[4]; } si_u32x4;

/* One Philox4x32 round: two 32x32 -> 64-bit products, xor-mixed with the key. */
SI_FN si_u32x4 si_philox_round(si_u32x4 c, uint32_t k0, uint32_t k1)
{
    const uint64_t p0 = (uint64_t)0xD2511F53u * (uint64_t)c.w[0];
    const uint64_t p1 = (uint64_t)0xCD9E8D57u * (uint64_t)c.w[2];
    si_u32x4 r;
    r.w[0] = (uint32_t)(p1 >> 32) ^ c.w[1] ^ k0;
    r.w[1] = (uint32_t)p1;
    r.w[2] = (uint32_t)(p0 >> 32) ^ c.w[3] ^ k1;
    r.w[3] = (uint32_t)p0;
    return r;
}

/* Philox4x32-10: ten rounds; the key advances by the Weyl increments between rounds. */
SI_FN si_u32x4 si_philox4x32_10(si_u32x4 ctr, uint32_t k0, uint32_t k1)
{
    for (int round = 0; round < 10; ++round) {
        if (round > 0) {
            k0 += 0x9E3779B9u;
            k1 += 0xBB67AE85u;
        }
        ctr = si_philox_round(ctr, k0, k1);
    }
    return ctr;
}

/* Block j of the random stream (seed, stream) at element index i. */
SI_FN si_u32x4 si_block(uint32_t seed, uint32_t stream, uint64_t index, uint32_t j)
{
    si_u32x4 c;
    c.w[0] = (uint32_t)index;
    c.w[1] = (uint32_t)(index >> 32);
    c.w[2] = j;
    c.w[3] = 0u;
    return si_philox4x32_10(c, seed, stream);
}

/* Irwin-Hall(12) integer: sum of twelve 24-bit uniforms minus 6*2^24. */
SI_FN int32_t si_irwin_hall12(uint32_t seed, uint32_t stream, uint64_t index)
{
    uint32_t sum = 0u;
    for (uint32_t j = 0; j < 3u; ++j) {
        const si_u32x4 b = si_block(seed, stream, index, j);
        sum += (b.w[0] >> 8) + (b.w[1] >> 8) + (b.w[2] >> 8) + (b.w[3] >> 8);
    }
    return (int32_t)sum - (int32_t)(6u << 24);
}

/* The 4th block supplies per-element uniform words (heavy-tail flag, size draws). */
SI_FN uint32_t si_extra_word(uint32_t seed, uint32_t stream, uint64_t index)
{
    return si_block(seed, stream, index, 3u).w[0];
}

/* Scale an Irwin-Hall integer to fp32: double(z) * (scale * 2^-24), rounded once. */
SI_FN float si_scaled_normal(int32_t z, double scale)
{
    const double unit = scale * (1.0 / 16777216.0); /* exact: power-of-two factor */
    return (float)((double)z * unit);
}

SI_FN uint32_t si_f32_bits(float f)
{
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    return u;
}

/* fp32 -> fp16 bits, round to nearest even, integer ops only (IEEE 754 binary16). */
SI_FN uint16_t si_f32_to_f16_rne(float f)
{
    const uint32_t x = si_f32_bits(f);
    const uint32_t sign = (x >> 16) & 0x8000u;
    const uint32_t ax = x & 0x7fffffffu;
    if (ax >= 0x7f800000u)                         /* inf or nan */
        return (uint16_t)(sign | (ax > 0x7f800000u ? 0x7e00u : 0x7c00u));
    if (ax >= 0x477ff000u)                         /* >= 65520: rounds to inf */
        return (uint16_t)(sign | 0x7c00u);
    if (ax >= 0x38800000u) {                       /* >= 2^-14: normal half */
        uint32_t h = (((ax >> 23) - 112u) << 10) | ((ax & 0x7fffffu) >> 13);
        const uint32_t rem = ax & 0x1fffu;
        if (rem > 0x1000u || (rem == 0x1000u && (h & 1u))) h += 1u;
        return (uint16_t)(sign | h);
    }
    if (ax < 0x33000000u)                          /* < 2^-25: rounds to zero */
        return (uint16_t)sign;
    {                                              /* subnormal half: units of 2^-24 */
        const uint32_t e = ax >> 23;               /* 102 .. 112 */
        const uint32_t m = (ax & 0x7fffffu) | 0x800000u;
        const uint32_t shift = 126u - e;           /* 14 .. 24 */
        uint32_t q = m >> shift;
        const uint32_t rem = m & ((1u << shift) - 1u);
        const uint32_t half = 1u << (shift - 1u);
        if (rem > half || (rem == half && (q & 1u))) q += 1u;
        return (uint16_t)(sign | q);
    }
}

/* ---- the input arrays, element by element ---------------------------------- */

/* fp32 value ~ N(0, sigma^2) of stream `stream` at index i. */
SI_FN float si_normal_f32(uint32_t seed, uint32_t stream, uint64_t i, double sigma)
{
    return si_scaled_normal(si_irwin_hall12(seed, stream, i), sigma);
}

/* |N(0, sigma^2)| (second-moment warm state). */
SI_FN float si_abs_normal_f32(uint32_t seed, uint32_t stream, uint64_t i, double sigma)
{
    const float f = si_normal_f32(seed, stream, i, sigma);
    return f < 0.0f ? -f : f;
}

/*
 * Rank r's fp16 gradient at flat index i: fp16(loss_scale * N(0, sigma^2)), where a
 * fraction heavy_frac_q32 / 2^32 of the entries (chosen by the stream's extra word)
 * is multiplied by heavy_mult (heavy-tailed workloads; 0 disables).
 */
SI_FN uint16_t si_grad_f16(uint32_t seed, int32_t rank, uint64_t i, double sigma,
                           double loss_scale, uint32_t heavy_frac_q32, double heavy_mult)
{
    const uint32_t stream = (uint32_t)SI_STREAM_GRAD0 + (uint32_t)rank;
    double scale = loss_scale * sigma;
    if (heavy_frac_q32 != 0u && si_extra_word(seed, stream, i) < heavy_frac_q32)
        scale = scale * heavy_mult;
    return si_f32_to_f16_rne(si_scaled_normal(si_irwin_hall12(seed, stream, i), scale));
}

#endif /* SEEDED_INPUTS_PHILOX_H */
