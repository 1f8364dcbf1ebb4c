/*
 * seeded_inputs/gen_host.c -- host-side fill of the seeded synthetic inputs.
 *
 * Every value comes from philox.h, so the device fill (gen_cuda.cu) writes the same
 * bits.  Elements at flat index >= `valid` (the tail padding of the flat buffer) are
 * zero, which is what the optimizer-step layout requires of padding.
 * Plain OpenMP loops: this is input generation, not the optimizer arithmetic.
 */
#include <stdint.h>
#include "philox.h"

#if defined(__GNUC__)
#define SI_EXPORT __attribute__((visibility("default")))
#else
#define SI_EXPORT
#endif

SI_EXPORT void si_philox4x32_10_host(const uint32_t ctr[4], const uint32_t key[2], uint32_t out[4])
{
    si_u32x4 c;
    for (int k = 0; k < 4; ++k) c.w[k] = ctr[k];
    const si_u32x4 r = si_philox4x32_10(c, key[0], key[1]);
    for (int k = 0; k < 4; ++k) out[k] = r.w[k];
}

SI_EXPORT void si_f32_to_f16_host(const float *in, uint16_t *out, int64_t n)
{
    for (int64_t i = 0; i < n; ++i) out[i] = si_f32_to_f16_rne(in[i]);
}

SI_EXPORT void si_irwin_hall_host(int32_t *out, int64_t n, uint32_t seed, uint32_t stream)
{
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) out[i] = si_irwin_hall12(seed, stream, (uint64_t)i);
}

SI_EXPORT void si_extra_words_host(uint32_t *out, int64_t n, uint32_t seed, uint32_t stream)
{
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) out[i] = si_extra_word(seed, stream, (uint64_t)i);
}

/* out[i] = N(0, sigma^2) (or its absolute value) for i < valid, 0 for valid <= i < n. */
SI_EXPORT void si_fill_f32_host(float *out, int64_t n, int64_t valid, uint32_t seed,
                                uint32_t stream, double sigma, int absval)
{
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) {
        if (i >= valid) { out[i] = 0.0f; continue; }
        out[i] = absval ? si_abs_normal_f32(seed, stream, (uint64_t)i, sigma)
                        : si_normal_f32(seed, stream, (uint64_t)i, sigma);
    }
}

/* Same values at the listed flat indices only (sampled checks at full size). */
SI_EXPORT void si_gather_f32_host(float *out, const int64_t *idx, int64_t n, int64_t valid,
                                  uint32_t seed, uint32_t stream, double sigma, int absval)
{
#pragma omp parallel for schedule(static)
    for (int64_t j = 0; j < n; ++j) {
        const int64_t i = idx[j];
        if (i >= valid) { out[j] = 0.0f; continue; }
        out[j] = absval ? si_abs_normal_f32(seed, stream, (uint64_t)i, sigma)
                        : si_normal_f32(seed, stream, (uint64_t)i, sigma);
    }
}

/* grads[r * rank_stride + i], r < n_ranks, i < rank_stride; zero for i >= valid. */
SI_EXPORT void si_fill_grads_host(uint16_t *out, int32_t n_ranks, int64_t rank_stride,
                                  int64_t valid, uint32_t seed, double sigma, double loss_scale,
                                  uint32_t heavy_frac_q32, double heavy_mult)
{
    for (int32_t r = 0; r < n_ranks; ++r) {
        uint16_t *row = out + (int64_t)r * rank_stride;
#pragma omp parallel for schedule(static)
        for (int64_t i = 0; i < rank_stride; ++i)
            row[i] = i < valid ? si_grad_f16(seed, r, (uint64_t)i, sigma, loss_scale,
                                             heavy_frac_q32, heavy_mult)
                               : (uint16_t)0;
    }
}

/* out[j * n_ranks + r] = rank r's gradient at flat index idx[j]. */
SI_EXPORT void si_gather_grads_host(uint16_t *out, const int64_t *idx, int64_t n, int32_t n_ranks,
                                    int64_t valid, uint32_t seed, double sigma, double loss_scale,
                                    uint32_t heavy_frac_q32, double heavy_mult)
{
#pragma omp parallel for schedule(static)
    for (int64_t j = 0; j < n; ++j)
        for (int32_t r = 0; r < n_ranks; ++r)
            out[j * n_ranks + r] = idx[j] < valid
                ? si_grad_f16(seed, r, (uint64_t)idx[j], sigma, loss_scale, heavy_frac_q32, heavy_mult)
                : (uint16_t)0;
}
