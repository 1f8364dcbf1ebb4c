/*
 * seeded_inputs/gen_cuda.cu -- device-side fill of the seeded synthetic inputs.
 *
 * Same values as gen_host.c (both evaluate philox.h element by element), written
 * straight into device memory so that multi-GB workloads never cross PCIe.  This is
 * input generation only; it is not part of the optimizer-step library.
 */
#include <cuda_runtime.h>
#include <stdint.h>
#include "philox.h"

#define SI_EXPORT extern "C" __attribute__((visibility("default")))

namespace {

constexpr int kThreads = 256;

__global__ void fill_f32_kernel(float *out, int64_t n, int64_t valid, uint32_t seed,
                                uint32_t stream, double sigma, int absval)
{
    const int64_t step = (int64_t)gridDim.x * blockDim.x;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += step) {
        float f = 0.0f;
        if (i < valid)
            f = absval ? si_abs_normal_f32(seed, stream, (uint64_t)i, sigma)
                       : si_normal_f32(seed, stream, (uint64_t)i, sigma);
        out[i] = f;
    }
}

__global__ void fill_grads_kernel(uint16_t *row, int32_t rank, int64_t lo, int64_t n, int64_t valid,
                                  uint32_t seed, double sigma, double loss_scale,
                                  uint32_t heavy_frac_q32, double heavy_mult)
{
    const int64_t step = (int64_t)gridDim.x * blockDim.x;
    for (int64_t i = lo + (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += step)
        row[i] = i < valid ? si_grad_f16(seed, rank, (uint64_t)i, sigma, loss_scale,
                                         heavy_frac_q32, heavy_mult)
                           : (uint16_t)0;
}

unsigned grid_for(int64_t n)
{
    int64_t blocks = (n + kThreads - 1) / kThreads;
    if (blocks > 148 * 64) blocks = 148 * 64;
    if (blocks < 1) blocks = 1;
    return (unsigned)blocks;
}

}  // namespace

/* Returns a cudaError_t value (0 = success). */
SI_EXPORT int si_fill_f32_cuda(float *out, int64_t n, int64_t valid, uint32_t seed,
                               uint32_t stream_id, double sigma, int absval, void *stream)
{
    if (n <= 0) return 0;
    fill_f32_kernel<<<grid_for(n), kThreads, 0, (cudaStream_t)stream>>>(
        out, n, valid, seed, stream_id, sigma, absval);
    return (int)cudaGetLastError();
}

SI_EXPORT int si_fill_grads_cuda(uint16_t *out, int32_t n_ranks, int64_t rank_stride,
                                 int64_t valid, uint32_t seed, double sigma, double loss_scale,
                                 uint32_t heavy_frac_q32, double heavy_mult, void *stream)
{
    if (rank_stride <= 0) return 0;
    for (int32_t r = 0; r < n_ranks; ++r) {
        fill_grads_kernel<<<grid_for(rank_stride), kThreads, 0, (cudaStream_t)stream>>>(
            out + (int64_t)r * rank_stride, r, 0, rank_stride, valid, seed, sigma, loss_scale,
            heavy_frac_q32, heavy_mult);
        const cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return (int)e;
    }
    return 0;
}

/* The same values for flat indices [lo, hi) of every rank only (a backward pass that
 * produces one bucket of gradients at a time). */
SI_EXPORT int si_fill_grads_range_cuda(uint16_t *out, int32_t n_ranks, int64_t rank_stride, int64_t lo,
                                       int64_t hi, int64_t valid, uint32_t seed, double sigma,
                                       double loss_scale, uint32_t heavy_frac_q32, double heavy_mult,
                                       void *stream)
{
    if (hi <= lo) return 0;
    if (lo < 0 || hi > rank_stride) return (int)cudaErrorInvalidValue;
    for (int32_t r = 0; r < n_ranks; ++r) {
        fill_grads_kernel<<<grid_for(hi - lo), kThreads, 0, (cudaStream_t)stream>>>(
            out + (int64_t)r * rank_stride, r, lo, hi, valid, seed, sigma, loss_scale, heavy_frac_q32,
            heavy_mult);
        const cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return (int)e;
    }
    return 0;
}
