// zero_step_noalloc: the fused optimizer step for callers that must not allocate.
//
// zero_step reads a segment table and tile index that zero_layout_to_device places in
// memory it obtains with cudaMalloc.  Some callers cannot let a library do that: their
// device memory is owned by another allocator (a framework's caching allocator or a
// fixed memory pool that has reserved the GPU), their loop cannot afford the implicit
// device-wide synchronisation an allocation may bring, or they call in from a context
// where allocation is forbidden.  This entry point keeps that scratch in the array
// below, a file-scope static device array that exists on every GPU that loads the
// library, from load until the process exits, so a call allocates nothing.
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>

#include "internal.h"

namespace {

constexpr int kMaxDevices = 64;

// Rows 0..n-1: the layout's segments with their first tile; row n: the closing row.
static __device__ __align__(256) zero::Seg g_step_scratch[ZERO_NOALLOC_MAX_SEGMENTS + 1];

std::mutex g_lock;
zero::Seg *g_scratch_addr[kMaxDevices] = {};

// Device address of g_step_scratch on the current device, looked up on the first call on
// each device and kept for the life of the process.  (In host code the array's name is
// only a host-side handle; the kernels need this.)  A cudaDeviceReset tears down the
// device's context and with it the array's mapping, so the kept address is stale after
// one: a process that resets a device must not call this entry point on it again.
zero_status scratch_address(zero::Seg **out)
{
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return ZERO_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return ZERO_ERR_STATE;
    std::lock_guard<std::mutex> hold(g_lock);
    if (!g_scratch_addr[dev]) {
        void *p = nullptr;
        const cudaError_t e = cudaGetSymbolAddress(&p, g_step_scratch);
        if (e != cudaSuccess || !p) return ZERO_ERR_CUDA;
        g_scratch_addr[dev] = static_cast<zero::Seg *>(p);
    }
    *out = g_scratch_addr[dev];
    return ZERO_OK;
}

bool aligned16(const void *p) { return ((uintptr_t)p & 15u) == 0; }

}  // namespace

extern "C" zero_status zero_step_noalloc(const zero_layout *L, const uint16_t *grads, int64_t rank_stride,
                                         float *master, float *m, float *v, uint16_t *p16_shard,
                                         uint16_t *p16_full, const zero_adamw_hparams *hp,
                                         int32_t *nonfinite, void *stream)
{
    ZERO_RANGE("zero_step_noalloc");
    if (!L || zero::check_hparams(hp) != ZERO_OK) return ZERO_ERR_INVALID;
    if (L->padded == 0) return ZERO_OK;
    const int64_t n_seg = (int64_t)L->segs.size();
    if (n_seg > ZERO_NOALLOC_MAX_SEGMENTS) return ZERO_ERR_INVALID;   // table would not fit
    if (!grads || rank_stride < L->padded || !master || !m || !v || !p16_full ||
        (L->stage == 3 && !p16_shard))
        return ZERO_ERR_INVALID;
    if (rank_stride % 8 != 0 || !aligned16(grads) || !aligned16(master) || !aligned16(m) ||
        !aligned16(v) || !aligned16(p16_full) || (p16_shard && !aligned16(p16_shard)))
        return ZERO_ERR_ALIGN;

    zero::Seg *table = nullptr;
    zero_status s = scratch_address(&table);
    if (s != ZERO_OK) return s;
    cudaStream_t st = (cudaStream_t)stream;

    // Every call rewrites rows 0..n_seg before any kernel reads them (the row contents
    // from the layout's host table and closing row, then the first-tile column from the
    // device scan), so nothing left over from an earlier call is ever read.  Both host
    // sources belong to the layout and live as long as it does.
    cudaError_t e = cudaMemcpyAsync(table, L->segs.data(), (size_t)n_seg * sizeof(zero::Seg),
                                    cudaMemcpyHostToDevice, st);
    if (e == cudaSuccess)
        e = cudaMemcpyAsync(table + n_seg, &L->closing, sizeof(zero::Seg), cudaMemcpyHostToDevice, st);
    if (e == cudaSuccess) e = zero::launch_tile_index(table, n_seg, st);
    const zero::AdamScalars c = zero::step_scalars(L->n_ranks, *hp);

    zero::TileWork w;
    w.segs = table;
    w.seg_first = 0;
    w.tile_first = 0;
    w.n_tiles = L->n_tiles;
    w.bounds = zero::tile_bounds(*L, 0, L->padded);   // no error word: a failed check only skips
    uint16_t *p16 = L->stage == 3 ? p16_shard : p16_full;
    if (e == cudaSuccess)
        e = zero::launch_fused_step(*L, w, grads, rank_stride, master, m, v, p16, c, nonfinite, st);
    if (e == cudaSuccess && L->stage == 3) e = zero::launch_copy_range(*L, 0, L->padded, p16_shard, p16_full, st);
    return e == cudaSuccess ? ZERO_OK : ZERO_ERR_CUDA;
}
