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
#include <math.h>
#include <stdint.h>

#include <mutex>

#include "internal.h"

namespace {

constexpr int kMaxDevices = 64;

// Rows 0..n-1: the layout's segments with their first tile; row n: the closing row.
static __device__ __align__(256) zero::Seg g_step_scratch[ZERO_NOALLOC_MAX_SEGMENTS + 1];

std::mutex g_lock;
zero::Seg *g_scratch_addr[kMaxDevices] = {};

// Device address of g_step_scratch on the current device, looked up once per device.
// (In host code the array's name is only a host-side handle; the kernels need this.)
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

bool hparams_ok(const zero_adamw_hparams *h)
{
    return h && h->step >= 1 && isfinite(h->lr) && isfinite(h->eps) && isfinite(h->weight_decay) &&
           isfinite(h->loss_scale) && h->loss_scale > 0.0 && h->beta1 >= 0.0 && h->beta1 < 1.0 &&
           h->beta2 >= 0.0 && h->beta2 < 1.0;
}

}  // namespace

extern "C" zero_status zero_step_noalloc(const zero_layout *L, const uint16_t *grads, int64_t rank_stride,
                                         float *master, float *m, float *v, uint16_t *p16_shard,
                                         uint16_t *p16_full, const zero_adamw_hparams *hp,
                                         int32_t *nonfinite, void *stream)
{
    if (!L || !hparams_ok(hp)) return ZERO_ERR_INVALID;
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
    // from the host, then the first-tile column from the device scan), so nothing left
    // over from an earlier call is ever read.  The host rows are pageable memory: the
    // copy has taken them by the time cudaMemcpyAsync returns.
    zero::Seg closing;
    closing.lo = closing.hi = L->padded;
    closing.tile_begin = -1;
    closing.shard = closing.bucket = -1;
    cudaError_t e = cudaMemcpyAsync(table, L->segs.data(), (size_t)n_seg * sizeof(zero::Seg),
                                    cudaMemcpyHostToDevice, st);
    if (e == cudaSuccess)
        e = cudaMemcpyAsync(table + n_seg, &closing, sizeof closing, cudaMemcpyHostToDevice, st);
    if (e == cudaSuccess) e = zero::launch_tile_index(table, n_seg, st);

    zero::AdamScalars c;
    const double t = (double)hp->step;
    c.inv_scale = (float)(1.0 / ((double)L->n_ranks * hp->loss_scale));
    c.decay = (float)(1.0 - hp->lr * hp->weight_decay);
    c.beta1 = (float)hp->beta1;
    c.omb1 = (float)(1.0 - hp->beta1);
    c.beta2 = (float)hp->beta2;
    c.omb2 = (float)(1.0 - hp->beta2);
    c.step_size = (float)(hp->lr / (1.0 - pow(hp->beta1, t)));
    c.sqrt_bc2 = (float)sqrt(1.0 - pow(hp->beta2, t));
    c.eps = (float)hp->eps;

    zero::TileWork w;
    w.segs = table;
    w.seg_first = 0;
    w.tile_first = 0;
    w.n_tiles = L->n_tiles;
    uint16_t *p16 = L->stage == 3 ? p16_shard : p16_full;
    if (e == cudaSuccess)
        e = zero::launch_fused_step(*L, w, grads, rank_stride, master, m, v, p16, c, nonfinite, st);
    if (e == cudaSuccess && L->stage == 3) e = zero::launch_copy_range(*L, 0, L->padded, p16_shard, p16_full, st);
    return e == cudaSuccess ? ZERO_OK : ZERO_ERR_CUDA;
}
