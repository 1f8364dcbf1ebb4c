// extern "C" entry points: argument checks, the AdamW step scalars, kernel launches.
#include <math.h>
#include <stdint.h>
#include <string.h>

#include <mutex>
#include <vector>

#include "gather_ranks.h"
#include "internal.h"

using zero::AdamScalars;
using zero::Seg;
using zero::TileWork;
using zero::check_hparams;
using zero::step_scalars;

namespace {

bool aligned16(const void *p) { return ((uintptr_t)p & 15u) == 0; }

bool finite_d(double x) { return isfinite(x) != 0; }

zero_status check_device(const zero_layout *L)
{
    if (!L) return ZERO_ERR_INVALID;
    if (L->dev.device < 0 || !L->dev.segs) return ZERO_ERR_STATE;
    int cur = -1;
    if (cudaGetDevice(&cur) != cudaSuccess) return ZERO_ERR_CUDA;
    return cur == L->dev.device ? ZERO_OK : ZERO_ERR_STATE;
}

zero_status cuda_status(cudaError_t e) { return e == cudaSuccess ? ZERO_OK : ZERO_ERR_CUDA; }

cudaError_t reduce(const zero_layout *L, const TileWork &w, const uint16_t *grads, int64_t stride, float *reduced,
                   int32_t *nonfinite, cudaStream_t st);   // defined with the step launchers below

TileWork all_tiles(const zero_layout *L)
{
    TileWork w;
    w.segs = L->dev.segs;
    w.seg_first = 0;
    w.tile_first = 0;
    w.n_tiles = L->n_tiles;
    w.bounds = zero::tile_bounds(*L, 0, L->padded);
    return w;
}

// The tiles of buckets [b0, b1): consecutive buckets' segments, and so their tiles, are
// contiguous in the bucket-major table.
TileWork bucket_range_tiles(const zero_layout *L, int64_t b0, int64_t b1)
{
    TileWork w;
    w.segs = L->dev.segs;
    w.seg_first = L->bucket_seg_begin[(size_t)b0];
    const int64_t seg_end = L->bucket_seg_begin[(size_t)b1];
    w.tile_first = L->segs[(size_t)w.seg_first].tile_begin;
    const int64_t tile_end = seg_end < (int64_t)L->segs.size() ? L->segs[(size_t)seg_end].tile_begin : L->n_tiles;
    w.n_tiles = tile_end - w.tile_first;
    w.bounds = zero::tile_bounds(*L, 0, L->padded);
    return w;
}

TileWork bucket_tiles(const zero_layout *L, int64_t b) { return bucket_range_tiles(L, b, b + 1); }

zero_status check_grads(const zero_layout *L, const void *grads, int64_t rank_stride)
{
    if (!grads) return ZERO_ERR_INVALID;
    if (rank_stride < L->padded) return ZERO_ERR_INVALID;
    if (!aligned16(grads) || rank_stride % 8 != 0) return ZERO_ERR_ALIGN;
    return ZERO_OK;
}

zero_status check_state(const float *master, const float *m, const float *v)
{
    if (!master || !m || !v) return ZERO_ERR_INVALID;
    if (!aligned16(master) || !aligned16(m) || !aligned16(v)) return ZERO_ERR_ALIGN;
    return ZERO_OK;
}

void release_device(zero_layout *L)
{
    if (L->dev.device < 0) return;
    int cur = -1;
    cudaGetDevice(&cur);
    if (cur != L->dev.device) cudaSetDevice(L->dev.device);
    for (cudaEvent_t e : L->dev.landed) cudaEventDestroy(e);
    for (cudaEvent_t e : L->dev.updated) cudaEventDestroy(e);
    L->dev.landed.clear();
    L->dev.updated.clear();
    if (L->dev.tuner.begin) cudaEventDestroy(L->dev.tuner.begin);
    if (L->dev.tuner.end) cudaEventDestroy(L->dev.tuner.end);
    if (L->dev.begin) cudaEventDestroy(L->dev.begin);
    if (L->dev.done) cudaEventDestroy(L->dev.done);
    if (L->dev.copy_in) cudaStreamDestroy(L->dev.copy_in);
    if (L->dev.copy_out) cudaStreamDestroy(L->dev.copy_out);
    if (L->dev.segs) cudaFree(L->dev.segs);
    if (L->dev.segs_by_shard) cudaFree(L->dev.segs_by_shard);
    if (L->dev.error) cudaFree(L->dev.error);
    if (cur >= 0 && cur != L->dev.device) cudaSetDevice(cur);
    L->dev = zero::DeviceState();
}

}  // namespace

namespace zero {

zero_status check_hparams(const zero_adamw_hparams *h)
{
    if (!h) return ZERO_ERR_INVALID;
    if (h->step < 1 || !finite_d(h->lr) || !finite_d(h->eps) || !finite_d(h->weight_decay) ||
        !finite_d(h->loss_scale) || !(h->loss_scale > 0.0) || !(h->beta1 >= 0.0 && h->beta1 < 1.0) ||
        !(h->beta2 >= 0.0 && h->beta2 < 1.0))
        return ZERO_ERR_INVALID;
    return ZERO_OK;
}

// The step's fp32 scalars, each evaluated in double and rounded once.
AdamScalars step_scalars(int32_t n_ranks, const zero_adamw_hparams &h)
{
    AdamScalars c;
    const double t = (double)h.step;
    c.inv_scale = (float)(1.0 / ((double)n_ranks * h.loss_scale));
    c.decay = (float)(1.0 - h.lr * h.weight_decay);
    c.beta1 = (float)h.beta1;
    c.omb1 = (float)(1.0 - h.beta1);
    c.beta2 = (float)h.beta2;
    c.omb2 = (float)(1.0 - h.beta2);
    c.step_size = (float)(h.lr / (1.0 - pow(h.beta1, t)));
    c.sqrt_bc2 = (float)sqrt(1.0 - pow(h.beta2, t));
    c.eps = (float)h.eps;
    return c;
}

}  // namespace zero

extern "C" void zero_layout_destroy(zero_layout *L)
{
    if (!L) return;
    release_device(L);
    delete L;
}

extern "C" const char *zero_status_string(zero_status s)
{
    switch (s) {
        case ZERO_OK: return "ok";
        case ZERO_ERR_INVALID: return "invalid argument";
        case ZERO_ERR_ALIGN: return "misaligned pointer or stride (need 16-byte pointers, strides multiple of 8)";
        case ZERO_ERR_CUDA: return "CUDA error";
        case ZERO_ERR_OOM: return "out of memory";
        case ZERO_ERR_TIMEOUT: return "a bounded wait in a kernel timed out";
        case ZERO_ERR_STATE: return "layout not uploaded to the current device";
        case ZERO_ERR_BOUNDS: return "a kernel found a segment or tile index out of bounds (debug build)";
    }
    return "unknown status";
}

extern "C" zero_status zero_layout_to_device(zero_layout *L, void *stream)
{
    ZERO_RANGE("zero_layout_to_device");
    if (!L) return ZERO_ERR_INVALID;
    int cur = -1;
    if (cudaGetDevice(&cur) != cudaSuccess) return ZERO_ERR_CUDA;
    if (L->dev.device >= 0) return L->dev.device == cur ? ZERO_OK : ZERO_ERR_STATE;
    cudaStream_t st = (cudaStream_t)stream;
    zero::DeviceState &d = L->dev;
    d.device = cur;
    int optin = 0;
    if (cudaDeviceGetAttribute(&d.num_sms, cudaDevAttrMultiProcessorCount, cur) != cudaSuccess ||
        cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, cur) != cudaSuccess) {
        release_device(L);
        return ZERO_ERR_CUDA;
    }
    d.smem_optin = (size_t)optin;
    // rows 0..n_seg-1 from the host partitioner with the tile numbers left blank (-1):
    // the device builds them; row n_seg is the sentinel.
    std::vector<Seg> rows(L->segs);
    for (Seg &s : rows) s.tile_begin = -1;
    Seg sentinel;
    sentinel.lo = sentinel.hi = L->padded;
    sentinel.tile_begin = -1;
    sentinel.shard = sentinel.bucket = -1;
    rows.push_back(sentinel);
    std::vector<Seg> rows2(L->segs_by_shard);
    for (Seg &s : rows2) s.tile_begin = -1;
    rows2.push_back(sentinel);
    if (cudaMalloc(&d.segs, rows.size() * sizeof(Seg)) != cudaSuccess ||
        cudaMalloc(&d.segs_by_shard, rows2.size() * sizeof(Seg)) != cudaSuccess ||
        cudaMalloc(&d.error, sizeof(int32_t)) != cudaSuccess) {
        cudaGetLastError();
        release_device(L);
        return ZERO_ERR_OOM;
    }
    cudaError_t e = cudaMemcpyAsync(d.segs, rows.data(), rows.size() * sizeof(Seg), cudaMemcpyHostToDevice, st);
    if (e == cudaSuccess) e = cudaMemsetAsync(d.error, 0, sizeof(int32_t), st);
    if (e == cudaSuccess) e = zero::launch_tile_index(d.segs, (int64_t)L->segs.size(), st);
    if (e == cudaSuccess)
        e = cudaMemcpyAsync(d.segs_by_shard, rows2.data(), rows2.size() * sizeof(Seg), cudaMemcpyHostToDevice, st);
    if (e == cudaSuccess) e = zero::launch_tile_index(d.segs_by_shard, (int64_t)L->segs_by_shard.size(), st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&d.copy_in, cudaStreamNonBlocking);
    if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&d.copy_out, cudaStreamNonBlocking);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&d.begin, cudaEventDisableTiming);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&d.done, cudaEventDisableTiming);
    if (e == cudaSuccess) e = cudaEventCreate(&d.tuner.begin);     // timing events
    if (e == cudaSuccess) e = cudaEventCreate(&d.tuner.end);
    for (size_t b = 0; e == cudaSuccess && b < L->bucket_lo.size(); ++b) {
        cudaEvent_t a = nullptr, u = nullptr;
        e = cudaEventCreateWithFlags(&a, cudaEventDisableTiming);
        if (e == cudaSuccess) d.landed.push_back(a);
        if (e == cudaSuccess) e = cudaEventCreateWithFlags(&u, cudaEventDisableTiming);
        if (e == cudaSuccess) d.updated.push_back(u);
    }
    if (e != cudaSuccess) {
        release_device(L);
        return ZERO_ERR_CUDA;
    }
    return ZERO_OK;
}

extern "C" zero_status zero_layout_device_segments(const zero_layout *L, int64_t *out, void *stream)
{
    ZERO_RANGE("zero_layout_device_segments");
    zero_status s = check_device(L);
    if (s != ZERO_OK) return s;
    if (!out) return ZERO_ERR_INVALID;
    std::vector<Seg> rows(L->segs.size() + 1);
    cudaStream_t st = (cudaStream_t)stream;
    cudaError_t e = cudaMemcpyAsync(rows.data(), L->dev.segs, rows.size() * sizeof(Seg), cudaMemcpyDeviceToHost, st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) return ZERO_ERR_CUDA;
    for (size_t i = 0; i < rows.size(); ++i) {
        out[5 * i + 0] = rows[i].bucket;
        out[5 * i + 1] = rows[i].shard;
        out[5 * i + 2] = rows[i].lo;
        out[5 * i + 3] = rows[i].hi;
        out[5 * i + 4] = rows[i].tile_begin;
    }
    return ZERO_OK;
}

extern "C" zero_status zero_reduce_scatter(const zero_layout *L, int64_t bucket, const uint16_t *grads,
                                           int64_t rank_stride, float *reduced, int32_t *nonfinite,
                                           void *stream)
{
    ZERO_RANGE("zero_reduce_scatter");
    zero_status s = check_device(L);
    if (s != ZERO_OK) return s;
    if (bucket < -1 || bucket >= (int64_t)L->bucket_lo.size()) return ZERO_ERR_INVALID;
    if (L->padded == 0) return ZERO_OK;
    if ((s = check_grads(L, grads, rank_stride)) != ZERO_OK) return s;
    if (!reduced) return ZERO_ERR_INVALID;
    if (!aligned16(reduced)) return ZERO_ERR_ALIGN;
    const TileWork w = bucket < 0 ? all_tiles(L) : bucket_tiles(L, bucket);
    return cuda_status(reduce(L, w, grads, rank_stride, reduced, nonfinite,
                                                   (cudaStream_t)stream));
}

extern "C" zero_status zero_adamw_shard_step(const zero_layout *L, int32_t shard, const float *reduced,
                                             float *master, float *m, float *v, uint16_t *p16_out,
                                             const zero_adamw_hparams *hp, void *stream)
{
    ZERO_RANGE("zero_adamw_shard_step");
    zero_status s = check_device(L);
    if (s != ZERO_OK) return s;
    if (shard < -1 || shard >= L->n_ranks) return ZERO_ERR_INVALID;
    if ((s = check_hparams(hp)) != ZERO_OK) return s;
    if (L->padded == 0) return ZERO_OK;
    if ((s = check_state(master, m, v)) != ZERO_OK) return s;
    if (!reduced || !p16_out) return ZERO_ERR_INVALID;
    if (!aligned16(reduced) || !aligned16(p16_out)) return ZERO_ERR_ALIGN;
    const int64_t lo = shard < 0 ? 0 : (int64_t)shard * L->shard;
    const int64_t hi = shard < 0 ? L->padded : lo + L->shard;
    return cuda_status(zero::launch_adamw_range(*L, lo, hi, reduced, master, m, v, p16_out,
                                                step_scalars(L->n_ranks, *hp), (cudaStream_t)stream));
}

extern "C" zero_status zero_allgather(const zero_layout *L, int64_t unit, const uint16_t *p16_shard,
                                      uint16_t *p16_full, void *stream)
{
    ZERO_RANGE("zero_allgather");
    zero_status s = check_device(L);
    if (s != ZERO_OK) return s;
    if (unit < -1 || unit >= (int64_t)L->unit_lo.size()) return ZERO_ERR_INVALID;
    if (L->padded == 0) return ZERO_OK;
    if (!p16_shard || !p16_full) return ZERO_ERR_INVALID;
    if (!aligned16(p16_shard) || !aligned16(p16_full)) return ZERO_ERR_ALIGN;
    const int64_t lo = unit < 0 ? 0 : L->unit_lo[(size_t)unit];
    const int64_t hi = unit < 0 ? L->padded : L->unit_hi[(size_t)unit];
    return cuda_status(zero::launch_copy_range(*L, lo, hi, p16_shard, p16_full, (cudaStream_t)stream));
}

extern "C" zero_status zero_gather_unit(const zero_layout *L, int64_t unit, const uint16_t *p16_shard,
                                        uint16_t *dst, void *stream)
{
    ZERO_RANGE("zero_gather_unit");
    zero_status s = check_device(L);
    if (s != ZERO_OK) return s;
    if (unit < 0 || unit >= (int64_t)L->unit_lo.size() || !p16_shard || !dst) return ZERO_ERR_INVALID;
    if (!aligned16(p16_shard) || !aligned16(dst)) return ZERO_ERR_ALIGN;
    const int64_t lo = L->unit_lo[(size_t)unit];
    return cuda_status(zero::launch_gather_unit(p16_shard, lo, L->unit_hi[(size_t)unit] - lo, dst, L->gather_ctas,
                                                L->dev.error, L->dev.wait_limit_ns,
                                                (cudaStream_t)stream));
}

extern "C" zero_status zero_gather_unit_ranks(const zero_layout *L, int64_t unit, const uint16_t *const *rank_p16,
                                              uint16_t *dst, void *stream)
{
    ZERO_RANGE("zero_gather_unit_ranks");
    zero_status s = check_device(L);
    if (s != ZERO_OK) return s;
    if (unit < 0 || unit >= (int64_t)L->unit_lo.size() || !rank_p16 || !dst) return ZERO_ERR_INVALID;
    if (L->n_ranks > zero::kMaxBulkRanks) return ZERO_ERR_INVALID;
    zero::ShardPtrs src = {};
    for (int r = 0; r < L->n_ranks; ++r) {
        if (!rank_p16[r]) return ZERO_ERR_INVALID;
        if (!aligned16(rank_p16[r])) return ZERO_ERR_ALIGN;
        src.rank[r] = rank_p16[r];
    }
    if (!aligned16(dst)) return ZERO_ERR_ALIGN;
    const int64_t lo = L->unit_lo[(size_t)unit];
    return cuda_status(zero::launch_gather_ranks(src, L->shard, lo, L->unit_hi[(size_t)unit] - lo, dst,
                                                 L->gather_ctas, (cudaStream_t)stream));
}

namespace {

// The buffers of a whole-layout step (hyper-parameters checked separately).
zero_status check_step_buffers(const zero_layout *L, const uint16_t *grads, int64_t rank_stride, float *master,
                               float *m, float *v, uint16_t *p16_shard, uint16_t *p16_full)
{
    zero_status s = check_device(L);
    if (s != ZERO_OK) return s;
    if (L->padded == 0) return ZERO_OK;
    if ((s = check_grads(L, grads, rank_stride)) != ZERO_OK) return s;
    if ((s = check_state(master, m, v)) != ZERO_OK) return s;
    if (!p16_full || (L->stage == 3 && !p16_shard)) return ZERO_ERR_INVALID;
    if (!aligned16(p16_full) || (p16_shard && !aligned16(p16_shard))) return ZERO_ERR_ALIGN;
    return ZERO_OK;
}

zero_status check_step(const zero_layout *L, const uint16_t *grads, int64_t rank_stride, float *master,
                       float *m, float *v, uint16_t *p16_shard, uint16_t *p16_full,
                       const zero_adamw_hparams *hp)
{
    zero_status s = check_device(L);
    if (s != ZERO_OK) return s;
    if ((s = check_hparams(hp)) != ZERO_OK) return s;
    return check_step_buffers(L, grads, rank_stride, master, m, v, p16_shard, p16_full);
}

void record(void *ev, cudaStream_t st)
{
    if (ev) cudaEventRecord((cudaEvent_t)ev, st);
}

// Rank r's gradients at grads + r * stride.
zero::GradSource strided(const zero_layout *L, const uint16_t *grads, int64_t stride)
{
    zero::GradSource src = {};
    for (int r = 0; r < L->n_ranks && r < zero::kMaxBulkRanks; ++r) src.rank[r] = grads + (int64_t)r * stride;
    return src;
}

// The reduce-scatter alone over the tiles of `w`, in the selected implementation (the
// automatic choice measured for this pass; results identical either way).
cudaError_t reduce(const zero_layout *L, const TileWork &w, const uint16_t *grads, int64_t stride, float *reduced,
                   int32_t *nonfinite, cudaStream_t st)
{
    if (zero::use_bulk_reduce(*L))
        return zero::launch_bulk_reduce(*L, w, strided(L, grads, stride), reduced, nonfinite, L->dev.wait_limit_ns,
                                        st);
    return zero::launch_reduce_scatter(*L, w, grads, stride, reduced, nonfinite, st);
}

// The fused reduce-scatter + update over the tiles of `w`, in the selected implementation.
cudaError_t fused(const zero_layout *L, const TileWork &w, const uint16_t *grads, int64_t stride, float *master,
                  float *m, float *v, uint16_t *p16, const AdamScalars &c, int32_t *nonfinite, cudaStream_t st,
                  const AdamScalars *c_dev = nullptr)
{
    const bool bulk = zero::use_bulk(*L);
    if (bulk)
        return zero::launch_bulk_step(*L, w, strided(L, grads, stride), master, m, v, 0, p16, 0, c, nonfinite,
                                      L->dev.wait_limit_ns, L->dev.skip_first_fill, st, nullptr, nullptr, nullptr,
                                      c_dev);
    return zero::launch_fused_step(*L, w, grads, stride, master, m, v, p16, c, nonfinite, st, c_dev);
}

}  // namespace

extern "C" zero_status zero_step(const zero_layout *L, const uint16_t *grads, int64_t rank_stride,
                                 float *master, float *m, float *v, uint16_t *p16_shard,
                                 uint16_t *p16_full, const zero_adamw_hparams *hp,
                                 int32_t *nonfinite, const zero_step_events *ev, void *stream)
{
    ZERO_RANGE("zero_step");
    zero_status s = check_step(L, grads, rank_stride, master, m, v, p16_shard, p16_full, hp);
    if (s != ZERO_OK || L->padded == 0) return s;
    cudaStream_t st = (cudaStream_t)stream;
    const AdamScalars c = step_scalars(L->n_ranks, *hp);
    uint16_t *p16 = L->stage == 3 ? p16_shard : p16_full;
    if (ev) record(ev->update_begin, st);
    cudaError_t e = fused(L, all_tiles(L), grads, rank_stride, master, m, v, p16, c, nonfinite, st);
    if (ev) record(ev->update_end, st);
    if (e == cudaSuccess && L->stage == 3) {
        if (ev) record(ev->gather_begin, st);
        e = zero::launch_copy_range(*L, 0, L->padded, p16_shard, p16_full, st);
        if (ev) record(ev->gather_end, st);
    }
    return cuda_status(e);
}

extern "C" zero_status zero_step_scalars_fill(const zero_layout *L, const zero_adamw_hparams *hp,
                                              zero_step_scalars *out)
{
    ZERO_RANGE("zero_step_scalars_fill");
    if (!L || !out) return ZERO_ERR_INVALID;
    zero_status s = check_hparams(hp);
    if (s != ZERO_OK) return s;
    const AdamScalars c = step_scalars(L->n_ranks, *hp);
    memcpy(out, &c, sizeof c);
    return ZERO_OK;
}

extern "C" zero_status zero_step_device_scalars(const zero_layout *L, const uint16_t *grads, int64_t rank_stride,
                                                float *master, float *m, float *v, uint16_t *p16_shard,
                                                uint16_t *p16_full, const zero_step_scalars *scalars_dev,
                                                int32_t *nonfinite, void *stream)
{
    ZERO_RANGE("zero_step_device_scalars");
    // the hyper-parameter rules of zero_step apply to whoever filled *scalars_dev
    zero_status s = check_step_buffers(L, grads, rank_stride, master, m, v, p16_shard, p16_full);
    if (s != ZERO_OK || L->padded == 0) return s;
    if (!scalars_dev) return ZERO_ERR_INVALID;
    if (((uintptr_t)scalars_dev & 3u) != 0) return ZERO_ERR_ALIGN;
    cudaStream_t st = (cudaStream_t)stream;
    const AdamScalars *c_dev = reinterpret_cast<const AdamScalars *>(scalars_dev);
    uint16_t *p16 = L->stage == 3 ? p16_shard : p16_full;
    cudaError_t e = fused(L, all_tiles(L), grads, rank_stride, master, m, v, p16, AdamScalars{}, nonfinite, st,
                          c_dev);
    if (e == cudaSuccess && L->stage == 3) e = zero::launch_copy_range(*L, 0, L->padded, p16_shard, p16_full, st);
    return cuda_status(e);
}

extern "C" zero_status zero_step_bucket(const zero_layout *L, int64_t bucket, const uint16_t *grads,
                                        int64_t rank_stride, float *master, float *m, float *v,
                                        uint16_t *p16_shard, uint16_t *p16_full, const zero_adamw_hparams *hp,
                                        int32_t *nonfinite, void *stream)
{
    ZERO_RANGE("zero_step_bucket");
    zero_status s = check_step(L, grads, rank_stride, master, m, v, p16_shard, p16_full, hp);
    if (s != ZERO_OK || L->padded == 0) return s;
    if (bucket < 0 || bucket >= (int64_t)L->bucket_lo.size()) return ZERO_ERR_INVALID;
    uint16_t *p16 = L->stage == 3 ? p16_shard : p16_full;
    return cuda_status(fused(L, bucket_tiles(L, bucket), grads, rank_stride, master, m, v, p16,
                             step_scalars(L->n_ranks, *hp), nonfinite, (cudaStream_t)stream));
}

namespace {

// Launches of at least this many elements when zero_step_overlapped coalesces small
// buckets (~0.5-1 GB of traffic, 80-150 us at full bandwidth: launch gaps stay negligible).
constexpr int64_t kMinOverlapLaunch = int64_t(1) << 24;

// Candidate plan i of the overlapped step's tuner: i < 4 follows the backward with the
// update's grid capped at SMs x {1, 2/3, 1/2, 1/3} (0 = no cap); i == 4 defers the whole
// update to one full-grid launch after the last bucket's event.
constexpr int kDeferred = 4;
static_assert(kDeferred + 1 == zero::OverlapTuner::kCands, "one plan per tuner candidate");
static_assert(zero::OverlapTuner::kCands == ZERO_OVERLAP_PLANS, "zero_overlap_plan fills ZERO_OVERLAP_PLANS means");

int32_t tuner_cap(const zero_layout *L, int i)
{
    static const int kSixths[4] = {6, 4, 3, 2};
    const int sms = L->dev.num_sms > 0 ? L->dev.num_sms : 148;
    return (i == 0 || i == kDeferred) ? 0 : sms * kSixths[i] / 6;
}

struct OverlapPlan {
    int32_t cap = 0;          // grid cap of every launch (0 = full grid)
    bool deferred = false;    // one launch after every bucket's event
    bool timed = false;       // record the tuner's events around this call
};

// The plan of this overlapped call: the caller's cap (zero_set_max_ctas) if set;
// otherwise the tuner's.  Harvests the previous timed call if its end event has
// completed (never waits), then times the next candidate in round-robin order that
// still lacks trials, or keeps the one with the lowest mean.
OverlapPlan overlap_plan(const zero_layout *L)
{
    OverlapPlan p;
    zero::OverlapTuner &T = L->dev.tuner;
    if (L->max_ctas > 0 || !T.begin || !T.end) {
        p.cap = L->max_ctas;
        return p;
    }
    const int K = zero::OverlapTuner::kCands;
    if (T.pending >= 0) {
        if (cudaEventQuery(T.end) != cudaSuccess) {            // still running: same plan, untimed
            p.cap = tuner_cap(L, T.pending);
            p.deferred = T.pending == kDeferred;
            return p;
        }
        float ms = 0.f;
        if (cudaEventElapsedTime(&ms, T.begin, T.end) == cudaSuccess) {
            T.sum_ms[T.pending] += ms;
            ++T.trials[T.pending];
        }
        T.pending = -1;
    }
    int pick = T.chosen;
    if (pick < 0 && T.calls++ > 0) {                           // the first call is a warm-up
        // the candidate with the fewest trials; rounds alternate direction (0..K-1, then
        // K-1..0), so that a steady drift of the clocks while the GPU warms up adds the
        // same to every candidate's sum
        int fewest = -1;
        for (int k = 0; k < K; ++k) {
            int lo = K;
            for (int i = 0; i < K; ++i) lo = T.trials[i] < lo ? T.trials[i] : lo;
            const int i = (lo % 2 == 0) ? k : K - 1 - k;
            if (T.trials[i] == lo) {
                fewest = i;
                break;
            }
        }
        if (T.trials[fewest] < zero::OverlapTuner::kTrials) {
            T.pending = fewest;
            p.timed = true;
            pick = fewest;
        } else {
            int best = 0;
            for (int i = 1; i < K; ++i)
                if (T.sum_ms[i] < T.sum_ms[best]) best = i;
            T.chosen = pick = best;
        }
    }
    if (pick < 0) pick = 0;
    p.cap = tuner_cap(L, pick);
    p.deferred = pick == kDeferred;
    return p;
}

// The overlapped step over launch groups: launch j covers buckets [first[j], first[j+1]).
zero_status overlapped(const zero_layout *L, void *const *ready_events, const std::vector<int64_t> &first,
                       const uint16_t *grads, int64_t rank_stride, float *master, float *m, float *v,
                       uint16_t *p16_shard, uint16_t *p16_full, const zero_adamw_hparams *hp, int32_t *nonfinite,
                       cudaStream_t st)
{
    const AdamScalars c = step_scalars(L->n_ranks, *hp);
    uint16_t *p16 = L->stage == 3 ? p16_shard : p16_full;
    const OverlapPlan plan = overlap_plan(L);
    const std::vector<int64_t> all = {0, (int64_t)L->bucket_lo.size()};
    const std::vector<int64_t> &launches = plan.deferred ? all : first;
    cudaError_t e = plan.timed ? cudaEventRecord(L->dev.tuner.begin, st) : cudaSuccess;
    for (size_t j = 0; e == cudaSuccess && j + 1 < launches.size(); ++j) {
        for (int64_t b = launches[j]; e == cudaSuccess && b < launches[j + 1]; ++b)
            e = cudaStreamWaitEvent(st, (cudaEvent_t)ready_events[b], 0);
        TileWork w = bucket_range_tiles(L, launches[j], launches[j + 1]);
        w.max_ctas = plan.cap;
        if (e == cudaSuccess) e = fused(L, w, grads, rank_stride, master, m, v, p16, c, nonfinite, st);
    }
    if (e == cudaSuccess && L->stage == 3) e = zero::launch_copy_range(*L, 0, L->padded, p16_shard, p16_full, st);
    if (e == cudaSuccess && plan.timed) e = cudaEventRecord(L->dev.tuner.end, st);
    if (e != cudaSuccess && plan.timed) L->dev.tuner.pending = -1;
    return cuda_status(e);
}

zero_status check_overlapped(const zero_layout *L, void *const *ready_events, const uint16_t *grads,
                             int64_t rank_stride, float *master, float *m, float *v, uint16_t *p16_shard,
                             uint16_t *p16_full, const zero_adamw_hparams *hp)
{
    zero_status s = check_step(L, grads, rank_stride, master, m, v, p16_shard, p16_full, hp);
    if (s != ZERO_OK || L->padded == 0) return s;
    if (!ready_events) return ZERO_ERR_INVALID;
    for (size_t b = 0; b < L->bucket_lo.size(); ++b)
        if (!ready_events[b]) return ZERO_ERR_INVALID;
    return ZERO_OK;
}

}  // namespace

extern "C" zero_status zero_overlap_plan(const zero_layout *L, int32_t *plan, float *mean_ms)
{
    ZERO_RANGE("zero_overlap_plan");
    if (!L || !plan) return ZERO_ERR_INVALID;
    const zero::OverlapTuner &T = L->dev.tuner;
    *plan = L->max_ctas > 0 ? -1 : T.chosen;
    if (mean_ms)
        for (int i = 0; i < zero::OverlapTuner::kCands; ++i)
            mean_ms[i] = T.trials[i] > 0 ? T.sum_ms[i] / (float)T.trials[i] : 0.f;
    return ZERO_OK;
}

extern "C" zero_status zero_step_overlapped_grouped(const zero_layout *L, void *const *ready_events, int64_t group,
                                                    const uint16_t *grads, int64_t rank_stride, float *master, float *m,
                                                    float *v, uint16_t *p16_shard, uint16_t *p16_full,
                                                    const zero_adamw_hparams *hp, int32_t *nonfinite, void *stream)
{
    ZERO_RANGE("zero_step_overlapped_grouped");
    if (group < 1) return ZERO_ERR_INVALID;
    zero_status s = check_overlapped(L, ready_events, grads, rank_stride, master, m, v, p16_shard, p16_full, hp);
    if (s != ZERO_OK || L->padded == 0) return s;
    const int64_t nb = (int64_t)L->bucket_lo.size();
    std::vector<int64_t> first;
    for (int64_t b = 0; b < nb; b += group) first.push_back(b);
    first.push_back(nb);
    return overlapped(L, ready_events, first, grads, rank_stride, master, m, v, p16_shard, p16_full, hp, nonfinite,
                      (cudaStream_t)stream);
}

extern "C" zero_status zero_step_overlapped(const zero_layout *L, void *const *ready_events, const uint16_t *grads,
                                            int64_t rank_stride, float *master, float *m, float *v,
                                            uint16_t *p16_shard, uint16_t *p16_full, const zero_adamw_hparams *hp,
                                            int32_t *nonfinite, void *stream)
{
    ZERO_RANGE("zero_step_overlapped");
    zero_status s = check_overlapped(L, ready_events, grads, rank_stride, master, m, v, p16_shard, p16_full, hp);
    if (s != ZERO_OK || L->padded == 0) return s;
    // one launch per bucket, except that consecutive buckets smaller than kMinOverlapLaunch
    // share a launch until they reach it (a launch waits for all of its buckets)
    const int64_t nb = (int64_t)L->bucket_lo.size();
    std::vector<int64_t> first;
    int64_t acc = 0;
    for (int64_t b = 0; b < nb; ++b) {
        if (acc == 0) first.push_back(b);
        acc += L->bucket_hi[(size_t)b] - L->bucket_lo[(size_t)b];
        if (acc >= kMinOverlapLaunch) acc = 0;
    }
    first.push_back(nb);
    return overlapped(L, ready_events, first, grads, rank_stride, master, m, v, p16_shard, p16_full, hp, nonfinite,
                      (cudaStream_t)stream);
}

namespace {

bool scaler_valid(const zero_loss_scaler *sc)
{
    return sc->scale > 0.0 && finite_d(sc->scale) && sc->factor > 1.0 && finite_d(sc->factor) && sc->window >= 1 &&
           sc->min_scale > 0.0 && finite_d(sc->min_scale) && sc->step >= 0;
}

// After a step: an applied one counts towards the growth window; a skipped one backs off.
void scaler_advance(zero_loss_scaler *sc, bool applied)
{
    if (applied) {
        sc->step += 1;
        sc->clean_steps += 1;
        if (sc->clean_steps == sc->window) {
            sc->scale *= sc->factor;
            sc->clean_steps = 0;
        }
    } else {
        const double lowered = sc->scale / sc->factor;
        sc->scale = lowered > sc->min_scale ? lowered : sc->min_scale;
        sc->clean_steps = 0;
        sc->skipped += 1;
    }
}

// The per-bucket counts back on the host (synchronises the stream); their sum.
cudaError_t total_nonfinite(const zero_layout *L, const int32_t *nonfinite, cudaStream_t st, int64_t *bad)
{
    std::vector<int32_t> counts(L->bucket_lo.size(), 0);
    cudaError_t e = cudaMemcpyAsync(counts.data(), nonfinite, counts.size() * sizeof(int32_t),
                                    cudaMemcpyDeviceToHost, st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    *bad = 0;
    for (int32_t c : counts) *bad += c;
    return e;
}

bool overlaps(const void *a, const void *b, int64_t bytes)
{
    const uintptr_t x = (uintptr_t)a, y = (uintptr_t)b;
    return x < y + (uintptr_t)bytes && y < x + (uintptr_t)bytes;
}

}  // namespace

extern "C" zero_status zero_step_dynamic(const zero_layout *L, const uint16_t *grads, int64_t rank_stride,
                                         float *reduced, float *master, float *m, float *v, uint16_t *p16_shard,
                                         uint16_t *p16_full, const zero_adamw_hparams *hp, zero_loss_scaler *sc,
                                         int32_t *nonfinite, int32_t *applied, void *stream)
{
    ZERO_RANGE("zero_step_dynamic");
    if (!L || !hp || !sc || !applied) return ZERO_ERR_INVALID;
    if (!scaler_valid(sc)) return ZERO_ERR_INVALID;
    zero_adamw_hparams h = *hp;
    h.loss_scale = sc->scale;
    h.step = sc->step + 1;
    zero_status s = check_step(L, grads, rank_stride, master, m, v, p16_shard, p16_full, &h);
    if (s != ZERO_OK) return s;
    *applied = 0;
    if (L->padded == 0) return ZERO_OK;
    if (!reduced || !nonfinite) return ZERO_ERR_INVALID;
    if (!aligned16(reduced)) return ZERO_ERR_ALIGN;
    cudaStream_t st = (cudaStream_t)stream;
    const size_t nb = L->bucket_lo.size();
    int64_t bad = 0;
    cudaError_t e = cudaMemsetAsync(nonfinite, 0, nb * sizeof(int32_t), st);
    if (e == cudaSuccess) e = reduce(L, all_tiles(L), grads, rank_stride, reduced, nonfinite, st);
    if (e == cudaSuccess) e = total_nonfinite(L, nonfinite, st, &bad);
    if (e != cudaSuccess) return ZERO_ERR_CUDA;
    if (bad == 0) {
        uint16_t *p16 = L->stage == 3 ? p16_shard : p16_full;
        e = zero::launch_adamw_range(*L, 0, L->padded, reduced, master, m, v, p16, step_scalars(L->n_ranks, h), st);
        if (e == cudaSuccess && L->stage == 3) e = zero::launch_copy_range(*L, 0, L->padded, p16_shard, p16_full, st);
        if (e != cudaSuccess) return ZERO_ERR_CUDA;
        *applied = 1;
    }
    scaler_advance(sc, bad == 0);
    return ZERO_OK;
}

extern "C" zero_status zero_step_dynamic_commit(const zero_layout *L, const uint16_t *grads, int64_t rank_stride,
                                                const float *master_in, const float *m_in, const float *v_in,
                                                float *master_out, float *m_out, float *v_out, uint16_t *p16_out,
                                                uint16_t *p16_full, const zero_adamw_hparams *hp,
                                                zero_loss_scaler *sc, int32_t *nonfinite, int32_t *applied,
                                                void *stream)
{
    ZERO_RANGE("zero_step_dynamic_commit");
    if (!L || !hp || !sc || !applied) return ZERO_ERR_INVALID;
    if (!scaler_valid(sc)) return ZERO_ERR_INVALID;
    zero_adamw_hparams h = *hp;
    h.loss_scale = sc->scale;
    h.step = sc->step + 1;
    // the out set goes through the usual step checks; the in set is checked alike here
    zero_status s = check_step(L, grads, rank_stride, master_out, m_out, v_out, p16_out,
                               L->stage == 3 ? p16_full : p16_out, &h);
    if (s != ZERO_OK) return s;
    *applied = 0;
    if (L->padded == 0) return ZERO_OK;
    if ((s = check_state(master_in, m_in, v_in)) != ZERO_OK) return s;
    if (!nonfinite) return ZERO_ERR_INVALID;
    const int64_t fb = L->padded * 4;
    const float *ins[3] = {master_in, m_in, v_in};
    const float *outs[3] = {master_out, m_out, v_out};
    for (const float *a : ins)
        for (const float *b : outs)
            if (overlaps(a, b, fb)) return ZERO_ERR_INVALID;
    cudaStream_t st = (cudaStream_t)stream;
    int64_t bad = 0;
    cudaError_t e = cudaMemsetAsync(nonfinite, 0, L->bucket_lo.size() * sizeof(int32_t), st);
    const bool bulk = zero::use_bulk(*L);
    if (e == cudaSuccess && bulk)
        e = zero::launch_bulk_step(*L, all_tiles(L), strided(L, grads, rank_stride), master_out, m_out, v_out, 0,
                                   p16_out, 0, step_scalars(L->n_ranks, h), nonfinite, L->dev.wait_limit_ns,
                                   L->dev.skip_first_fill, st, master_in, m_in, v_in);
    else if (e == cudaSuccess)
        e = zero::launch_fused_step_to(*L, all_tiles(L), grads, rank_stride, master_in, m_in, v_in, master_out,
                                       m_out, v_out, p16_out, step_scalars(L->n_ranks, h), nonfinite, st);
    if (e == cudaSuccess) e = total_nonfinite(L, nonfinite, st, &bad);
    if (e != cudaSuccess) return ZERO_ERR_CUDA;
    if (bad == 0) {
        if (L->stage == 3 && zero::launch_copy_range(*L, 0, L->padded, p16_out, p16_full, st) != cudaSuccess)
            return ZERO_ERR_CUDA;
        *applied = 1;
    }
    scaler_advance(sc, bad == 0);
    return ZERO_OK;
}

namespace {

TileWork shard_tiles(const zero_layout *L, int64_t k)
{
    TileWork w;
    w.segs = L->dev.segs_by_shard;
    w.seg_first = L->shard_seg_begin[(size_t)k];
    const int64_t seg_end = L->shard_seg_begin[(size_t)k + 1];
    w.tile_first = w.seg_first < (int64_t)L->segs_by_shard.size() ? L->segs_by_shard[(size_t)w.seg_first].tile_begin
                                                                    : L->n_tiles;
    const int64_t tile_end =
        seg_end < (int64_t)L->segs_by_shard.size() ? L->segs_by_shard[(size_t)seg_end].tile_begin : L->n_tiles;
    w.n_tiles = tile_end - w.tile_first;
    w.bounds = zero::tile_bounds(*L, k * L->shard, (k + 1) * L->shard);   // shard-local state
    return w;
}

zero_status rank_source(const zero_layout *L, const uint16_t *const *rank_grads, zero::GradSource *src)
{
    if (!rank_grads) return ZERO_ERR_INVALID;
    if (L->n_ranks > zero::kMaxBulkRanks) return ZERO_ERR_INVALID;
    *src = {};
    for (int r = 0; r < L->n_ranks; ++r) {
        if (!rank_grads[r]) return ZERO_ERR_INVALID;
        if (!aligned16(rank_grads[r])) return ZERO_ERR_ALIGN;
        src->rank[r] = rank_grads[r];
    }
    return ZERO_OK;
}

}  // namespace

extern "C" zero_status zero_step_ranks(const zero_layout *L, const uint16_t *const *rank_grads, float *master,
                                       float *m, float *v, uint16_t *p16_shard, uint16_t *p16_full,
                                       const zero_adamw_hparams *hp, int32_t *nonfinite, void *stream)
{
    ZERO_RANGE("zero_step_ranks");
    zero_status s = check_device(L);
    if (s != ZERO_OK) return s;
    if ((s = check_hparams(hp)) != ZERO_OK) return s;
    if (L->padded == 0) return ZERO_OK;
    zero::GradSource src;
    if ((s = rank_source(L, rank_grads, &src)) != ZERO_OK) return s;
    if ((s = check_state(master, m, v)) != ZERO_OK) return s;
    if (!p16_full || (L->stage == 3 && !p16_shard)) return ZERO_ERR_INVALID;
    if (!aligned16(p16_full) || (p16_shard && !aligned16(p16_shard))) return ZERO_ERR_ALIGN;
    cudaStream_t st = (cudaStream_t)stream;
    uint16_t *p16 = L->stage == 3 ? p16_shard : p16_full;
    cudaError_t e = zero::launch_bulk_step(*L, all_tiles(L), src, master, m, v, 0, p16, 0,
                                           step_scalars(L->n_ranks, *hp), nonfinite, L->dev.wait_limit_ns,
                                           L->dev.skip_first_fill, st);
    if (e == cudaSuccess && L->stage == 3) e = zero::launch_copy_range(*L, 0, L->padded, p16_shard, p16_full, st);
    return cuda_status(e);
}

extern "C" zero_status zero_step_shard(const zero_layout *L, int32_t shard, const uint16_t *const *rank_grads,
                                       float *master_k, float *m_k, float *v_k, uint16_t *p16_out,
                                       const zero_adamw_hparams *hp, int32_t *nonfinite, void *stream)
{
    ZERO_RANGE("zero_step_shard");
    zero_status s = check_device(L);
    if (s != ZERO_OK) return s;
    if ((s = check_hparams(hp)) != ZERO_OK) return s;
    if (shard < 0 || shard >= L->n_ranks) return ZERO_ERR_INVALID;
    if (L->padded == 0) return ZERO_OK;
    if (L->shard % 8 != 0) return ZERO_ERR_ALIGN;
    zero::GradSource src;
    if ((s = rank_source(L, rank_grads, &src)) != ZERO_OK) return s;
    if ((s = check_state(master_k, m_k, v_k)) != ZERO_OK) return s;
    if (!p16_out) return ZERO_ERR_INVALID;
    if (!aligned16(p16_out)) return ZERO_ERR_ALIGN;
    const int64_t off = (int64_t)shard * L->shard;
    return cuda_status(zero::launch_bulk_step(*L, shard_tiles(L, shard), src, master_k, m_k, v_k, off, p16_out,
                                              L->stage == 3 ? off : 0, step_scalars(L->n_ranks, *hp), nonfinite,
                                              L->dev.wait_limit_ns, L->dev.skip_first_fill, (cudaStream_t)stream));
}

extern "C" zero_status zero_step_shard_commit(const zero_layout *L, int32_t shard, const uint16_t *const *rank_grads,
                                              const float *master_in, const float *m_in, const float *v_in,
                                              float *master_out, float *m_out, float *v_out, uint16_t *p16_out,
                                              const zero_adamw_hparams *hp, const zero_loss_scaler *sc,
                                              int32_t *nonfinite, int64_t *nonfinite_total, void *stream)
{
    ZERO_RANGE("zero_step_shard_commit");
    if (!L || !hp || !sc || !nonfinite_total) return ZERO_ERR_INVALID;
    if (!scaler_valid(sc)) return ZERO_ERR_INVALID;
    zero_status s = check_device(L);
    if (s != ZERO_OK) return s;
    zero_adamw_hparams h = *hp;
    h.loss_scale = sc->scale;
    h.step = sc->step + 1;
    if ((s = check_hparams(&h)) != ZERO_OK) return s;
    if (shard < 0 || shard >= L->n_ranks) return ZERO_ERR_INVALID;
    *nonfinite_total = 0;
    if (L->padded == 0) return ZERO_OK;
    if (L->shard % 8 != 0) return ZERO_ERR_ALIGN;
    zero::GradSource src;
    if ((s = rank_source(L, rank_grads, &src)) != ZERO_OK) return s;
    if ((s = check_state(master_in, m_in, v_in)) != ZERO_OK) return s;
    if ((s = check_state(master_out, m_out, v_out)) != ZERO_OK) return s;
    if (!p16_out || !nonfinite) return ZERO_ERR_INVALID;
    if (!aligned16(p16_out)) return ZERO_ERR_ALIGN;
    const int64_t fb = L->shard * 4;
    const float *ins[3] = {master_in, m_in, v_in};
    const float *outs[3] = {master_out, m_out, v_out};
    for (const float *a : ins)
        for (const float *b : outs)
            if (overlaps(a, b, fb)) return ZERO_ERR_INVALID;
    cudaStream_t st = (cudaStream_t)stream;
    const int64_t off = (int64_t)shard * L->shard;
    cudaError_t e = cudaMemsetAsync(nonfinite, 0, L->bucket_lo.size() * sizeof(int32_t), st);
    if (e == cudaSuccess)
        e = zero::launch_bulk_step(*L, shard_tiles(L, shard), src, master_out, m_out, v_out, off, p16_out,
                                   L->stage == 3 ? off : 0, step_scalars(L->n_ranks, h), nonfinite,
                                   L->dev.wait_limit_ns, L->dev.skip_first_fill, st, master_in, m_in, v_in);
    if (e == cudaSuccess) e = total_nonfinite(L, nonfinite, st, nonfinite_total);
    return cuda_status(e);
}

extern "C" zero_status zero_loss_scaler_advance(zero_loss_scaler *sc, int32_t applied)
{
    ZERO_RANGE("zero_loss_scaler_advance");
    if (!sc || !scaler_valid(sc) || applied < 0 || applied > 1) return ZERO_ERR_INVALID;
    scaler_advance(sc, applied == 1);
    return ZERO_OK;
}

extern "C" zero_status zero_copy_shard(const zero_layout *L, int32_t shard, const uint16_t *src, uint16_t *dst,
                                       void *stream)
{
    ZERO_RANGE("zero_copy_shard");
    zero_status s = check_device(L);
    if (s != ZERO_OK) return s;
    if (shard < 0 || shard >= L->n_ranks || !src || !dst) return ZERO_ERR_INVALID;
    if (!aligned16(src) || !aligned16(dst)) return ZERO_ERR_ALIGN;
    const int64_t lo = (int64_t)shard * L->shard;
    return cuda_status(zero::launch_copy_range(*L, lo, lo + L->shard, src, dst, (cudaStream_t)stream));
}

namespace {

// cuMemGetAddressRange (driver API), fetched at run time so that the library does not
// link against the driver library: it finds the allocation a device pointer lies in.
typedef int (*MemRangeFn)(unsigned long long *base, size_t *size, unsigned long long ptr);

MemRangeFn mem_range_fn()
{
    static MemRangeFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuMemGetAddressRange", &p, 12000, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<MemRangeFn>(p);
    });
    return fn;
}

}  // namespace

extern "C" zero_status zero_ipc_get_handle(const void *dev_ptr, void *handle_out, int64_t *offset_out)
{
    ZERO_RANGE("zero_ipc_get_handle");
    if (!dev_ptr || !handle_out || !offset_out) return ZERO_ERR_INVALID;
    MemRangeFn range = mem_range_fn();
    if (!range) return ZERO_ERR_CUDA;
    unsigned long long base = 0;
    size_t size = 0;
    if (range(&base, &size, (unsigned long long)(uintptr_t)dev_ptr) != 0) return ZERO_ERR_CUDA;
    cudaIpcMemHandle_t h;
    if (cudaIpcGetMemHandle(&h, (void *)(uintptr_t)base) != cudaSuccess) return ZERO_ERR_CUDA;
    static_assert(sizeof(h) == 64, "CUDA IPC handles are 64 bytes");
    memcpy(handle_out, &h, sizeof h);
    *offset_out = (int64_t)((uintptr_t)dev_ptr - (uintptr_t)base);
    return ZERO_OK;
}

extern "C" zero_status zero_ipc_open(const void *handle, int64_t offset, void **dev_ptr_out)
{
    ZERO_RANGE("zero_ipc_open");
    if (!handle || !dev_ptr_out || offset < 0) return ZERO_ERR_INVALID;
    cudaIpcMemHandle_t h;
    memcpy(&h, handle, sizeof h);
    void *base = nullptr;
    *dev_ptr_out = nullptr;
    if (cudaIpcOpenMemHandle(&base, h, cudaIpcMemLazyEnablePeerAccess) != cudaSuccess) return ZERO_ERR_CUDA;
    *dev_ptr_out = static_cast<char *>(base) + offset;
    return ZERO_OK;
}

extern "C" zero_status zero_ipc_close(void *dev_ptr, int64_t offset)
{
    ZERO_RANGE("zero_ipc_close");
    if (!dev_ptr || offset < 0) return ZERO_ERR_INVALID;
    return cudaIpcCloseMemHandle(static_cast<char *>(dev_ptr) - offset) == cudaSuccess ? ZERO_OK : ZERO_ERR_CUDA;
}

extern "C" zero_status zero_step_host(const zero_layout *L, const uint16_t *grads_host, uint16_t *grads_dev,
                                      int64_t rank_stride, float *master, float *m, float *v,
                                      uint16_t *p16_shard, uint16_t *p16_full, uint16_t *p16_host,
                                      const zero_adamw_hparams *hp, int32_t *nonfinite, void *stream)
{
    ZERO_RANGE("zero_step_host");
    zero_status s = check_step(L, grads_dev, rank_stride, master, m, v, p16_shard, p16_full, hp);
    if (s != ZERO_OK || L->padded == 0) return s;
    if (!grads_host || !p16_host) return ZERO_ERR_INVALID;
    cudaStream_t st = (cudaStream_t)stream;
    const zero::DeviceState &d = L->dev;
    const AdamScalars c = step_scalars(L->n_ranks, *hp);
    const size_t nb = L->bucket_lo.size();
    uint16_t *p16 = L->stage == 3 ? p16_shard : p16_full;

    // the staging buffer may still be read by earlier work on `stream`
    cudaError_t e = cudaEventRecord(d.begin, st);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(d.copy_in, d.begin, 0);
    for (size_t b = 0; e == cudaSuccess && b < nb; ++b) {
        const int64_t lo = L->bucket_lo[b], bytes = 2 * (L->bucket_hi[b] - lo);
        for (int32_t r = 0; e == cudaSuccess && r < L->n_ranks; ++r) {
            const int64_t off = (int64_t)r * rank_stride + lo;
            e = cudaMemcpyAsync(grads_dev + off, grads_host + off, (size_t)bytes, cudaMemcpyHostToDevice,
                                d.copy_in);
        }
        if (e == cudaSuccess) e = cudaEventRecord(d.landed[b], d.copy_in);
    }
    for (size_t b = 0; e == cudaSuccess && b < nb; ++b) {
        e = cudaStreamWaitEvent(st, d.landed[b], 0);
        if (e == cudaSuccess)
            e = fused(L, bucket_tiles(L, (int64_t)b), grads_dev, rank_stride, master, m, v, p16, c, nonfinite, st);
        if (e == cudaSuccess && L->stage != 3) {
            e = cudaEventRecord(d.updated[b], st);
            if (e == cudaSuccess) e = cudaStreamWaitEvent(d.copy_out, d.updated[b], 0);
            const int64_t lo = L->bucket_lo[b], bytes = 2 * (L->bucket_hi[b] - lo);
            if (e == cudaSuccess)
                e = cudaMemcpyAsync(p16_host + lo, p16_full + lo, (size_t)bytes, cudaMemcpyDeviceToHost,
                                    d.copy_out);
        }
    }
    if (e == cudaSuccess && L->stage == 3) {
        e = zero::launch_copy_range(*L, 0, L->padded, p16_shard, p16_full, st);
        if (e == cudaSuccess)
            e = cudaMemcpyAsync(p16_host, p16_full, (size_t)(2 * L->padded), cudaMemcpyDeviceToHost, st);
    } else if (e == cudaSuccess) {
        // `stream` completes only after the last parameter copy has landed
        e = cudaEventRecord(d.done, d.copy_out);
        if (e == cudaSuccess) e = cudaStreamWaitEvent(st, d.done, 0);
    }
    return cuda_status(e);
}

extern "C" zero_status zero_get_error(const zero_layout *L, void *stream)
{
    ZERO_RANGE("zero_get_error");
    zero_status s = check_device(L);
    if (s != ZERO_OK) return s;
    cudaStream_t st = (cudaStream_t)stream;
    int32_t word = 0;
    cudaError_t e = cudaStreamSynchronize(st);
    if (e == cudaSuccess) e = cudaMemcpy(&word, L->dev.error, sizeof word, cudaMemcpyDeviceToHost);
    if (e == cudaSuccess && word != 0) e = cudaMemset(L->dev.error, 0, sizeof word);
    if (e != cudaSuccess) return ZERO_ERR_CUDA;
    return word == 0 ? ZERO_OK : (zero_status)word;
}

extern "C" zero_status zero_debug_set_wait(zero_layout *L, int64_t wait_limit_ns, int32_t skip_first_fill)
{
    ZERO_RANGE("zero_debug_set_wait");
    if (!L || wait_limit_ns <= 0 || skip_first_fill < 0 || skip_first_fill > 1) return ZERO_ERR_INVALID;
    if (L->dev.device < 0) return ZERO_ERR_STATE;
    L->dev.wait_limit_ns = (uint64_t)wait_limit_ns;
    L->dev.skip_first_fill = skip_first_fill;
    return ZERO_OK;
}
