// Host-side partitioner: flat buffer, shards, buckets, segments, gather units, counters.
//
// Flat buffer and N-way shards: rkmt.cn/news/44736, "Deepspeed ZeRO-1" (each of the
// GPUs is responsible for one third of the gradients and optimizer state).
// Buckets: rkmt.cn/news/44736 "DDP" / "Deepspeed ZeRO-2" and en.pswp.cn/web/84187
// "DDP" (gradients are grouped into buckets that are reduced as soon as they are
// complete, which happens back to front during the backward pass), so bucket 0 is the
// tail of the flat buffer.
// Counters: rkmt.cn/news/44736 "Deepspeed ZeRO" (2+2+12 bytes per parameter for DDP)
// and the communication analyses of "DDP", "ZeRO-1/-2", "ZeRO-3".
#include <stdlib.h>

#include <new>

#include "internal.h"

namespace {

int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

constexpr int64_t kMaxElems = int64_t(1) << 52;   // flat sizes stay far from int64 overflow

}  // namespace

extern "C" zero_status zero_layout_create(const zero_layout_desc *d, zero_layout **out)
{
    if (!d || !out) return ZERO_ERR_INVALID;
    *out = nullptr;
    if (d->n_ranks < 1 || d->n_ranks > 4096 || d->stage < 0 || d->stage > 3 ||
        d->wire_fp16 < 0 || d->wire_fp16 > 1 ||
        d->n_tensors < 0 || (d->n_tensors > 0 && !d->tensor_numel) || d->pad_align < 1 ||
        d->pad_align > (int64_t(1) << 30) || d->n_units < 0 ||
        (d->n_units > 0 && !d->unit_first_tensor))
        return ZERO_ERR_INVALID;

    zero_layout *L = new (std::nothrow) zero_layout();
    if (!L) return ZERO_ERR_OOM;
    try {
        L->n_ranks = d->n_ranks;
        L->stage = d->stage;
        L->wire16 = d->wire_fp16;
        L->pad_align = d->pad_align;
        L->bucket_elems = d->bucket_elems;

        int64_t acc = 0;
        L->tensor_off.resize((size_t)d->n_tensors);
        for (int64_t t = 0; t < d->n_tensors; ++t) {
            const int64_t n = d->tensor_numel[t];
            if (n < 0 || n > kMaxElems || acc > kMaxElems - n) { delete L; return ZERO_ERR_INVALID; }
            L->tensor_off[(size_t)t] = acc;
            acc += n;
        }
        L->psi = acc;
        const int64_t N = d->n_ranks;
        L->shard = acc == 0 ? 0 : ceil_div(ceil_div(acc, N), d->pad_align) * d->pad_align;
        if (L->shard > kMaxElems / N) { delete L; return ZERO_ERR_INVALID; }
        L->padded = N * L->shard;
        const int64_t P = L->padded, S = L->shard;

        // buckets, cut from the tail
        if (P > 0) {
            const int64_t B = d->bucket_elems <= 0 ? P : d->bucket_elems;
            for (int64_t hi = P; hi > 0;) {
                const int64_t lo = hi > B ? hi - B : 0;
                L->bucket_lo.push_back(lo);
                L->bucket_hi.push_back(hi);
                hi = lo;
            }
        }
        if (L->bucket_lo.size() > (size_t)INT32_MAX) { delete L; return ZERO_ERR_INVALID; }

        // segments = bucket x shard, bucket order then shard order; tiles per segment
        int64_t tiles = 0;
        for (size_t b = 0; b < L->bucket_lo.size(); ++b) {
            L->bucket_seg_begin.push_back((int64_t)L->segs.size());
            const int64_t lo = L->bucket_lo[b], hi = L->bucket_hi[b];
            for (int64_t k = lo / S; k < N && k * S < hi; ++k) {
                const int64_t a = lo > k * S ? lo : k * S;
                const int64_t z = hi < (k + 1) * S ? hi : (k + 1) * S;
                if (z <= a) continue;
                zero::Seg s;
                s.lo = a;
                s.hi = z;
                s.shard = (int32_t)k;
                s.bucket = (int32_t)b;
                s.tile_begin = tiles;
                tiles += ceil_div(z, zero::kTileElems) - a / zero::kTileElems;
                L->segs.push_back(s);
            }
        }
        L->bucket_seg_begin.push_back((int64_t)L->segs.size());
        L->n_tiles = tiles;
        L->closing.lo = L->closing.hi = P;
        L->closing.tile_begin = -1;
        L->closing.shard = L->closing.bucket = -1;

        // the same segments shard-major (one shard's segments contiguous), renumbered
        for (int64_t k = 0; k < N; ++k) {
            L->shard_seg_begin.push_back((int64_t)L->segs_by_shard.size());
            for (const zero::Seg &sg : L->segs)
                if (sg.shard == k) L->segs_by_shard.push_back(sg);
        }
        L->shard_seg_begin.push_back((int64_t)L->segs_by_shard.size());
        int64_t t2 = 0;
        for (zero::Seg &sg : L->segs_by_shard) {
            sg.tile_begin = t2;
            t2 += ceil_div(sg.hi, zero::kTileElems) - sg.lo / zero::kTileElems;
        }

        // gather units: tensor ranges; the last unit also takes the tail padding
        if (P > 0) {
            if (d->n_units == 0) {
                L->unit_lo.push_back(0);
                L->unit_hi.push_back(P);
            } else {
                const int64_t *u = d->unit_first_tensor;
                if (u[0] != 0) { delete L; return ZERO_ERR_INVALID; }
                for (int64_t j = 0; j < d->n_units; ++j) {
                    if (u[j] < 0 || u[j] >= d->n_tensors || (j > 0 && u[j] <= u[j - 1])) {
                        delete L;
                        return ZERO_ERR_INVALID;
                    }
                    L->unit_lo.push_back(L->tensor_off[(size_t)u[j]]);
                }
                for (int64_t j = 0; j + 1 < d->n_units; ++j) L->unit_hi.push_back(L->unit_lo[(size_t)j + 1]);
                L->unit_hi.push_back(P);
            }
        }
    } catch (...) {
        delete L;
        return ZERO_ERR_OOM;
    }
    *out = L;
    return ZERO_OK;
}

extern "C" zero_status zero_layout_get_info(const zero_layout *L, zero_layout_info *info)
{
    if (!L || !info) return ZERO_ERR_INVALID;
    info->psi = L->psi;
    info->shard = L->shard;
    info->padded = L->padded;
    info->n_buckets = (int64_t)L->bucket_lo.size();
    info->n_segments = (int64_t)L->segs.size();
    info->n_units = (int64_t)L->unit_lo.size();
    info->tile_elems = zero::kTileElems;
    info->n_tiles = L->n_tiles;
    return ZERO_OK;
}

extern "C" zero_status zero_layout_get_tables(const zero_layout *L, int64_t *tensor_off,
                                              int64_t *bucket_lohi, int64_t *segments,
                                              int64_t *unit_lohi)
{
    if (!L) return ZERO_ERR_INVALID;
    if (tensor_off)
        for (size_t t = 0; t < L->tensor_off.size(); ++t) tensor_off[t] = L->tensor_off[t];
    if (bucket_lohi)
        for (size_t b = 0; b < L->bucket_lo.size(); ++b) {
            bucket_lohi[2 * b] = L->bucket_lo[b];
            bucket_lohi[2 * b + 1] = L->bucket_hi[b];
        }
    if (segments)
        for (size_t s = 0; s < L->segs.size(); ++s) {
            segments[4 * s + 0] = L->segs[s].bucket;
            segments[4 * s + 1] = L->segs[s].shard;
            segments[4 * s + 2] = L->segs[s].lo;
            segments[4 * s + 3] = L->segs[s].hi;
        }
    if (unit_lohi)
        for (size_t u = 0; u < L->unit_lo.size(); ++u) {
            unit_lohi[2 * u] = L->unit_lo[u];
            unit_lohi[2 * u + 1] = L->unit_hi[u];
        }
    return ZERO_OK;
}

extern "C" zero_status zero_layout_counters(const zero_layout *L, zero_counters *c)
{
    if (!L || !c) return ZERO_ERR_INVALID;
    const int64_t psi = L->psi, S = L->shard, N = L->n_ranks;
    // what each stage shards (P1 "Deepspeed ZeRO"): 0 nothing, 1 optimizer state,
    // 2 + gradients, 3 + parameters
    c->mem_p16 = L->stage >= 3 ? 2 * S : 2 * psi;
    c->mem_g16 = L->stage >= 2 ? 2 * S : 2 * psi;
    c->mem_os = L->stage >= 1 ? 12 * S : 12 * psi;
    c->mem_total = c->mem_p16 + c->mem_g16 + c->mem_os;
    // ring phases of N-1 hops moving one S-element chunk each: scatter-reduce and
    // all-gather; ZeRO-3 gathers the parameters again for the backward pass
    const int64_t phases = L->stage == 3 ? 3 : 2;
    c->sent_elems = phases * (N - 1) * S;
    c->recv_elems = c->sent_elems;
    return ZERO_OK;
}

extern "C" zero_status zero_set_impl(zero_layout *L, int32_t impl)
{
    if (!L || impl < 0 || impl > 2) return ZERO_ERR_INVALID;
    L->impl = impl;
    return ZERO_OK;
}

extern "C" zero_status zero_set_max_ctas(zero_layout *L, int32_t max_ctas)
{
    if (!L || max_ctas < 0) return ZERO_ERR_INVALID;
    L->max_ctas = max_ctas;
    return ZERO_OK;
}

extern "C" zero_status zero_set_gather_ctas(zero_layout *L, int32_t max_ctas)
{
    if (!L || max_ctas < 0) return ZERO_ERR_INVALID;
    L->gather_ctas = max_ctas;
    return ZERO_OK;
}
