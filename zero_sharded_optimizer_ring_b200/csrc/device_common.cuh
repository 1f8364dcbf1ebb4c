// Device helpers shared by the step kernels (included by kernels.cu and bulk_step.cu).
//
// Every floating-point step is one explicitly rounded IEEE operation (__fadd_rn,
// __fmul_rn, __fdiv_rn, __fsqrt_rn; fp16 adds with __hadd2 / __hadd), so the kernels
// compute the same bits whatever the compiler's contraction settings.
#pragma once

#include <cuda_fp16.h>
#include <stdint.h>

#include "internal.h"

namespace zero {

constexpr int kVec = 8;   // elements per 16-byte fp16 vector

__device__ __forceinline__ float h2f(uint32_t bits16)
{
    return __half2float(__ushort_as_half((unsigned short)(bits16 & 0xffffu)));
}

__device__ __forceinline__ uint32_t f2h(float f)
{
    return (uint32_t)__half_as_ushort(__float2half_rn(f));
}

__device__ __forceinline__ void unpack8(const uint4 u, float (&f)[8])
{
    f[0] = h2f(u.x); f[1] = h2f(u.x >> 16);
    f[2] = h2f(u.y); f[3] = h2f(u.y >> 16);
    f[4] = h2f(u.z); f[5] = h2f(u.z >> 16);
    f[6] = h2f(u.w); f[7] = h2f(u.w >> 16);
}

__device__ __forceinline__ void add8(float (&acc)[8], const uint4 u)
{
    float f[8];
    unpack8(u, f);
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] = __fadd_rn(acc[e], f[e]);
}

// fp16-wire fold: the travelling partial is fp16 and every hop adds the next rank's fp16
// value with one correctly rounded fp16 add (add.rn.f16x2: two lanes, each rounded to
// nearest even, subnormals kept).
__device__ __forceinline__ uint4 hadd8(const uint4 a, const uint4 b)
{
    uint4 r;
    const __half2 x0 = __hadd2(*reinterpret_cast<const __half2 *>(&a.x), *reinterpret_cast<const __half2 *>(&b.x));
    const __half2 x1 = __hadd2(*reinterpret_cast<const __half2 *>(&a.y), *reinterpret_cast<const __half2 *>(&b.y));
    const __half2 x2 = __hadd2(*reinterpret_cast<const __half2 *>(&a.z), *reinterpret_cast<const __half2 *>(&b.z));
    const __half2 x3 = __hadd2(*reinterpret_cast<const __half2 *>(&a.w), *reinterpret_cast<const __half2 *>(&b.w));
    r.x = *reinterpret_cast<const uint32_t *>(&x0);
    r.y = *reinterpret_cast<const uint32_t *>(&x1);
    r.z = *reinterpret_cast<const uint32_t *>(&x2);
    r.w = *reinterpret_cast<const uint32_t *>(&x3);
    return r;
}

__device__ __forceinline__ uint32_t hadd1(uint32_t a, uint32_t b)
{
    return (uint32_t)__half_as_ushort(__hadd(__ushort_as_half((unsigned short)a), __ushort_as_half((unsigned short)b)));
}

// The shard update, order of operations as documented in zero.h, in two parts: the
// moments (p becomes the decayed weight), then the step from the new moments.
__device__ __forceinline__ void adamw_moments(float s, const AdamScalars &c, float &p, float &m, float &v)
{
    const float g = __fmul_rn(s, c.inv_scale);
    p = __fmul_rn(p, c.decay);
    m = __fadd_rn(__fmul_rn(m, c.beta1), __fmul_rn(g, c.omb1));
    v = __fadd_rn(__fmul_rn(v, c.beta2), __fmul_rn(__fmul_rn(g, g), c.omb2));
}

__device__ __forceinline__ void adamw_apply(const AdamScalars &c, float &p, float m, float v)
{
    const float denom = __fadd_rn(__fdiv_rn(__fsqrt_rn(v), c.sqrt_bc2), c.eps);
    p = __fsub_rn(p, __fmul_rn(c.step_size, __fdiv_rn(m, denom)));
}

// The same step for moments that may be exactly zero.  Zero operands send the IEEE
// square-root and divide sequences off their fast path (a parameter with zero gradient
// and zero moments, e.g. an embedding row no batch has touched, then costs about twice
// as much), so they are skipped by two exact identities: sqrt(+-0) / c = +-0 for the
// step's c = sqrt(1 - beta2^t) > 0, and +-0 / denom = +-0 for denom > 0 (0 / 0 and NaN
// still divide, and give NaN as before).
__device__ __forceinline__ void adamw_apply_zeros(const AdamScalars &c, float &p, float m, float v)
{
    const float q = v == 0.0f ? v : __fdiv_rn(__fsqrt_rn(v), c.sqrt_bc2);
    const float denom = __fadd_rn(q, c.eps);
    const float ratio = (m == 0.0f && denom > 0.0f) ? m : __fdiv_rn(m, denom);
    p = __fsub_rn(p, __fmul_rn(c.step_size, ratio));
}

// One element (ragged edges).
__device__ __forceinline__ void adamw_elem(float s, const AdamScalars &c, float &p, float &m,
                                           float &v, uint32_t &h)
{
    adamw_moments(s, c, p, m, v);
    adamw_apply_zeros(c, p, m, v);
    h = f2h(p);
}

// Eight elements.  The branch is decided on the incoming second moments, before any
// arithmetic: a group where all are nonzero (dense training after its first step: every
// group) runs the plain straight-line update; a group holding a zero (cold start,
// untouched or frozen rows) takes the element-wise shortcuts.  Both give the same bits,
// so the choice only decides speed.
__device__ __forceinline__ void adamw8(const float *s, const AdamScalars &c, float *p, float *m, float *v,
                                       uint32_t *h)
{
    bool zero = false;
#pragma unroll
    for (int e = 0; e < 8; ++e) zero |= v[e] == 0.0f;
    if (!zero) {
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            adamw_moments(s[e], c, p[e], m[e], v[e]);
            adamw_apply(c, p[e], m[e], v[e]);
            h[e] = f2h(p[e]);
        }
    } else {
#pragma unroll
        for (int e = 0; e < 8; ++e) adamw_elem(s[e], c, p[e], m[e], v[e], h[e]);
    }
}

__device__ __forceinline__ int is_nonfinite(float x) { return !isfinite(x); }

// Adds this thread's non-finite count into counts[bucket]: one atomic per warp.
__device__ __forceinline__ void flush_nonfinite(int32_t *counts, int32_t bucket, int mine)
{
    if (counts == nullptr) return;
    const unsigned full = 0xffffffffu;
    if (__any_sync(full, mine != 0)) {
        const int total = __reduce_add_sync(full, mine);
        if ((threadIdx.x & 31) == 0) atomicAdd(counts + bucket, total);
    }
}

struct TileRange {
    int64_t a, b;      // [a, b): the tile's elements
    int32_t shard, bucket;
};

// Locate tile t: advance the segment cursor s (tiles are visited in increasing order
// by each CTA, so the cursor only moves forward), then clip the tile's cell of the
// global kTileElems grid to the segment.  A debug build never lets the cursor pass the
// closing row.
__device__ __forceinline__ TileRange locate_tile(const TileWork &w, int64_t &s, int64_t t)
{
    const Seg *__restrict__ segs = w.segs;
#ifdef ZERO_DEBUG
    while (s < w.bounds.n_seg && __ldg(&segs[s + 1].tile_begin) <= t) ++s;
#else
    while (__ldg(&segs[s + 1].tile_begin) <= t) ++s;
#endif
    const int64_t lo = __ldg(&segs[s].lo), hi = __ldg(&segs[s].hi);
    const int64_t cell = lo / kTileElems + (t - __ldg(&segs[s].tile_begin));
    TileRange r;
    r.a = cell * kTileElems > lo ? cell * kTileElems : lo;
    r.b = (cell + 1) * kTileElems < hi ? (cell + 1) * kTileElems : hi;
    r.shard = __ldg(&segs[s].shard);
    r.bucket = __ldg(&segs[s].bucket);
    return r;
}

// Debug builds: does the located tile lie inside the table, its shard, the padded buffer
// and the launch's state buffers?  If not, record ZERO_ERR_BOUNDS (first error wins) and
// tell the caller to skip it.  Release builds: always true, compiled away.
__device__ __forceinline__ bool tile_in_bounds(const TileWork &w, int64_t s, const TileRange &r)
{
#ifdef ZERO_DEBUG
    const TileBounds &B = w.bounds;
    const bool ok = s >= w.seg_first && s < B.n_seg && r.a >= 0 && r.a < r.b && r.b <= B.padded &&
                    r.b - r.a <= kTileElems && r.shard >= 0 && r.shard < B.n_ranks && r.bucket >= 0 &&
                    r.bucket < B.n_buckets && r.a >= (int64_t)r.shard * B.shard &&
                    r.b <= ((int64_t)r.shard + 1) * B.shard && r.a >= B.state_lo && r.b <= B.state_hi;
    if (!ok && B.error) atomicCAS(B.error, 0, (int32_t)ZERO_ERR_BOUNDS);
    return ok;
#else
    (void)w;
    (void)s;
    (void)r;
    return true;
#endif
}

// Rank at position j of the ring fold that starts at rank k.
__device__ __forceinline__ int ring_rank(int k, int j, int n)
{
    const int r = k + j;
    return r >= n ? r - n : r;
}

}  // namespace zero
