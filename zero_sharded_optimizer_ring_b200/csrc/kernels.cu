// Device kernels of the sharded optimizer step (sm_100a).
//
// Everything here is HBM-bound streaming work: no dense contraction, so no tensor
// cores.  The kernels move 16-byte vectors (8 fp16 or 4 fp32 values) per thread per
// access, walk the segment table tile by tile with a persistent grid sized to the SM
// count, and do every floating-point step as one explicitly rounded IEEE operation
// (__fadd_rn / __fmul_rn / __fdiv_rn / __fsqrt_rn, no contraction into FMA).
//
// Ring order (en.pswp.cn/web/84187, "DDP" walk-through; rkmt.cn/news/44736 "DDP"):
// chunk k of a bucket starts at rank k and each later rank of the ring adds its own
// fp32-converted gradient, so the sum for an element of shard k is folded in the fixed
// order k, k+1, ..., k+N-1 (mod N).  All N ranks' slices are loaded before the fold;
// only the order of the additions matters for the result.
//
// Update (rkmt.cn/news/44736, "Deepspeed ZeRO-1", update step): fp16 -> fp32 without
// storing it, scale, fp32 first and second moments, fp32 master weights, fp16 params.
#include <cuda_fp16.h>
#include <stdint.h>

#include "bulk_ptx.cuh"
#include "device_common.cuh"
#include "gather_ranks.h"

namespace zero {
namespace {

constexpr int kThreads = 256;

// Scalar ring fold of one element (ragged tile edges, runtime-N path).
template <bool kWire>
__device__ __forceinline__ float fold_scalar(const uint16_t *__restrict__ grads, int64_t stride,
                                             int k, int n, int64_t i)
{
    if constexpr (kWire) {
        uint32_t h = __ldcs(grads + (int64_t)k * stride + i);
        for (int j = 1; j < n; ++j) h = hadd1(h, __ldcs(grads + (int64_t)ring_rank(k, j, n) * stride + i));
        return h2f(h);
    } else {
        float acc = h2f(__ldcs(grads + (int64_t)k * stride + i));
        for (int j = 1; j < n; ++j)
            acc = __fadd_rn(acc, h2f(__ldcs(grads + (int64_t)ring_rank(k, j, n) * stride + i)));
        return acc;
    }
}

// ---------------------------------------------------------------------------------
// Tile kernel: ring reduce-scatter of every tile of the launch, then either the
// fused shard update (kFused) or a store of the fp32 sums.
//   NT = compile-time rank count (0 = runtime n_ranks), U = vectors per thread whose
//   loads are in flight together, kWire = fp16 wire (partials rounded to fp16 per hop),
//   kOut = the fused update reads the state from `in` and writes it to master / mom1 /
//   mom2 (two buffer sets that do not overlap); otherwise it updates them in place.
//   kMinBlocks = the launch bound's minimum of resident CTAs per SM, i.e. a register
//   budget of 65536 / (kThreads * kMinBlocks) per thread (0: no bound, the compiler's
//   own choice); the grid then takes as many CTAs per SM as the registers actually used
//   allow.
struct StateIn {
    const float *master, *mom1, *mom2;
};

template <int NT, int U, bool kFused, bool kWire, bool kOut = false, int kMinBlocks = 0>
__global__ void __launch_bounds__(kThreads, kMinBlocks)
tile_kernel(TileWork w, int n_ranks, const uint16_t *__restrict__ grads, int64_t stride,
            float *__restrict__ reduced, float *__restrict__ master, float *__restrict__ mom1,
            float *__restrict__ mom2, uint16_t *__restrict__ p16, AdamScalars c_arg,
            int32_t *__restrict__ nonfinite, StateIn in, const AdamScalars *__restrict__ c_dev)
{
    const AdamScalars c = c_dev ? *c_dev : c_arg;     // run-time scalars when given (graph replays)
    const float *__restrict__ master_in = kOut ? in.master : master;
    const float *__restrict__ mom1_in = kOut ? in.mom1 : mom1;
    const float *__restrict__ mom2_in = kOut ? in.mom2 : mom2;
    const int n = NT > 0 ? NT : n_ranks;
    int64_t s = w.seg_first;
    const int64_t t_end = w.tile_first + w.n_tiles;
    for (int64_t t = w.tile_first + blockIdx.x; t < t_end; t += gridDim.x) {
        const TileRange tr = locate_tile(w, s, t);
        if (!tile_in_bounds(w, s, tr)) continue;
        const int k = tr.shard;
        int bad = 0;
        const int64_t va = (tr.a + kVec - 1) / kVec * kVec;
        const int64_t vb = tr.b / kVec * kVec;

        // aligned body: 8 elements per vector, U vectors per thread in flight
        for (int64_t q0 = va + (int64_t)threadIdx.x * kVec; q0 < vb; q0 += (int64_t)U * kThreads * kVec) {
            float acc[U][8];
            if constexpr (NT > 0) {
                uint4 g[U][NT];
#pragma unroll
                for (int u = 0; u < U; ++u) {
                    const int64_t q = q0 + (int64_t)u * kThreads * kVec;
                    if (q < vb) {
#pragma unroll
                        for (int j = 0; j < NT; ++j)
                            g[u][j] = __ldcs(reinterpret_cast<const uint4 *>(
                                grads + (int64_t)ring_rank(k, j, NT) * stride + q));
                    }
                }
#pragma unroll
                for (int u = 0; u < U; ++u) {
                    if constexpr (kWire) {
                        uint4 h = g[u][0];
#pragma unroll
                        for (int j = 1; j < NT; ++j) h = hadd8(h, g[u][j]);
                        unpack8(h, acc[u]);
                    } else {
                        unpack8(g[u][0], acc[u]);
#pragma unroll
                        for (int j = 1; j < NT; ++j) add8(acc[u], g[u][j]);
                    }
                }
            } else {
#pragma unroll
                for (int u = 0; u < U; ++u) {
                    const int64_t q = q0 + (int64_t)u * kThreads * kVec;
                    if (q < vb) {
                        const uint4 first = __ldcs(reinterpret_cast<const uint4 *>(grads + (int64_t)k * stride + q));
                        if constexpr (kWire) {
                            uint4 h = first;
#pragma unroll 4
                            for (int j = 1; j < n; ++j)
                                h = hadd8(h, __ldcs(reinterpret_cast<const uint4 *>(
                                                 grads + (int64_t)ring_rank(k, j, n) * stride + q)));
                            unpack8(h, acc[u]);
                        } else {
                            unpack8(first, acc[u]);
#pragma unroll 4
                            for (int j = 1; j < n; ++j)
                                add8(acc[u], __ldcs(reinterpret_cast<const uint4 *>(
                                                 grads + (int64_t)ring_rank(k, j, n) * stride + q)));
                        }
                    }
                }
            }

#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int64_t q = q0 + (int64_t)u * kThreads * kVec;
                if (q >= vb) continue;
#pragma unroll
                for (int e = 0; e < 8; ++e) bad += is_nonfinite(acc[u][e]);
                if constexpr (kFused) {
                    float4 *pp = reinterpret_cast<float4 *>(master + q);
                    float4 *mp = reinterpret_cast<float4 *>(mom1 + q);
                    float4 *vp = reinterpret_cast<float4 *>(mom2 + q);
                    const float4 *pi = reinterpret_cast<const float4 *>(master_in + q);
                    const float4 *mi = reinterpret_cast<const float4 *>(mom1_in + q);
                    const float4 *vi = reinterpret_cast<const float4 *>(mom2_in + q);
                    float4 p4[2] = {__ldcs(pi), __ldcs(pi + 1)};
                    float4 m4[2] = {__ldcs(mi), __ldcs(mi + 1)};
                    float4 v4[2] = {__ldcs(vi), __ldcs(vi + 1)};
                    float *pf = reinterpret_cast<float *>(p4);
                    float *mf = reinterpret_cast<float *>(m4);
                    float *vf = reinterpret_cast<float *>(v4);
                    uint32_t h[8];
                    adamw8(acc[u], c, pf, mf, vf, h);
                    __stcs(pp, p4[0]); __stcs(pp + 1, p4[1]);
                    __stcs(mp, m4[0]); __stcs(mp + 1, m4[1]);
                    __stcs(vp, v4[0]); __stcs(vp + 1, v4[1]);
                    __stcs(reinterpret_cast<uint4 *>(p16 + q),
                           make_uint4(h[0] | (h[1] << 16), h[2] | (h[3] << 16),
                                      h[4] | (h[5] << 16), h[6] | (h[7] << 16)));
                } else {
                    float4 *rp = reinterpret_cast<float4 *>(reduced + q);
                    __stcs(rp, make_float4(acc[u][0], acc[u][1], acc[u][2], acc[u][3]));
                    __stcs(rp + 1, make_float4(acc[u][4], acc[u][5], acc[u][6], acc[u][7]));
                }
            }
        }

        // ragged edges of the tile (segment boundaries that are not 8-aligned)
        const int64_t head_end = va < tr.b ? va : tr.b;
        const int64_t tail_begin = vb > head_end ? vb : head_end;
        const int64_t n_head = head_end - tr.a, n_tail = tr.b - tail_begin;
        if (threadIdx.x < n_head + n_tail) {
            const int64_t i = threadIdx.x < n_head ? tr.a + threadIdx.x : tail_begin + (threadIdx.x - n_head);
            const float acc = fold_scalar<kWire>(grads, stride, k, n, i);
            bad += is_nonfinite(acc);
            if constexpr (kFused) {
                float p = master_in[i], m = mom1_in[i], v = mom2_in[i];
                uint32_t h;
                adamw_elem(acc, c, p, m, v, h);
                master[i] = p;
                mom1[i] = m;
                mom2[i] = v;
                p16[i] = (uint16_t)h;
            } else {
                reduced[i] = acc;
            }
        }
        flush_nonfinite(nonfinite, tr.bucket, bad);
    }
}

// ---------------------------------------------------------------------------------
// Range kernels over [lo, hi) with an aligned 16-byte body and scalar edges.

__global__ void __launch_bounds__(kThreads)
adamw_range_kernel(int64_t lo, int64_t hi, const float *__restrict__ reduced, float *__restrict__ master,
                   float *__restrict__ mom1, float *__restrict__ mom2, uint16_t *__restrict__ p16,
                   AdamScalars c)
{
    const int64_t va = (lo + kVec - 1) / kVec * kVec, vb = hi / kVec * kVec;
    const int64_t stride = (int64_t)gridDim.x * kThreads * kVec;
    for (int64_t q = va + ((int64_t)blockIdx.x * kThreads + threadIdx.x) * kVec; q < vb; q += stride) {
        const float4 *rp = reinterpret_cast<const float4 *>(reduced + q);
        float4 *pp = reinterpret_cast<float4 *>(master + q);
        float4 *mp = reinterpret_cast<float4 *>(mom1 + q);
        float4 *vp = reinterpret_cast<float4 *>(mom2 + q);
        float4 r4[2] = {__ldcs(rp), __ldcs(rp + 1)};
        float4 p4[2] = {__ldcs(pp), __ldcs(pp + 1)};
        float4 m4[2] = {__ldcs(mp), __ldcs(mp + 1)};
        float4 v4[2] = {__ldcs(vp), __ldcs(vp + 1)};
        const float *rf = reinterpret_cast<const float *>(r4);
        float *pf = reinterpret_cast<float *>(p4);
        float *mf = reinterpret_cast<float *>(m4);
        float *vf = reinterpret_cast<float *>(v4);
        uint32_t h[8];
        adamw8(rf, c, pf, mf, vf, h);
        __stcs(pp, p4[0]); __stcs(pp + 1, p4[1]);
        __stcs(mp, m4[0]); __stcs(mp + 1, m4[1]);
        __stcs(vp, v4[0]); __stcs(vp + 1, v4[1]);
        __stcs(reinterpret_cast<uint4 *>(p16 + q),
               make_uint4(h[0] | (h[1] << 16), h[2] | (h[3] << 16), h[4] | (h[5] << 16), h[6] | (h[7] << 16)));
    }
    if (blockIdx.x == 0) {
        const int64_t head_end = va < hi ? va : hi;
        const int64_t tail_begin = vb > head_end ? vb : head_end;
        const int64_t n_head = head_end - lo, n_tail = hi - tail_begin;
        if (threadIdx.x < n_head + n_tail) {
            const int64_t i = threadIdx.x < n_head ? lo + threadIdx.x : tail_begin + (threadIdx.x - n_head);
            float p = master[i], m = mom1[i], v = mom2[i];
            uint32_t h;
            adamw_elem(reduced[i], c, p, m, v, h);
            master[i] = p;
            mom1[i] = m;
            mom2[i] = v;
            p16[i] = (uint16_t)h;
        }
    }
}

// Copy [lo, hi): one block per 4 x 256 16-byte vectors, each thread holding its 4 loads in
// flight before storing.  A grid of short blocks keeps the blocks in flight on a compact
// window of the buffer (a persistent grid-stride loop lets the blocks drift apart over
// the buffer and costs ~15 % of copy bandwidth on B200: 5.9 vs 6.9 TB/s measured).
constexpr int kCopyUnroll = 4;

__global__ void __launch_bounds__(kThreads)
copy_range_kernel(int64_t lo, int64_t hi, const uint16_t *__restrict__ src, uint16_t *__restrict__ dst)
{
    const int64_t va = (lo + kVec - 1) / kVec * kVec, vb = hi / kVec * kVec;
    const int64_t base = va + (int64_t)blockIdx.x * kThreads * kVec * kCopyUnroll;
    uint4 x[kCopyUnroll];
#pragma unroll
    for (int u = 0; u < kCopyUnroll; ++u) {
        const int64_t q = base + ((int64_t)u * kThreads + threadIdx.x) * kVec;
        if (q < vb) x[u] = *reinterpret_cast<const uint4 *>(src + q);
    }
#pragma unroll
    for (int u = 0; u < kCopyUnroll; ++u) {
        const int64_t q = base + ((int64_t)u * kThreads + threadIdx.x) * kVec;
        if (q < vb) *reinterpret_cast<uint4 *>(dst + q) = x[u];
    }
    if (blockIdx.x == 0) {
        const int64_t head_end = va < hi ? va : hi;
        const int64_t tail_begin = vb > head_end ? vb : head_end;
        const int64_t n_head = head_end - lo, n_tail = hi - tail_begin;
        if (threadIdx.x < n_head + n_tail) {
            const int64_t i = threadIdx.x < n_head ? lo + threadIdx.x : tail_begin + (threadIdx.x - n_head);
            dst[i] = src[i];
        }
    }
}

// Copy on a capped grid of persistent CTAs, through shared memory with bulk copies:
// d[j] = s[j] for j < n (s and d 16-byte aligned), plus hn < 8 head elements hd[j] = hs[j].
// One thread per CTA drives a ring of kBulkCopyStages stages of kBulkCopyChunk elements:
// cp.async.bulk loads (global -> shared, completion on the stage's mbarrier) run
// kBulkCopyStages - 1 chunks ahead of cp.async.bulk stores (shared -> global); a stage is
// reloaded only once its store has read it.  With ~144 KB of loads in flight per SM, a
// few SMs draw a large share of HBM bandwidth while the rest of the GPU computes (the
// gathers of a ZeRO-3 pass beside the layer GEMMs).  The vector body's last < 8 elements
// and the head go through other lanes of CTA 0.  Every wait is bounded: on expiry the
// kernel records ZERO_ERR_TIMEOUT, waits (bounded) for the loads it issued, and returns.
constexpr int kBulkCopyStages = 4;
constexpr int64_t kBulkCopyChunk = 24576;                                   // 48 KB
constexpr size_t kBulkCopySmem = 128 + (size_t)kBulkCopyStages * kBulkCopyChunk * 2;

__global__ void __launch_bounds__(32, 1)
copy_bulk_kernel(const uint16_t *__restrict__ s, uint16_t *__restrict__ d, int64_t n,
                 const uint16_t *__restrict__ hs, uint16_t *__restrict__ hd, int hn, int32_t *error,
                 uint64_t limit_ns)
{
    extern __shared__ __align__(128) unsigned char smem[];
    uint64_t *full = reinterpret_cast<uint64_t *>(smem);
    unsigned char *ring = smem + 128;
    const int64_t nv = n / kVec * kVec;                   // the bulk-copied body
    if (blockIdx.x == 0 && threadIdx.x >= 1) {            // head and tail, element by element
        const int l = threadIdx.x - 1;
        if (l < hn) hd[l] = hs[l];
        if (l < n - nv) d[nv + l] = s[nv + l];
    }
    if (threadIdx.x != 0) return;
    for (int i = 0; i < kBulkCopyStages; ++i) mbar_init(smem_addr(&full[i]), 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");

    const int64_t n_chunks = (nv + kBulkCopyChunk - 1) / kBulkCopyChunk;
    const int64_t K = (int64_t)blockIdx.x < n_chunks ? (n_chunks - 1 - blockIdx.x) / gridDim.x + 1 : 0;
    int64_t issued = 0;
    auto chunk_of = [&](int64_t k) { return (int64_t)blockIdx.x + k * (int64_t)gridDim.x; };
    auto bytes_of = [&](int64_t c) {
        const int64_t e = nv - c * kBulkCopyChunk;
        return (uint32_t)((e < kBulkCopyChunk ? e : kBulkCopyChunk) * 2);
    };
    auto issue = [&](int64_t k) {
        const int st = (int)(k % kBulkCopyStages);
        const int64_t c = chunk_of(k);
        const uint32_t bar = smem_addr(&full[st]);
        mbar_arrive_expect_tx(bar, bytes_of(c));
        bulk_load(smem_addr(ring + (size_t)st * kBulkCopyChunk * 2), s + c * kBulkCopyChunk, bytes_of(c), bar);
        issued = k + 1;
    };
    for (int64_t k = 0; k < K && k < kBulkCopyStages - 1; ++k) issue(k);
    int64_t k = 0;
    for (; k < K; ++k) {
        const int64_t j = k + kBulkCopyStages - 1;       // the chunk that refills stage (k - 1) % S
        if (j < K) {
            if (k >= 1) bulk_wait_read_all();            // the store of chunk k - 1 has read it
            issue(j);
        }
        const int st = (int)(k % kBulkCopyStages);
        if (!mbar_wait_bounded(smem_addr(&full[st]), (uint32_t)((k / kBulkCopyStages) & 1), limit_ns)) {
            if (error) atomicExch(error, (int32_t)ZERO_ERR_TIMEOUT);
            break;
        }
        bulk_store(d + chunk_of(k) * kBulkCopyChunk, smem_addr(ring + (size_t)st * kBulkCopyChunk * 2),
                   bytes_of(chunk_of(k)));
        bulk_commit_group();
    }
    for (int64_t i = k + 1; i < issued; ++i)             // after a timeout: loads still in flight
        mbar_wait_bounded(smem_addr(&full[i % kBulkCopyStages]), (uint32_t)((i / kBulkCopyStages) & 1), limit_ns);
    bulk_wait_all();                                      // every store complete before the CTA leaves
}

cudaError_t launch_copy_capped(const uint16_t *s, uint16_t *d, int64_t n, const uint16_t *hs, uint16_t *hd, int hn,
                               int32_t max_ctas, int32_t *error, uint64_t limit_ns, cudaStream_t st)
{
    if (n <= 0 && hn <= 0) return cudaSuccess;
    const int64_t n_chunks = (n / kVec * kVec + kBulkCopyChunk - 1) / kBulkCopyChunk;
    int64_t grid = n_chunks < max_ctas ? n_chunks : max_ctas;
    if (grid < 1) grid = 1;
    cudaError_t e = cudaFuncSetAttribute(copy_bulk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)kBulkCopySmem);
    if (e != cudaSuccess) return e;
    copy_bulk_kernel<<<(unsigned)grid, 32, kBulkCopySmem, st>>>(s, d, n > 0 ? n : 0, hs, hd, hn, error, limit_ns);
    return cudaGetLastError();
}

// Gather of one unit into a buffer of its own: dst[j] = src[lo + j], j < n.  With lo a
// multiple of 8 both sides are 16-byte aligned and each thread moves 4 vectors; otherwise
// each thread moves 8 scalars (still coalesced).  A grid of short blocks, as for the copy.
__global__ void __launch_bounds__(kThreads)
gather_unit_kernel(const uint16_t *__restrict__ src, int64_t lo, int64_t n, uint16_t *__restrict__ dst)
{
    if ((lo & 7) == 0) {
        const uint16_t *s = src + lo;
        const int64_t nv = n / kVec;
        const int64_t base = (int64_t)blockIdx.x * kThreads * kCopyUnroll;
        uint4 x[kCopyUnroll];
#pragma unroll
        for (int u = 0; u < kCopyUnroll; ++u) {
            const int64_t q = base + (int64_t)u * kThreads + threadIdx.x;
            if (q < nv) x[u] = *reinterpret_cast<const uint4 *>(s + q * kVec);
        }
#pragma unroll
        for (int u = 0; u < kCopyUnroll; ++u) {
            const int64_t q = base + (int64_t)u * kThreads + threadIdx.x;
            if (q < nv) *reinterpret_cast<uint4 *>(dst + q * kVec) = x[u];
        }
        if (blockIdx.x == 0 && threadIdx.x < n - nv * kVec) dst[nv * kVec + threadIdx.x] = s[nv * kVec + threadIdx.x];
    } else {
        const int64_t base = (int64_t)blockIdx.x * kThreads * kCopyUnroll * kVec;
        for (int u = 0; u < kCopyUnroll * kVec; ++u) {
            const int64_t j = base + (int64_t)u * kThreads + threadIdx.x;
            if (j < n) dst[j] = src[lo + j];
        }
    }
}

// Gather of one unit from the ranks' shard buffers: dst[j] = shard k's element lo + j - kS,
// k = (lo + j) / S, where rank k's buffer holds flat elements [kS, (k+1)S) (on this GPU or a
// peer's).  With lo and S multiples of 8 no 16-byte vector straddles two shards, so each
// thread moves 4 vectors per block of work, every source and destination 16-byte aligned;
// otherwise each thread moves 8 scalars.  Blocks of work are dealt to the CTAs by a grid
// stride: a grid of one CTA per block of work (short blocks, as for the copy), or a few
// persistent CTAs (zero_set_gather_ctas) that leave the other SMs to concurrent work.
__global__ void __launch_bounds__(kThreads)
gather_ranks_kernel(const __grid_constant__ ShardPtrs src, int64_t S, int64_t lo, int64_t n,
                    uint16_t *__restrict__ dst)
{
    if ((lo & 7) == 0 && (S & 7) == 0) {
        const int64_t nv = n / kVec;
        const int64_t per = (int64_t)kThreads * kCopyUnroll;              // vectors per block of work
        for (int64_t blk = blockIdx.x; blk * per < nv; blk += gridDim.x) {
            const int64_t base = blk * per;
            uint4 x[kCopyUnroll];
#pragma unroll
            for (int u = 0; u < kCopyUnroll; ++u) {
                const int64_t q = base + (int64_t)u * kThreads + threadIdx.x;
                if (q < nv) {
                    const int64_t i = lo + q * kVec, k = i / S;
                    x[u] = *reinterpret_cast<const uint4 *>(src.rank[k] + (i - k * S));
                }
            }
#pragma unroll
            for (int u = 0; u < kCopyUnroll; ++u) {
                const int64_t q = base + (int64_t)u * kThreads + threadIdx.x;
                if (q < nv) *reinterpret_cast<uint4 *>(dst + q * kVec) = x[u];
            }
        }
        if (blockIdx.x == 0 && threadIdx.x < n - nv * kVec) {
            const int64_t j = nv * kVec + threadIdx.x, i = lo + j, k = i / S;
            dst[j] = src.rank[k][i - k * S];
        }
    } else {
        const int64_t per = (int64_t)kThreads * kCopyUnroll * kVec;      // elements per block of work
        for (int64_t blk = blockIdx.x; blk * per < n; blk += gridDim.x) {
            const int64_t base = blk * per;
            for (int u = 0; u < kCopyUnroll * kVec; ++u) {
                const int64_t j = base + (int64_t)u * kThreads + threadIdx.x;
                if (j < n) {
                    const int64_t i = lo + j, k = i / S;
                    dst[j] = src.rank[k][i - k * S];
                }
            }
        }
    }
}

// ---------------------------------------------------------------------------------
// Tile index: one warp scans the segments' tile counts (exclusive prefix sum with
// __shfl_up_sync, 32 segments per pass, carried across passes).  Row n_seg receives
// the total, closing the table.
__global__ void tile_index_kernel(Seg *segs, int64_t n_seg)
{
    const unsigned full = 0xffffffffu;
    const int lane = threadIdx.x;
    int64_t carry = 0;
    for (int64_t base = 0; base < n_seg; base += 32) {
        const int64_t i = base + lane;
        int64_t cnt = 0;
        if (i < n_seg) {
            const int64_t lo = segs[i].lo, hi = segs[i].hi;
            cnt = (hi + kTileElems - 1) / kTileElems - lo / kTileElems;
        }
        int64_t x = cnt;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int64_t y = __shfl_up_sync(full, x, off);
            if (lane >= off) x += y;
        }
        if (i < n_seg) segs[i].tile_begin = carry + x - cnt;
        carry += __shfl_sync(full, x, 31);
    }
    if (lane == 0) segs[n_seg].tile_begin = carry;
}

// The SM count a layout recorded on upload; a layout that was never uploaded (the
// allocation-free step) asks the current device.
int sm_count(int recorded)
{
    if (recorded > 0) return recorded;
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) == cudaSuccess &&
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess && n > 0)
        return n;
    return 148;
}

template <class K>
int grid_for(K kernel, int64_t work_items, int num_sms, int max_ctas = 0)
{
    int per_sm = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, kThreads, 0) != cudaSuccess ||
        per_sm < 1)
        per_sm = 1;
    int64_t g = (int64_t)per_sm * sm_count(num_sms);
    if (max_ctas > 0 && g > max_ctas) g = max_ctas;
    if (g > work_items) g = work_items;
    return (int)(g < 1 ? 1 : g);
}

template <int NT, int U, bool kFused, int kMinBlocks = 0>
cudaError_t launch_tiles(const zero_layout &L, const TileWork &w, const uint16_t *grads, int64_t stride,
                         float *reduced, float *master, float *m, float *v, uint16_t *p16,
                         const AdamScalars &c, int32_t *nonfinite, cudaStream_t st, const AdamScalars *c_dev)
{
    auto kern = L.wire16 ? tile_kernel<NT, U, kFused, true, false, kMinBlocks>
                         : tile_kernel<NT, U, kFused, false, false, kMinBlocks>;
    const int grid = grid_for(kern, w.n_tiles, L.dev.num_sms, w.max_ctas > 0 ? w.max_ctas : L.max_ctas);
    kern<<<grid, kThreads, 0, st>>>(w, L.n_ranks, grads, stride, reduced, master, m, v, p16, c, nonfinite,
                                    StateIn{nullptr, nullptr, nullptr}, c_dev);
    return cudaGetLastError();
}

template <bool kFused>
cudaError_t dispatch_tiles(const zero_layout &L, const TileWork &w, const uint16_t *grads, int64_t stride,
                           float *reduced, float *master, float *m, float *v, uint16_t *p16,
                           const AdamScalars &c, int32_t *nonfinite, cudaStream_t st,
                           const AdamScalars *c_dev = nullptr)
{
    if (w.n_tiles <= 0) return cudaSuccess;
    // Shapes (vectors in flight per thread, the launch bound's minimum CTAs per SM), from
    // sweeps on flat lists of 2^28 parameters, one B200.  Fused: for 1-4 ranks one vector
    // with the two-CTA register budget (at 4 ranks 112 registers: two CTAs per SM) beats
    // two vectors per thread by 3-8 %; at 8 and 16 ranks one vector with no bound is as
    // fast or faster.  Reduce-only: one vector with the two-CTA budget (at 4 ranks 62
    // registers instead of 40: four CTAs per SM instead of six) is the fastest or level at
    // every rank count up to 16, 14-17 % ahead of no bound at 8 and 16 ranks.
#define ZERO_CASE(NV, UV, BV) \
    case NV: \
        if constexpr (kFused) \
            return launch_tiles<NV, UV, true, BV>(L, w, grads, stride, reduced, master, m, v, p16, c, nonfinite, st, c_dev); \
        else \
            return launch_tiles<NV, 1, false, 2>(L, w, grads, stride, reduced, master, m, v, p16, c, nonfinite, st, c_dev);
    switch (L.n_ranks) {
        ZERO_CASE(1, 1, 2)
        ZERO_CASE(2, 1, 2)
        ZERO_CASE(3, 1, 2)
        ZERO_CASE(4, 1, 2)
        ZERO_CASE(5, 1, 0)
        ZERO_CASE(6, 1, 0)
        ZERO_CASE(7, 1, 0)
        ZERO_CASE(8, 1, 0)
        ZERO_CASE(16, 1, 0)
        default:
            return launch_tiles<0, 1, kFused>(L, w, grads, stride, reduced, master, m, v, p16, c, nonfinite, st,
                                              c_dev);
    }
#undef ZERO_CASE
}

}  // namespace

TileBounds tile_bounds(const zero_layout &L, int64_t state_lo, int64_t state_hi)
{
    TileBounds b;
    b.n_seg = (int64_t)L.segs.size();
    b.padded = L.padded;
    b.shard = L.shard;
    b.state_lo = state_lo;
    b.state_hi = state_hi;
    b.n_ranks = L.n_ranks;
    b.n_buckets = (int32_t)L.bucket_lo.size();
    b.error = L.dev.error;
    return b;
}

cudaError_t launch_gather_unit(const uint16_t *src, int64_t lo, int64_t n, uint16_t *dst, int32_t max_ctas,
                               int32_t *error, uint64_t limit_ns, cudaStream_t s)
{
    if (n <= 0) return cudaSuccess;
    if (max_ctas > 0 && (lo & 7) == 0)
        return launch_copy_capped(src + lo, dst, n, nullptr, nullptr, 0, max_ctas, error, limit_ns, s);
    const int64_t per_block = (int64_t)kThreads * kCopyUnroll * kVec;
    gather_unit_kernel<<<(unsigned)((n + per_block - 1) / per_block), kThreads, 0, s>>>(src, lo, n, dst);
    return cudaGetLastError();
}

cudaError_t launch_gather_ranks(const ShardPtrs &src, int64_t S, int64_t lo, int64_t n, uint16_t *dst,
                                int32_t max_ctas, cudaStream_t s)
{
    if (n <= 0) return cudaSuccess;
    const int64_t per_block = (int64_t)kThreads * kCopyUnroll * kVec;
    int64_t grid = (n + per_block - 1) / per_block;
    if (max_ctas > 0 && grid > max_ctas) grid = max_ctas;
    gather_ranks_kernel<<<(unsigned)grid, kThreads, 0, s>>>(src, S, lo, n, dst);
    return cudaGetLastError();
}

cudaError_t launch_tile_index(Seg *segs, int64_t n_seg, cudaStream_t s)
{
    tile_index_kernel<<<1, 32, 0, s>>>(segs, n_seg);
    return cudaGetLastError();
}

cudaError_t launch_reduce_scatter(const zero_layout &L, const TileWork &w, const uint16_t *grads,
                                  int64_t stride, float *reduced, int32_t *nonfinite, cudaStream_t s)
{
    return dispatch_tiles<false>(L, w, grads, stride, reduced, nullptr, nullptr, nullptr, nullptr,
                                 AdamScalars{}, nonfinite, s);
}

cudaError_t launch_fused_step(const zero_layout &L, const TileWork &w, const uint16_t *grads,
                              int64_t stride, float *master, float *m, float *v, uint16_t *p16,
                              const AdamScalars &c, int32_t *nonfinite, cudaStream_t s, const AdamScalars *c_dev)
{
    return dispatch_tiles<true>(L, w, grads, stride, nullptr, master, m, v, p16, c, nonfinite, s, c_dev);
}

cudaError_t launch_fused_step_to(const zero_layout &L, const TileWork &w, const uint16_t *grads,
                                 int64_t stride, const float *master_in, const float *m_in, const float *v_in,
                                 float *master, float *m, float *v, uint16_t *p16, const AdamScalars &c,
                                 int32_t *nonfinite, cudaStream_t s)
{
    if (w.n_tiles <= 0) return cudaSuccess;
    auto kern = L.wire16 ? tile_kernel<0, 1, true, true, true> : tile_kernel<0, 1, true, false, true>;
    const int grid = grid_for(kern, w.n_tiles, L.dev.num_sms, w.max_ctas > 0 ? w.max_ctas : L.max_ctas);
    kern<<<grid, kThreads, 0, s>>>(w, L.n_ranks, grads, stride, nullptr, master, m, v, p16, c, nonfinite,
                                   StateIn{master_in, m_in, v_in}, nullptr);
    return cudaGetLastError();
}

cudaError_t launch_adamw_range(const zero_layout &L, int64_t lo, int64_t hi, const float *reduced,
                               float *master, float *m, float *v, uint16_t *p16,
                               const AdamScalars &c, cudaStream_t s)
{
    if (hi <= lo) return cudaSuccess;
    // one vector per thread: a grid of short blocks keeps the blocks in flight on a compact
    // window of the buffers (see copy_range_kernel)
    const int64_t blocks = (hi - lo + kThreads * kVec - 1) / (kThreads * kVec);
    (void)L;
    adamw_range_kernel<<<(unsigned)(blocks > 0 ? blocks : 1), kThreads, 0, s>>>(lo, hi, reduced, master, m, v, p16, c);
    return cudaGetLastError();
}

cudaError_t launch_copy_range(const zero_layout &L, int64_t lo, int64_t hi, const uint16_t *src,
                              uint16_t *dst, cudaStream_t s)
{
    if (hi <= lo) return cudaSuccess;
    const int64_t per_block = (int64_t)kThreads * kVec * kCopyUnroll;
    const int64_t va = (lo + kVec - 1) / kVec * kVec, vb = hi / kVec * kVec;
    if (L.gather_ctas > 0) {
        // head [lo, min(va, hi)) by one block's scalar pass, then [va, hi) vectorised
        const int64_t head_end = va < hi ? va : hi;
        return launch_copy_capped(src + head_end, dst + head_end, hi - head_end, src + lo, dst + lo,
                                  (int)(head_end - lo), L.gather_ctas, L.dev.error, L.dev.wait_limit_ns, s);
    }
    const int64_t blocks = vb > va ? (vb - va + per_block - 1) / per_block : 1;
    copy_range_kernel<<<(unsigned)blocks, kThreads, 0, s>>>(lo, hi, src, dst);
    return cudaGetLastError();
}

}  // namespace zero
