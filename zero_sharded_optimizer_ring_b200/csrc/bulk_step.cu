// Fused step, bulk-copy pipeline variant (sm_100a).
//
// Same computation as the register-streaming tile kernel (ring-order fp32 fold of the N
// ranks' fp16 gradients, scale, AdamW, fp16 write; rkmt.cn/news/44736 "DDP" and
// "Deepspeed ZeRO-1", en.pswp.cn/web/84187 "DDP"), staged differently:
//
//   warp 0, lane 0 (producer): for each chunk (2048 or 4096 elements) of its tiles, waits for a free
//     stage of a shared-memory ring, posts the stage's byte count on the stage's "full"
//     mbarrier and issues one plain cp.async.bulk (global -> this CTA's shared memory, no
//     tensor map) per gradient slice (ranks in ring order) and per state array;
//   warps 1..8 or 1..16 (consumers): wait for the stage to fill, fold / update from shared memory
//     (16-byte vectors, conflict-free for the gradients), store results with 16-byte
//     streaming stores, and release the stage on its "empty" mbarrier.
//
// Up to `stages` chunks are in flight per SM without holding any of them in registers,
// which is what the register-streaming variant lacks at high register counts.
//
// Every wait is bounded by the global timer.  When a wait expires the kernel writes
// ZERO_ERR_TIMEOUT to the error word, raises a CTA-wide abort flag that every other
// wait polls, the producer waits (again bounded) for the copies it has issued to land,
// and all threads return.  No trap, no unbounded spin.
#include <cuda_fp16.h>
#include <stdint.h>

#include "bulk_ptx.cuh"
#include "device_common.cuh"

namespace zero {
namespace {

// Pipeline shape per rank count, measured on B200 (kernel GB/s of the full step on the
// flat N=4, GPT-2 N=8, Llama N=8 and ragged N=16 workloads): larger single copies pay,
// but more than about 120-170 KB in flight per SM costs DRAM efficiency.  Few ranks:
// 4096-element chunks (one tile), 16 consumer warps, 2 stages.  More ranks: 2048-element
// chunks, 8 consumer warps, at most 3 stages.
//
// N = 0 is the runtime rank count (17..kMaxBulkRanks): a stage of (2n + 12) bytes per
// element grows with n, so the chunk is 1024 elements while two stages of it fit in
// shared memory and 512 above.  Folding that many ranks takes more consumer time per
// chunk than a few warps have, so this instance runs one group of 4 consumer warps per
// stage (group g takes the chunks of stage g), and consecutive chunks are folded in
// parallel; kConsumerWarps is then the size of one group.
template <int N>
struct BulkShape {
    static constexpr int kChunk = N <= 4 ? 4096 : 2048;        // elements per stage
    static constexpr int kConsumerWarps = N <= 4 ? 16 : 8;
    static constexpr int kThreads = 32 * (1 + kConsumerWarps);
    // stages in flight: two of the 4096-element chunks, three of the 2048-element ones (a
    // sweep of 2 against 3 on flat lists of 2^28 parameters: the third 4096-element stage,
    // 56-72 KB at 1-3 ranks, slows the step by 4-5 %; the third 2048-element stage at 8
    // ranks speeds it up by 7 %)
    static constexpr int kMaxStages = N <= 4 ? 2 : 3;
};

template <>
struct BulkShape<0> {
    static constexpr int kConsumerWarps = 4;      // per group; one group per stage
    static constexpr int kMaxStages = 3;
    static constexpr int kThreads = 32 * (1 + kConsumerWarps * kMaxStages);
};

// Bounded wait for the phase of `parity` to complete.  Returns false when the wait
// gave up (time limit, or another thread of the CTA raised the abort flag).
__device__ __forceinline__ bool wait_phase(uint32_t bar, uint32_t parity, volatile int *abort_flag,
                                           int32_t *error, uint64_t limit_ns)
{
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_ns();
    for (uint32_t i = 1;; ++i) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((i & 63u) == 0) {
            if (*abort_flag) return false;
            if (global_ns() - t0 > limit_ns) {
                atomicExch(error, (int32_t)ZERO_ERR_TIMEOUT);
                *abort_flag = 1;
                return false;
            }
        }
    }
}

struct BulkArgs {
    TileWork w;
    GradSource src;              // rank r's gradient of flat element i: src.rank[r][i]
    const float *master_in, *mom1_in, *mom2_in;  // state read: element i at [i - state_off]
    float *master, *mom1, *mom2;                 // state written (the same buffers, or a second set)
    int64_t state_off;
    uint16_t *p16;                // element i at [i - p16_off]
    int64_t p16_off;
    AdamScalars c;
    const AdamScalars *c_dev;    // non-null: the step's scalars are read from here at run time
    float *reduced;              // reduce-only instances: fp32 sums, element i at [i]
    int32_t *nonfinite;
    int32_t *error;
    uint64_t wait_limit_ns;
    int32_t stages;
    int32_t skip_first_fill;   // test hook: never post chunk 0, so its consumers' wait expires
    int32_t n_ranks, chunk;    // the runtime-N instance's rank count and elements per stage
};

// Shared memory: [full[S], empty[S] mbarriers][abort flag] ... stage ring (128-B aligned):
// stage s = N gradient slices of kChunk fp16, then master, m, v slices of kChunk fp32.
// The ring fold of one 16-byte vector (8 elements) from a stage: rank slices j = 0..n-1
// (already in ring order) at base + j * chunk elements.
template <int N, bool kWire>
__device__ __forceinline__ void fold8(const unsigned char *base, int64_t e0, int n, int chunk, float (&acc)[8])
{
    if constexpr (kWire) {
        uint4 h = *reinterpret_cast<const uint4 *>(base + e0 * 2);
        if constexpr (N > 0) {
#pragma unroll
            for (int j = 1; j < N; ++j)
                h = hadd8(h, *reinterpret_cast<const uint4 *>(base + ((size_t)j * chunk + e0) * 2));
        } else {
#pragma unroll 4
            for (int j = 1; j < n; ++j)
                h = hadd8(h, *reinterpret_cast<const uint4 *>(base + ((size_t)j * chunk + e0) * 2));
        }
        unpack8(h, acc);
    } else {
        unpack8(*reinterpret_cast<const uint4 *>(base + e0 * 2), acc);
        if constexpr (N > 0) {
#pragma unroll
            for (int j = 1; j < N; ++j) add8(acc, *reinterpret_cast<const uint4 *>(base + ((size_t)j * chunk + e0) * 2));
        } else {
#pragma unroll 4
            for (int j = 1; j < n; ++j) add8(acc, *reinterpret_cast<const uint4 *>(base + ((size_t)j * chunk + e0) * 2));
        }
    }
}

// kReduce: the reduce-scatter alone (zero_reduce_scatter): only the N gradient slices are
// staged, and the consumers store the fp32 sums instead of updating the state.
template <int N, bool kWire, bool kReduce>
__global__ void __launch_bounds__(BulkShape<N>::kThreads, 1) bulk_step_kernel(const __grid_constant__ BulkArgs A)
{
    constexpr int kConsumerWarps = BulkShape<N>::kConsumerWarps;
    // compile-time for N > 0, from the launch for the runtime-N instance
    int kChunk, n_r;
    if constexpr (N > 0) {
        kChunk = BulkShape<N>::kChunk;
        n_r = N;
    } else {
        kChunk = A.chunk;
        n_r = A.n_ranks;
    }
    const uint32_t kElemBytes = 2u * (uint32_t)n_r + (kReduce ? 0u : 12u);   // staged bytes per element
    const uint32_t kStageBytes = (uint32_t)kChunk * kElemBytes;
    const int groups = N > 0 ? 1 : A.stages;      // consumer groups (see BulkShape<0>)
    extern __shared__ __align__(128) unsigned char smem[];
    uint64_t *full = reinterpret_cast<uint64_t *>(smem);
    uint64_t *empty = full + A.stages;
    volatile int *abort_flag = reinterpret_cast<volatile int *>(empty + A.stages);
    unsigned char *ring = smem + ((16 * A.stages + 4 + 127) / 128) * 128;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < A.stages; ++s) {
            mbar_init(smem_addr(&full[s]), 1);
            mbar_init(smem_addr(&empty[s]), kConsumerWarps);
        }
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();

    const int64_t t_end = A.w.tile_first + A.w.n_tiles;
    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane != 0) return;
        int64_t s = A.w.seg_first;
        uint32_t it = 0;          // chunks issued (or deliberately skipped by the test hook)
        uint32_t posted = 0;      // chunks whose copies were issued
        bool ok = true;
        for (int64_t t = A.w.tile_first + blockIdx.x; ok && t < t_end; t += gridDim.x) {
            const TileRange tr = locate_tile(A.w, s, t);
            if (!tile_in_bounds(A.w, s, tr)) continue;     // debug builds; the consumers skip it too
            const int64_t va = (tr.a + kVec - 1) / kVec * kVec, vb = tr.b / kVec * kVec;
            for (int64_t q0 = va; ok && q0 < vb; q0 += kChunk, ++it) {
                const uint32_t st = it % (uint32_t)A.stages, ph = (it / (uint32_t)A.stages) & 1u;
                if (!wait_phase(smem_addr(&empty[st]), ph ^ 1u, abort_flag, A.error, A.wait_limit_ns)) {
                    ok = false;
                    break;
                }
                if (A.skip_first_fill && it == 0) continue;
                const uint32_t n = (uint32_t)((vb - q0) < kChunk ? (vb - q0) : kChunk);
                const uint32_t bar = smem_addr(&full[st]);
                unsigned char *base = ring + (size_t)st * kStageBytes;
                mbar_arrive_expect_tx(bar, n * kElemBytes);
                if constexpr (N > 0) {
#pragma unroll
                    for (int j = 0; j < N; ++j)
                        bulk_load(smem_addr(base + (size_t)j * kChunk * 2),
                                  A.src.rank[ring_rank(tr.shard, j, N)] + q0, n * 2u, bar);
                } else {
                    for (int j = 0; j < n_r; ++j)
                        bulk_load(smem_addr(base + (size_t)j * kChunk * 2),
                                  A.src.rank[ring_rank(tr.shard, j, n_r)] + q0, n * 2u, bar);
                }
                if constexpr (!kReduce) {
                    unsigned char *st_base = base + (size_t)n_r * kChunk * 2;
                    bulk_load(smem_addr(st_base), A.master_in + (q0 - A.state_off), n * 4u, bar);
                    bulk_load(smem_addr(st_base + kChunk * 4), A.mom1_in + (q0 - A.state_off), n * 4u, bar);
                    bulk_load(smem_addr(st_base + kChunk * 8), A.mom2_in + (q0 - A.state_off), n * 4u, bar);
                }
                posted = it + 1;
            }
        }
        // Drain: every stage whose copies were issued must have landed before the CTA's
        // shared memory goes away (normally the consumers have already seen them).
        const uint32_t first = posted > (uint32_t)A.stages ? posted - (uint32_t)A.stages : 0u;
        for (uint32_t i = first; i < posted; ++i) {
            if (A.skip_first_fill && i == 0) continue;
            const uint32_t st = i % (uint32_t)A.stages, ph = (i / (uint32_t)A.stages) & 1u;
            const uint64_t t0 = global_ns();
            while (!mbar_try_wait(smem_addr(&full[st]), ph) && global_ns() - t0 < A.wait_limit_ns) {
            }
        }
        return;
    }

    // ---------------------------------------------------------------- consumers
    const int grp = (warp - 1) / kConsumerWarps;  // consumer group: takes the chunks of stage grp
    if (grp >= groups) return;
    const int ct = threadIdx.x - 32 - grp * 32 * kConsumerWarps;   // 0 .. 32 * kConsumerWarps - 1
    const AdamScalars c = (!kReduce && A.c_dev) ? *A.c_dev : A.c;
    int64_t s = A.w.seg_first;
    uint32_t it = 0;
    for (int64_t t = A.w.tile_first + blockIdx.x; t < t_end; t += gridDim.x) {
        const TileRange tr = locate_tile(A.w, s, t);
        if (!tile_in_bounds(A.w, s, tr)) continue;
        const int64_t va = (tr.a + kVec - 1) / kVec * kVec, vb = tr.b / kVec * kVec;
        int bad = 0;
        for (int64_t q0 = va; q0 < vb; q0 += kChunk, ++it) {
            if (groups > 1 && (int)(it % (uint32_t)groups) != grp) continue;   // another group's stage
            const uint32_t st = it % (uint32_t)A.stages, ph = (it / (uint32_t)A.stages) & 1u;
            // every lane waits (acquiring the stage's data); the warp leaves together
            const bool got = wait_phase(smem_addr(&full[st]), ph, abort_flag, A.error, A.wait_limit_ns);
            if (!__all_sync(0xffffffffu, got)) return;
            const int64_t n = (vb - q0) < kChunk ? (vb - q0) : kChunk;
            const unsigned char *base = ring + (size_t)st * kStageBytes;
            for (int64_t vi = ct; vi * kVec < n; vi += 32 * kConsumerWarps) {
                const int64_t e0 = vi * kVec;
                float acc[8];
                fold8<N, kWire>(base, e0, n_r, kChunk, acc);
                if constexpr (kReduce) {
#pragma unroll
                    for (int e = 0; e < 8; ++e) bad += !isfinite(acc[e]);
                    float4 *rp = reinterpret_cast<float4 *>(A.reduced + (q0 + e0));
                    __stcs(rp, make_float4(acc[0], acc[1], acc[2], acc[3]));
                    __stcs(rp + 1, make_float4(acc[4], acc[5], acc[6], acc[7]));
                    continue;
                }
                const float *sp = reinterpret_cast<const float *>(base + (size_t)n_r * kChunk * 2);
                float4 p4[2] = {*reinterpret_cast<const float4 *>(sp + e0), *reinterpret_cast<const float4 *>(sp + e0 + 4)};
                float4 m4[2] = {*reinterpret_cast<const float4 *>(sp + kChunk + e0),
                                *reinterpret_cast<const float4 *>(sp + kChunk + e0 + 4)};
                float4 v4[2] = {*reinterpret_cast<const float4 *>(sp + 2 * kChunk + e0),
                                *reinterpret_cast<const float4 *>(sp + 2 * kChunk + e0 + 4)};
                float *pf = reinterpret_cast<float *>(p4);
                float *mf = reinterpret_cast<float *>(m4);
                float *vf = reinterpret_cast<float *>(v4);
                uint32_t h[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) bad += !isfinite(acc[e]);
                adamw8(acc, c, pf, mf, vf, h);
                const int64_t q = q0 + e0;
                float4 *pp = reinterpret_cast<float4 *>(A.master + (q - A.state_off));
                float4 *mp = reinterpret_cast<float4 *>(A.mom1 + (q - A.state_off));
                float4 *vp = reinterpret_cast<float4 *>(A.mom2 + (q - A.state_off));
                __stcs(pp, p4[0]); __stcs(pp + 1, p4[1]);
                __stcs(mp, m4[0]); __stcs(mp + 1, m4[1]);
                __stcs(vp, v4[0]); __stcs(vp + 1, v4[1]);
                __stcs(reinterpret_cast<uint4 *>(A.p16 + (q - A.p16_off)),
                       make_uint4(h[0] | (h[1] << 16), h[2] | (h[3] << 16), h[4] | (h[5] << 16), h[6] | (h[7] << 16)));
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_addr(&empty[st]));
        }

        // ragged edges of the tile, straight from global memory
        const int64_t head_end = va < tr.b ? va : tr.b;
        const int64_t tail_begin = vb > head_end ? vb : head_end;
        const int64_t n_head = head_end - tr.a, n_tail = tr.b - tail_begin;
        if (grp == 0 && ct < n_head + n_tail) {
            const int64_t i = ct < n_head ? tr.a + ct : tail_begin + (ct - n_head);
            float acc;
            if constexpr (kWire) {
                uint32_t h = A.src.rank[tr.shard][i];
                for (int j = 1; j < n_r; ++j) h = hadd1(h, A.src.rank[ring_rank(tr.shard, j, n_r)][i]);
                acc = h2f(h);
            } else {
                acc = h2f(A.src.rank[tr.shard][i]);
                for (int j = 1; j < n_r; ++j) acc = __fadd_rn(acc, h2f(A.src.rank[ring_rank(tr.shard, j, n_r)][i]));
            }
            bad += !isfinite(acc);
            if constexpr (kReduce) {
                A.reduced[i] = acc;
            } else {
            const int64_t si = i - A.state_off;
            float p = A.master_in[si], m = A.mom1_in[si], v = A.mom2_in[si];
            uint32_t h;
            adamw_elem(acc, c, p, m, v, h);
            A.master[si] = p;
            A.mom1[si] = m;
            A.mom2[si] = v;
            A.p16[i - A.p16_off] = (uint16_t)h;
            }
        }
        if (A.nonfinite) {
            if (__any_sync(0xffffffffu, bad != 0)) {
                const int total = __reduce_add_sync(0xffffffffu, bad);
                if (lane == 0) atomicAdd(A.nonfinite + tr.bucket, total);
            }
        }
    }
}

template <int N, bool kReduce>
cudaError_t launch_bulk_n(const zero_layout &L, BulkArgs &a, cudaStream_t st)
{
    const size_t budget = L.dev.smem_optin > 0 ? L.dev.smem_optin : 227 * 1024;
    const size_t per_elem = 2 * (size_t)L.n_ranks + (kReduce ? 0 : 12);
    size_t stage_bytes;
    if constexpr (N > 0) {
        stage_bytes = (size_t)BulkShape<N>::kChunk * per_elem;
    } else {
        a.n_ranks = L.n_ranks;
        a.chunk = 2 * 1024 * per_elem + 256 <= budget ? 1024 : 512;
        stage_bytes = (size_t)a.chunk * per_elem;
    }
    int stages = (int)((budget - 256) / stage_bytes);
    int max_stages = BulkShape<N>::kMaxStages;
    if (kReduce && N > 0) {
        // the smaller reduce-only stages: as many as keep about 170 KB in flight per SM
        // (the sweep's sweet spot for the fused step), at most 5
        const int by_flight = (int)((170 * 1024) / stage_bytes);
        max_stages = by_flight < 5 ? by_flight : 5;
        if (max_stages < 2) max_stages = 2;
    }
    if (stages > max_stages) stages = max_stages;
    if (stages < 2) return cudaErrorInvalidConfiguration;
    a.stages = stages;
    const size_t smem = ((16 * (size_t)stages + 4 + 127) / 128) * 128 + (size_t)stages * stage_bytes;
    auto kern = L.wire16 ? bulk_step_kernel<N, true, kReduce> : bulk_step_kernel<N, false, kReduce>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    int64_t grid = L.dev.num_sms > 0 ? L.dev.num_sms : 148;
    const int32_t cap = a.w.max_ctas > 0 ? a.w.max_ctas : L.max_ctas;
    if (cap > 0 && grid > cap) grid = cap;
    if (grid > a.w.n_tiles) grid = a.w.n_tiles;
    kern<<<(unsigned)grid, BulkShape<N>::kThreads, smem, st>>>(a);
    return cudaGetLastError();
}

template <bool kReduce>
cudaError_t dispatch_bulk(const zero_layout &L, BulkArgs &a, cudaStream_t st)
{
    switch (L.n_ranks) {
        case 1: return launch_bulk_n<1, kReduce>(L, a, st);
        case 2: return launch_bulk_n<2, kReduce>(L, a, st);
        case 3: return launch_bulk_n<3, kReduce>(L, a, st);
        case 4: return launch_bulk_n<4, kReduce>(L, a, st);
        case 5: return launch_bulk_n<5, kReduce>(L, a, st);
        case 6: return launch_bulk_n<6, kReduce>(L, a, st);
        case 7: return launch_bulk_n<7, kReduce>(L, a, st);
        case 8: return launch_bulk_n<8, kReduce>(L, a, st);
        case 9: return launch_bulk_n<9, kReduce>(L, a, st);
        case 10: return launch_bulk_n<10, kReduce>(L, a, st);
        case 11: return launch_bulk_n<11, kReduce>(L, a, st);
        case 12: return launch_bulk_n<12, kReduce>(L, a, st);
        case 13: return launch_bulk_n<13, kReduce>(L, a, st);
        case 14: return launch_bulk_n<14, kReduce>(L, a, st);
        case 15: return launch_bulk_n<15, kReduce>(L, a, st);
        case 16: return launch_bulk_n<16, kReduce>(L, a, st);
        default:
            if (L.n_ranks > kMaxBulkRanks || L.n_ranks < 1) return cudaErrorInvalidValue;
            return launch_bulk_n<0, kReduce>(L, a, st);
    }
}

}  // namespace

bool bulk_supported(int n_ranks) { return n_ranks >= 1 && n_ranks <= kMaxBulkRanks; }

// The automatic choice (impl 0) for a strided gradient buffer, from B200 measurements of
// both kernels: the pipeline where it has a compiled instance (N <= 16; level with
// register streaming at 1-4 ranks, 9 % ahead of it on the Llama-shaped list at 8 ranks and
// 2 % on the ragged list at 16), register streaming above (0.99-1.01 of the
// measured copy bandwidth at N = 24-64, where the runtime-N pipeline instance reaches
// 0.48-0.87: its few consumer warps cannot fold that many ranks fast enough).
bool use_bulk(const zero_layout &L)
{
    if (L.impl == 1) return false;
    if (L.impl == 2) return bulk_supported(L.n_ranks);
    return L.n_ranks >= 1 && L.n_ranks <= 16;
}

// The same for the reduce-scatter alone: the reduce-only pipeline for 5-16 ranks (6 % and
// 10 % ahead of register streaming at 8 and 16), register streaming for 1-4 ranks (level
// at 3, 3-12 % ahead at 1, 2 and 4, where the pipeline's 16 consumer warps have little
// to fold per byte staged) and above 16 (0.97-1.00 of the copy bandwidth at 24-48 ranks,
// the runtime-N pipeline instance 0.77-0.83).
bool use_bulk_reduce(const zero_layout &L)
{
    if (L.impl == 1) return false;
    if (L.impl == 2) return bulk_supported(L.n_ranks);
    return L.n_ranks >= 5 && L.n_ranks <= 16;
}

cudaError_t launch_bulk_step(const zero_layout &L, const TileWork &w, const GradSource &src, float *master,
                             float *m, float *v, int64_t state_off, uint16_t *p16, int64_t p16_off,
                             const AdamScalars &c, int32_t *nonfinite, uint64_t wait_limit_ns,
                             int skip_first_fill, cudaStream_t st, const float *master_in,
                             const float *m_in, const float *v_in, const AdamScalars *c_dev)
{
    if (w.n_tiles <= 0) return cudaSuccess;
    if ((state_off & 7) != 0 || (p16_off & 7) != 0) return cudaErrorMisalignedAddress;
    BulkArgs a;
    a.w = w;
    a.src = src;
    a.master = master;
    a.mom1 = m;
    a.mom2 = v;
    a.master_in = master_in ? master_in : master;
    a.mom1_in = m_in ? m_in : m;
    a.mom2_in = v_in ? v_in : v;
    a.state_off = state_off;
    a.p16 = p16;
    a.p16_off = p16_off;
    a.c = c;
    a.c_dev = c_dev;
    a.nonfinite = nonfinite;
    a.error = L.dev.error;
    a.wait_limit_ns = wait_limit_ns;
    a.stages = 0;
    a.skip_first_fill = skip_first_fill;
    a.n_ranks = L.n_ranks;
    a.chunk = 0;
    a.reduced = nullptr;
    return dispatch_bulk<false>(L, a, st);
}

cudaError_t launch_bulk_reduce(const zero_layout &L, const TileWork &w, const GradSource &src, float *reduced,
                               int32_t *nonfinite, uint64_t wait_limit_ns, cudaStream_t st)
{
    if (w.n_tiles <= 0) return cudaSuccess;
    BulkArgs a = {};
    a.w = w;
    a.src = src;
    a.reduced = reduced;
    a.nonfinite = nonfinite;
    a.error = L.dev.error;
    a.wait_limit_ns = wait_limit_ns;
    a.n_ranks = L.n_ranks;
    return dispatch_bulk<true>(L, a, st);
}

}  // namespace zero
