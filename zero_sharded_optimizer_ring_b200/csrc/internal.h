// Internal definitions shared by the library's translation units (not installed).
#pragma once

#include <cuda_runtime.h>
#include <nvtx3/nvToolsExt.h>
#include <stdint.h>

#include <vector>

#include "zero.h"

// One named NVTX range per ABI call, so that a profiler's timeline (or an ncu --nvtx
// filter) shows which entry point launched which kernels.  Without an attached tool the
// push and pop are a test of a null pointer each.
#define ZERO_RANGE(name) zero::CallRange zero_call_range_(name)

namespace zero {

struct CallRange {
    explicit CallRange(const char *name) { nvtxRangePushA(name); }
    ~CallRange() { nvtxRangePop(); }
    CallRange(const CallRange &) = delete;
    CallRange &operator=(const CallRange &) = delete;
};

// Elements per tile: the unit of work one CTA picks up.  A multiple of 8 so that
// tile boundaries fall on 16-byte fp16 vectors.
constexpr int64_t kTileElems = 4096;

// One row of the segment table: chunk `shard` of bucket `bucket`, flat range [lo, hi),
// whose tiles are numbered tile_begin .. next row's tile_begin - 1.
struct Seg {
    int64_t lo, hi, tile_begin;
    int32_t shard, bucket;
};
static_assert(sizeof(Seg) == 32, "device table row is 32 bytes");

// Where each rank's gradients live for the bulk pipeline: rank r's value of flat element i
// is rank[r][i].  One strided buffer (rank[r] = grads + r * stride), separate buffers on
// this GPU, or other GPUs' buffers mapped into this process.
constexpr int kMaxBulkRanks = 64;
struct GradSource {
    const uint16_t *rank[kMaxBulkRanks];
};

// fp32 scalars of one AdamW step, each computed on the host in double and rounded once
// (the layout of zero_step_scalars in zero.h, which the library copies it to and from).
struct AdamScalars {
    float inv_scale;   // 1 / (N * loss_scale)
    float decay;       // 1 - lr * weight_decay
    float beta1, omb1; // beta1, 1 - beta1
    float beta2, omb2; // beta2, 1 - beta2
    float step_size;   // lr / (1 - beta1^t)
    float sqrt_bc2;    // sqrt(1 - beta2^t)
    float eps;
};
static_assert(sizeof(AdamScalars) == sizeof(zero_step_scalars), "same layout as zero_step_scalars");

// What a debug build (ZERO_DEBUG) checks every located tile against; filled by the
// launch wrappers, read by no release kernel.  A tile that fails the check is skipped and
// ZERO_ERR_BOUNDS is recorded in `error` (when non-null); nothing is read or written out
// of bounds and nothing traps.
struct TileBounds {
    int64_t n_seg = 0;                   // table rows before the closing row
    int64_t padded = 0, shard = 0;       // P, S
    int64_t state_lo = 0, state_hi = 0;  // flat range the state buffers of the launch cover
    int32_t n_ranks = 0, n_buckets = 0;
    int32_t *error = nullptr;            // device error word
};

// Launch arguments of the tile-walking kernels (reduce-scatter, fused step).
struct TileWork {
    const Seg *segs;       // device segment table (n_seg + 1 rows, last = sentinel)
    int64_t seg_first;     // first row of the launch's range
    int64_t tile_first;    // first global tile of the launch
    int64_t n_tiles;       // tiles in the launch
    TileBounds bounds;     // debug builds only
    int32_t max_ctas = 0;  // > 0: this launch's grid cap (overrides the layout's)
};

// Launch-plan tuning of the overlapped step: candidate plans (the update's grid capped at
// 1, 2/3, 1/2 or 1/3 of the SMs while it follows the backward bucket by bucket, or the
// whole update deferred to one full-grid launch after the last bucket) are each timed
// over whole calls (CUDA events on the caller's stream, first wait to last launch),
// round-robin after one untimed warm-up call, kTrials times each, rounds alternating
// direction; then the plan with the lowest mean is kept.  Nothing ever waits on these events: a call issued before the
// previous timed call has finished on the GPU is not timed.
struct OverlapTuner {
    static constexpr int kCands = 5, kTrials = 2;
    float sum_ms[kCands] = {0.f, 0.f, 0.f, 0.f, 0.f};
    int32_t trials[kCands] = {0, 0, 0, 0, 0};
    int32_t calls = 0;                    // calls seen (the first is a warm-up)
    int32_t pending = -1;                 // candidate whose timed call is in flight
    int32_t chosen = -1;                  // the kept plan, once every candidate is timed
    cudaEvent_t begin = nullptr, end = nullptr;
};

struct DeviceState {
    int device = -1;
    Seg *segs = nullptr;          // n_seg + 1 rows
    Seg *segs_by_shard = nullptr; // the same rows ordered by shard, then bucket (+ closing row)
    int32_t *error = nullptr;     // device error word (timeouts)
    int num_sms = 0;
    size_t smem_optin = 0;
    cudaStream_t copy_in = nullptr, copy_out = nullptr;   // zero_step_host
    std::vector<cudaEvent_t> landed, updated;              // per bucket
    cudaEvent_t begin = nullptr, done = nullptr;           // per zero_step_host call
    mutable OverlapTuner tuner;               // zero_step_overlapped's default grid choice
    uint64_t wait_limit_ns = 2000000000ull;   // bound of every in-kernel wait (2 s)
    int32_t skip_first_fill = 0;              // test hook of the bulk pipeline (see zero.h)
};

}  // namespace zero

struct zero_layout {
    int32_t n_ranks = 0, stage = 0;
    int32_t wire16 = 0;                        // 1: partials travel the ring as fp16
    int64_t psi = 0, shard = 0, padded = 0, pad_align = 1, bucket_elems = 0;
    std::vector<int64_t> tensor_off;
    std::vector<int64_t> bucket_lo, bucket_hi;
    std::vector<int64_t> bucket_seg_begin;     // n_buckets + 1: first segment of each bucket
    std::vector<zero::Seg> segs;               // host copy, tile_begin filled on the host too
    zero::Seg closing{};                       // the table's closing row: lo = hi = P, shard = bucket = -1
    std::vector<zero::Seg> segs_by_shard;      // shard-major order, with its own tile numbering
    std::vector<int64_t> shard_seg_begin;      // n_ranks + 1: first shard-major row of each shard
    std::vector<int64_t> unit_lo, unit_hi;
    int64_t n_tiles = 0;
    int32_t impl = 0;
    int32_t max_ctas = 0;                      // > 0: cap on the grid of the tile-walking kernels
    int32_t gather_ctas = 0;                   // > 0: the gathers run as that many persistent CTAs
    zero::DeviceState dev;
};

namespace zero {

// abi.cu: hyper-parameter rules shared by every step entry point, and the step's fp32
// scalars (each evaluated in double and rounded once).
zero_status check_hparams(const zero_adamw_hparams *h);
AdamScalars step_scalars(int32_t n_ranks, const zero_adamw_hparams &h);

// kernels.cu
// The bounds of a launch over layout L whose state buffers cover flat [state_lo, state_hi).
TileBounds tile_bounds(const zero_layout &L, int64_t state_lo, int64_t state_hi);
cudaError_t launch_tile_index(Seg *segs, int64_t n_seg, cudaStream_t s);
cudaError_t launch_reduce_scatter(const zero_layout &L, const TileWork &w, const uint16_t *grads,
                                  int64_t stride, float *reduced, int32_t *nonfinite, cudaStream_t s);
cudaError_t launch_adamw_range(const zero_layout &L, int64_t lo, int64_t hi, const float *reduced,
                               float *master, float *m, float *v, uint16_t *p16,
                               const AdamScalars &c, cudaStream_t s);
cudaError_t launch_copy_range(const zero_layout &L, int64_t lo, int64_t hi, const uint16_t *src,
                              uint16_t *dst, cudaStream_t s);
// max_ctas > 0 (and lo a multiple of 8): the capped bulk copy, whose bounded waits report
// to `error` (may be null)
cudaError_t launch_gather_unit(const uint16_t *src, int64_t lo, int64_t n, uint16_t *dst, int32_t max_ctas,
                               int32_t *error, uint64_t limit_ns, cudaStream_t s);
// c_dev non-null: the scalars are read from device memory when the kernel runs (c unused)
cudaError_t launch_fused_step(const zero_layout &L, const TileWork &w, const uint16_t *grads,
                              int64_t stride, float *master, float *m, float *v, uint16_t *p16,
                              const AdamScalars &c, int32_t *nonfinite, cudaStream_t s,
                              const AdamScalars *c_dev = nullptr);
// The same update out of place (register streaming, any N): state read from *_in,
// written to master / m / v (buffers that do not overlap the in set).
cudaError_t launch_fused_step_to(const zero_layout &L, const TileWork &w, const uint16_t *grads,
                                 int64_t stride, const float *master_in, const float *m_in, const float *v_in,
                                 float *master, float *m, float *v, uint16_t *p16, const AdamScalars &c,
                                 int32_t *nonfinite, cudaStream_t s);

// bulk_step.cu
bool bulk_supported(int n_ranks);
// The reduce-scatter alone through the bulk-copy pipeline: reduced[i] = the ring-order
// fp32 sum of element i, for the tiles of `w` (rank r's gradient of i at src.rank[r][i]).
cudaError_t launch_bulk_reduce(const zero_layout &L, const TileWork &w, const GradSource &src, float *reduced,
                               int32_t *nonfinite, uint64_t wait_limit_ns, cudaStream_t st);
bool use_bulk(const zero_layout &L);          // the fused step's implementation for a strided buffer
bool use_bulk_reduce(const zero_layout &L);   // the same for the reduce-scatter alone
// master / m / v hold flat elements [state_off, ...) and p16 [p16_off, ...): element i is
// at index i - off (both offsets multiples of 8).  The state is read from master_in /
// m_in / v_in where given (same indexing; a second buffer set), else from master / m / v.
cudaError_t launch_bulk_step(const zero_layout &L, const TileWork &w, const GradSource &src, float *master,
                             float *m, float *v, int64_t state_off, uint16_t *p16, int64_t p16_off,
                             const AdamScalars &c, int32_t *nonfinite, uint64_t wait_limit_ns,
                             int skip_first_fill, cudaStream_t st, const float *master_in = nullptr,
                             const float *m_in = nullptr, const float *v_in = nullptr,
                             const AdamScalars *c_dev = nullptr);

}  // namespace zero
