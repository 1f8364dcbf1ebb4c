/*
 * zero.h -- C ABI of the sharded data-parallel optimizer step (DDP, ZeRO-1/2/3) on one
 * B200: N data-parallel ranks are simulated as N gradient buffers in one GPU's HBM.
 *
 * Sources (page address, then section):
 *   P1 = rkmt.cn/news/44736           (sections DP, DDP, Deepspeed ZeRO, ZeRO-1/-2/-3, 总结)
 *   P2 = wangyh.co PaperReading:DeepSpeed (sections 1.1-1.5, 2.1-2.6, 3)
 *   P3 = en.pswp.cn/web/84187          (sections DP, DDP, FSDP)
 *
 * Conventions shared by every call:
 *  - psi  = number of parameters (sum of the tensor sizes), N = ranks,
 *    S    = shard = roundup(ceil(psi / N), pad_align), P = padded = N * S.
 *    All flat buffers are indexed by the flat parameter index 0 .. P-1; tensors are
 *    concatenated in list order with no per-tensor padding; [psi, P) is tail padding,
 *    which must hold zeros in gradients and state on entry (it then stays zero).
 *  - Shard k is [k*S, (k+1)*S) (P1 Deepspeed ZeRO-1: each of 3 GPUs is responsible for
 *    one third).  Buckets are fixed ranges of bucket_elems elements cut from the TAIL of
 *    the padded buffer: bucket 0 = [P - B, P), the gradients a backward pass produces
 *    first (P1 DDP and ZeRO-1/-2: gradients are computed back to front and synced group
 *    by group; P3 DDP: parameters are reduced bucket by bucket).  A segment is a bucket
 *    intersected with a shard: chunk k of that bucket's ring.
 *  - fp16 values are passed as uint16_t bit patterns.  Device pointers are caller-owned
 *    device memory (e.g. from PyTorch), 16-byte aligned; element strides are multiples
 *    of 8.  The library never frees or retains caller memory.
 *  - Every device call is asynchronous on `stream` (a cudaStream_t, NULL = legacy
 *    default stream) of the CUDA device the layout was uploaded to, which must be the
 *    current device.  Argument errors return before anything is launched.  Launch
 *    failures return ZERO_ERR_CUDA.  A kernel that gives up a bounded wait records
 *    ZERO_ERR_TIMEOUT in a device error word that zero_get_error() reports.
 *  - Arithmetic: every reduction and update step is one IEEE-754 binary32 operation,
 *    rounded to nearest even, no fused multiply-add, no flush of subnormals.
 */
#ifndef ZERO_H
#define ZERO_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    ZERO_OK = 0,
    ZERO_ERR_INVALID = 1,   /* bad argument: NULL where required, size or index out of range */
    ZERO_ERR_ALIGN = 2,     /* a device pointer not 16-byte aligned, or a stride not a multiple of 8 */
    ZERO_ERR_CUDA = 3,      /* a CUDA runtime call or kernel launch failed */
    ZERO_ERR_OOM = 4,       /* allocation of the layout's own tables failed */
    ZERO_ERR_TIMEOUT = 5,   /* a bounded wait inside a kernel gave up (see zero_get_error) */
    ZERO_ERR_STATE = 6,     /* layout not uploaded, or uploaded to another device */
    ZERO_ERR_BOUNDS = 7     /* debug build only (ZERO_DEBUG): a kernel found a segment or tile
                               index outside the layout's table or buffers, skipped that tile
                               and recorded this code (see zero_get_error) */
} zero_status;

typedef struct zero_layout zero_layout;   /* opaque; owned by the library */

/* Layout description: what a DeepSpeed-style config names (P2 section 2.2-2.4:
 * zero_optimization.stage), plus the model's parameter list and the bucket size. */
typedef struct {
    int32_t n_ranks;                    /* N >= 1 simulated data-parallel ranks */
    int32_t stage;                      /* 0 = DDP (ZeRO-0), 1, 2, 3 (P2 section 1) */
    int64_t n_tensors;                  /* >= 0 */
    const int64_t *tensor_numel;        /* [n_tensors], each >= 0 (host memory, copied) */
    int64_t bucket_elems;               /* bucket size in elements; <= 0: one bucket */
    int64_t pad_align;                  /* shard rounding in elements, >= 1 (128 typical) */
    int64_t n_units;                    /* stage-3 gather units (layers); 0 = one unit */
    const int64_t *unit_first_tensor;   /* [n_units]: first tensor of each unit; [0] == 0,
                                           strictly increasing (host memory, copied) */
    int32_t wire_fp16;                  /* 0: the ring's partial sums are fp32 (one fp32
                                           rounding per add); 1: they travel as fp16, each
                                           hop's sum rounded to fp16 (P1 Deepspeed ZeRO-1:
                                           each GPU ends with its part's gradient mean in
                                           fp16); sums beyond 65504 then overflow to inf */
} zero_layout_desc;

typedef struct {
    int64_t psi, shard, padded;         /* psi, S, P */
    int64_t n_buckets, n_segments, n_units;
    int64_t tile_elems, n_tiles;        /* the kernels' work decomposition of the segments */
} zero_layout_info;

/* AdamW hyper-parameters of one step (step >= 1, counted from 1 for every run). */
typedef struct {
    double lr, beta1, beta2, eps, weight_decay;
    double loss_scale;                  /* L > 0: gradients arrive multiplied by L */
    int64_t step;
} zero_adamw_hparams;

/* Modelled per-rank memory (bytes) and communication (elements) of one training step.
 * Memory: P1 Deepspeed ZeRO (2B fp16 params + 2B fp16 grads + 12B optimizer state per
 * parameter for DDP; ZeRO-1 shards the optimizer state, ZeRO-2 also the gradients,
 * ZeRO-3 also the parameters).  Communication: P1 DDP (N-1 rounds of psi/N per phase,
 * two phases), ZeRO-1/-2 (same as DDP), ZeRO-3 (a third phase: 3 psi, 1.5x DDP). */
typedef struct {
    int64_t mem_p16, mem_g16, mem_os, mem_total;
    int64_t sent_elems, recv_elems;
} zero_counters;

/* Dynamic loss scaling state (host memory, updated by zero_step_dynamic).  Mixed-precision
 * practice (the pages do not spell it out): gradients arrive multiplied by `scale`; a
 * step whose reduced gradients hold a non-finite value is skipped and the scale divided by
 * `factor` (not below `min_scale`); after `window` applied steps in a row it is multiplied
 * by `factor`.  `step` counts applied AdamW steps: the next applied step uses step + 1. */
typedef struct {
    double scale;           /* > 0 */
    double factor;          /* > 1 */
    int64_t window;         /* >= 1 */
    double min_scale;       /* > 0 */
    int64_t clean_steps;    /* state: applied steps since the scale last changed */
    int64_t step;           /* state: applied AdamW steps so far */
    int64_t skipped;        /* state: steps skipped for overflow */
} zero_loss_scaler;

/* The fp32 scalars of one AdamW step as the kernels read them (the update formula of
 * zero_adamw_shard_step): 1/(N L), 1 - lr wd, beta1, 1 - beta1, beta2, 1 - beta2,
 * lr / (1 - beta1^t), sqrt(1 - beta2^t), eps; each evaluated in double and rounded once
 * to fp32.  zero_step_scalars_fill computes them; zero_step_device_scalars reads them from
 * device memory. */
typedef struct {
    float inv_scale, decay, beta1, omb1, beta2, omb2, step_size, sqrt_bc2, eps;
} zero_step_scalars;

/* Optional CUDA events (cudaEvent_t, created by the caller; any may be NULL) that
 * zero_step records on `stream` around its kernels, for per-kernel timing. */
typedef struct {
    void *update_begin, *update_end;    /* the fused reduce-scatter + update kernel */
    void *gather_begin, *gather_end;    /* the stage-3 all-gather kernel */
} zero_step_events;

/* ---- layout (host) ------------------------------------------------------------ */

/* Partition the flat parameter buffer into shards, buckets, segments and gather units.
 * Host-only work; no CUDA call.  *out must be released with zero_layout_destroy. */
zero_status zero_layout_create(const zero_layout_desc *desc, zero_layout **out);
void zero_layout_destroy(zero_layout *layout);
zero_status zero_layout_get_info(const zero_layout *layout, zero_layout_info *info);

/* Host copies of the tables (any pointer may be NULL):
 *   tensor_off [n_tensors]        flat offset of each tensor
 *   bucket_lohi [n_buckets][2]    bucket ranges, bucket order (bucket 0 = tail)
 *   segments [n_segments][4]      bucket, shard, lo, hi; bucket order, then shard order
 *   unit_lohi [n_units][2]        gather-unit ranges, ascending, covering [0, P) */
zero_status zero_layout_get_tables(const zero_layout *layout, int64_t *tensor_off,
                                   int64_t *bucket_lohi, int64_t *segments, int64_t *unit_lohi);
zero_status zero_layout_counters(const zero_layout *layout, zero_counters *out);

/* Upload the segment table to the current CUDA device and build the tile index on it
 * (a one-warp prefix scan of the segments' tile counts).  Allocates the layout's small
 * device tables (about 40 bytes per segment); must precede every device call. */
zero_status zero_layout_to_device(zero_layout *layout, void *stream);

/* Copy back the device-built table: [n_segments + 1][5] = bucket, shard, lo, hi,
 * first tile (the last row holds -1, -1, P, P, total tiles).  Synchronises `stream`. */
zero_status zero_layout_device_segments(const zero_layout *layout, int64_t *host_out, void *stream);

/* ---- the hot path (device) ------------------------------------------------------ */

/* Ring reduce-scatter of bucket `bucket` (-1 = every bucket, in bucket order).
 * P3 DDP (three-GPU walk-through) and P1 DDP (scatter-reduce: values passed on and
 * added): chunk k of the bucket starts at rank k and accumulates ranks k+1, k+2, ...
 * (mod N).  For each flat index i of the bucket, in shard k:
 *     reduced[i] = (...((f32(g_k[i]) + f32(g_{k+1}[i])) + f32(g_{k+2}[i])) ...)
 * with g_r[i] = grads[r * rank_stride + i] (fp16, rank_stride >= P, multiple of 8).
 * reduced: fp32 [P] (only the bucket's indices are written).
 * nonfinite: optional device int32 [n_buckets]; each bucket's count of non-finite sums
 * is ADDED to its entry (zero it first). */
zero_status zero_reduce_scatter(const zero_layout *layout, int64_t bucket, const uint16_t *grads,
                                int64_t rank_stride, float *reduced, int32_t *nonfinite,
                                void *stream);

/* Shard update of shard `shard` (-1 = every shard), P1 Deepspeed ZeRO-1 update step:
 * the reduced fp32 sum is scaled by 1/(N * loss_scale), then AdamW updates the fp32
 * first and second moments and the fp32 master weights, then the fp16 parameters:
 *     g = s * fp32(1/(N L));  p = p * fp32(1 - lr wd)
 *     m = fp32(b1) m + fp32(1 - b1) g;  v = fp32(b2) v + fp32(1 - b2) (g g)
 *     p = p - fp32(lr / (1 - b1^t)) * (m / (sqrt(v) / fp32(sqrt(1 - b2^t)) + fp32(eps)))
 *     p16_out[i] = fp16_rne(p)
 * (scalars computed on the host in double, each rounded once to fp32).
 * reduced, master, m, v: fp32 [P]; p16_out: fp16 [P] (the full buffer for stages 0-2,
 * the shard buffer for stage 3); only the shard's indices are touched. */
zero_status zero_adamw_shard_step(const zero_layout *layout, int32_t shard, const float *reduced,
                                  float *master, float *m, float *v, uint16_t *p16_out,
                                  const zero_adamw_hparams *hp, void *stream);

/* All-gather of gather unit `unit` (-1 = all units): every shard's fp16 parameters of the
 * unit are written into the full flat buffer, p16_full[i] = p16_shard[i] for i in the
 * unit (P1 ZeRO-1 broadcast step; P2 section 2.5: the full parameter is the
 * concatenation of all ranks' partitions; P1 ZeRO-3: parameters are gathered layer by
 * layer for the forward and again for the backward pass).  Both fp16 [P]. */
zero_status zero_allgather(const zero_layout *layout, int64_t unit, const uint16_t *p16_shard,
                           uint16_t *p16_full, void *stream);

/* ZeRO-3's per-layer gather into a buffer of its own (P1 ZeRO-3: before a layer's
 * forward, and again before its backward, the layer's parameters are gathered from the
 * ranks that hold them, and released once the layer is done; P2 section 2.5).
 * dst[j] = p16_shard[lo + j] for j < hi - lo, where [lo, hi) is unit `unit`'s range:
 * dst receives the unit's full fp16 parameters contiguously, so a caller can keep only
 * a few layers materialised at a time (a ring of unit-sized buffers, the next layer's
 * gather overlapping the current layer's compute).  dst: device, 16-byte aligned,
 * >= hi - lo elements. */
zero_status zero_gather_unit(const zero_layout *layout, int64_t unit, const uint16_t *p16_shard,
                             uint16_t *dst, void *stream);

/* The same gather when every rank keeps only its own shard ([P1] "ZeRO-3" on N GPUs: a
 * layer's parameters are fetched from the ranks that hold them before its forward and
 * again before its backward).  rank_p16: host array of N device pointers (N <= 64), rank
 * k's buffer holding flat elements [k*S, (k+1)*S) of the fp16 parameters (its shard, as
 * zero_step_shard writes it for stage 3), each 16-byte aligned; they may point into this
 * GPU's memory or into other GPUs' memory mapped with zero_ipc_open (plain loads over
 * NVLink).  dst[j] = element unit_lo + j, j < unit_hi - unit_lo; dst 16-byte aligned.
 * Bit-identical to zero_gather_unit on the concatenated shards. */
zero_status zero_gather_unit_ranks(const zero_layout *layout, int64_t unit, const uint16_t *const *rank_p16,
                                   uint16_t *dst, void *stream);

/* One whole optimizer step of the layout's stage: the reduce-scatter of every bucket
 * fused with the shard update, each gradient and state byte crossing HBM once; the
 * reduced sums stay in registers.  Stages 0-2 write the fp16 parameters straight into
 * p16_full (the owner's slice of the replicated buffer: the broadcast is the write
 * itself; p16_shard may be NULL).  Stage 3 writes p16_shard, then runs the all-gather
 * of every unit into p16_full.  Results are bit-identical to zero_reduce_scatter +
 * zero_adamw_shard_step (+ zero_allgather).  nonfinite and events may be NULL. */
zero_status zero_step(const zero_layout *layout, const uint16_t *grads, int64_t rank_stride,
                      float *master, float *m, float *v, uint16_t *p16_shard, uint16_t *p16_full,
                      const zero_adamw_hparams *hp, int32_t *nonfinite,
                      const zero_step_events *events, void *stream);

/* The scalars of step hp->step for this layout's rank count (host only, no CUDA call);
 * hp as for zero_step. */
zero_status zero_step_scalars_fill(const zero_layout *layout, const zero_adamw_hparams *hp,
                                   zero_step_scalars *out);

/* zero_step with the step's scalars read from device memory when the kernels run, instead
 * of passed at launch: scalars_dev points to a zero_step_scalars in device memory (4-byte
 * aligned), typically filled by zero_step_scalars_fill and a copy.  Nothing in the launch
 * then depends on the step number or the hyper-parameters, so the call can be captured
 * once in a CUDA graph and the graph replayed every step, the caller updating
 * *scalars_dev before each replay (for instance with a captured cudaMemcpyAsync from a
 * page-locked host copy it rewrites with zero_step_scalars_fill once the previous replay
 * has finished).  For small models, whose step is a few tens of microseconds, that
 * removes the per-step launch work.  Make one ordinary call (or zero_step) on the layout
 * before capturing, so that the kernels are loaded.  Same results as zero_step with
 * the same scalars; the same kernels, the same automatic implementation choice.  The
 * pages have no counterpart. */
zero_status zero_step_device_scalars(const zero_layout *layout, const uint16_t *grads, int64_t rank_stride,
                                     float *master, float *m, float *v, uint16_t *p16_shard,
                                     uint16_t *p16_full, const zero_step_scalars *scalars_dev,
                                     int32_t *nonfinite, void *stream);

/* One bucket's share of zero_step: the fused reduce-scatter + update of bucket `bucket`
 * only, so that it can start as soon as that bucket's gradients exist (P1 DDP: the first
 * group of gradients computed starts its ring while the next group is still being
 * computed; P1 ZeRO-2: each bucket goes to its owner as soon as it is complete; P3 DDP:
 * buckets).  Running every bucket once, in any order, gives exactly zero_step's result.
 * Stage 3 writes p16_shard only: call zero_allgather after the last bucket. */
zero_status zero_step_bucket(const zero_layout *layout, int64_t bucket, const uint16_t *grads,
                             int64_t rank_stride, float *master, float *m, float *v, uint16_t *p16_shard,
                             uint16_t *p16_full, const zero_adamw_hparams *hp, int32_t *nonfinite,
                             void *stream);

/* zero_step overlapped with the backward pass that produces the gradients: for each
 * bucket b in bucket order (the order a backward pass completes them), `stream` waits
 * for ready_events[b] (a cudaEvent_t the caller records once bucket b's gradients are
 * written, typically on another stream), then runs bucket b's fused update.  Consecutive
 * buckets smaller than 2^24 elements share one launch, which waits for all of them,
 * until the launch holds at least 2^24 elements (many small buckets otherwise interleave
 * hundreds of short launches with the backward pass).  Stage 3 then runs the
 * all-gather.  ready_events: host array [n_buckets], none NULL.  As for any
 * cudaStreamWaitEvent, each wait takes the event's most recent record at the time of
 * this call: enqueue the producer's records first (the producer's work itself may still
 * be running).  Result identical to zero_step.
 *
 * Launch plan: the update shares the GPU with the backward pass, and whether and how to
 * split the SMs depends on the two workloads (and on the power budget they share).
 * Unless zero_set_max_ctas fixed a cap, the library chooses a plan by measurement: after
 * one untimed warm-up call it times whole calls (CUDA events on `stream`, from the first
 * wait to the last launch) under ZERO_OVERLAP_PLANS plans, round-robin, two calls each:
 * the update following the backward bucket by bucket with its grid capped at 1, 2/3,
 * 1/2 or 1/3 of the SMs, or deferred to one full-grid launch after the last bucket's
 * event (the back-to-back order, for workloads where sharing the GPU does not pay); it
 * then keeps the plan with the lowest mean for every later call.  It never waits for these
 * events: a call issued before the previous timed call has finished on the GPU is not
 * timed.  The plan never changes a result. */
zero_status zero_step_overlapped(const zero_layout *layout, void *const *ready_events,
                                 const uint16_t *grads, int64_t rank_stride, float *master, float *m,
                                 float *v, uint16_t *p16_shard, uint16_t *p16_full,
                                 const zero_adamw_hparams *hp, int32_t *nonfinite, void *stream);

/* The launch plan the overlapped steps settled on for this layout: -1 while the plans
 * are still being timed (or when zero_set_max_ctas fixed a cap), 0..3 = the update
 * following the backward with its grid capped at 1, 2/3, 1/2, 1/3 of the SMs, 4 = the
 * update deferred to one launch after the last bucket.  *mean_ms (optional, host array
 * of ZERO_OVERLAP_PLANS) receives each plan's mean timed call so far (0 where none).
 * Host only. */
#define ZERO_OVERLAP_PLANS 5
zero_status zero_overlap_plan(const zero_layout *layout, int32_t *plan, float *mean_ms);

/* zero_step_overlapped with one launch per `group` consecutive buckets (group >= 1; the
 * last group may be shorter; no other coalescing): `stream` waits for the ready events
 * of all the group's buckets, then runs their fused update as one kernel.  With many
 * small buckets (a bucket of 10^6 parameters is ~9 us of work at full bandwidth) this
 * trades a later start for fewer launches interleaved with the backward pass.  The grid
 * is chosen as for zero_step_overlapped.  Same results.  No counterpart on the pages
 * (their buckets are the launch unit). */
zero_status zero_step_overlapped_grouped(const zero_layout *layout, void *const *ready_events, int64_t group,
                                         const uint16_t *grads, int64_t rank_stride, float *master, float *m,
                                         float *v, uint16_t *p16_shard, uint16_t *p16_full,
                                         const zero_adamw_hparams *hp, int32_t *nonfinite, void *stream);

/* zero_step for gradients that live in HOST memory (page-locked), with the fp16
 * parameters returned to host memory: per bucket, the N gradient slices are copied to
 * the device staging buffer grads_dev on an internal copy stream, the bucket's fused
 * update runs on `stream` as soon as they land, and (stages 0-2) the bucket's new fp16
 * parameters are copied back to p16_host on a second internal stream, so transfers and
 * compute overlap bucket by bucket.  Stage 3 copies p16_full back after the gather.
 *   grads_host: [N][rank_stride] page-locked; grads_dev: device [N][rank_stride];
 *   p16_host: page-locked fp16 [P].  Completion: synchronise `stream`. */
zero_status zero_step_host(const zero_layout *layout, const uint16_t *grads_host,
                           uint16_t *grads_dev, int64_t rank_stride, float *master, float *m,
                           float *v, uint16_t *p16_shard, uint16_t *p16_full, uint16_t *p16_host,
                           const zero_adamw_hparams *hp, int32_t *nonfinite, void *stream);

/* The step for callers that cannot allocate device memory.  The pages have no
 * counterpart: this entry point exists for the library's users, not for the method.
 *
 * zero_step needs zero_layout_to_device, which obtains device memory with cudaMalloc for
 * the segment table and its tile index.  Callers whose device memory belongs to another
 * allocator (a framework's caching allocator or a fixed pool that has reserved the GPU),
 * whose loop cannot take the device-wide synchronisation an allocation may imply, or
 * that run where allocating is not allowed can call this instead: it computes exactly
 * what zero_step computes (register-streaming kernel, results bit-identical), with that
 * scratch held in a static device array of the library instead of allocated memory.
 *   - The layout does not need zero_layout_to_device.  Inputs and outputs are the
 *     caller's, as for zero_step.  Nothing is allocated and nothing is freed.
 *   - Limit: layouts of at most ZERO_NOALLOC_MAX_SEGMENTS segments (bucket x shard
 *     pieces); larger layouts return ZERO_ERR_INVALID before anything runs.  The array
 *     takes (ZERO_NOALLOC_MAX_SEGMENTS + 1) x 32 bytes = 256 KiB on every GPU that
 *     loads the library, until the process exits.
 *   - The first call on each device looks up the array's device address (which can load
 *     the library's device code onto that device) and keeps it; make that first call
 *     before any stream capture begins.  A cudaDeviceReset invalidates the kept address:
 *     do not call this entry point on a device after resetting it.
 *   - All calls on a device share the one array, and it keeps whatever the last call
 *     wrote.  Each call rewrites every row it reads (the rows are copied from the
 *     layout's host table, which waits for earlier work on `stream` to finish, and the
 *     tile index is rebuilt on the device), so no clearing is needed; but two calls
 *     whose work overlaps on the GPU (different streams, different layouts) race on
 *     the array and may compute garbage.  Serialise them.
 *   - nonfinite (optional) is added to, as in zero_step. */
#define ZERO_NOALLOC_MAX_SEGMENTS 8191
zero_status zero_step_noalloc(const zero_layout *layout, const uint16_t *grads, int64_t rank_stride,
                              float *master, float *m, float *v, uint16_t *p16_shard, uint16_t *p16_full,
                              const zero_adamw_hparams *hp, int32_t *nonfinite, void *stream);

/* One step under dynamic loss scaling (see zero_loss_scaler).  The gradients must carry
 * the scaler's current scale.  Runs the reduce-scatter of every bucket into `reduced`
 * (fp32 [P], caller's scratch) with per-bucket non-finite counts in `nonfinite` (device
 * int32 [n_buckets], required, zeroed here), copies the counts back and synchronises
 * `stream`; then, if every count is zero, applies the shard update with loss_scale =
 * scale and step = scaler->step + 1 (hp's loss_scale and step are ignored) and, for
 * stage 3, the all-gather; otherwise skips the update, leaving master, m, v and the fp16
 * parameters untouched.  Finally advances the scaler.  *applied = 1 if the update ran.
 * With the fp16 wire (zero_layout_desc.wire_fp16) a partial sum beyond 65504 overflows
 * and triggers a skip; with fp32 partials only non-finite inputs do. */
zero_status zero_step_dynamic(const zero_layout *layout, const uint16_t *grads, int64_t rank_stride,
                              float *reduced, float *master, float *m, float *v, uint16_t *p16_shard,
                              uint16_t *p16_full, const zero_adamw_hparams *hp, zero_loss_scaler *scaler,
                              int32_t *nonfinite, int32_t *applied, void *stream);

/* The same step as a two-phase commit: one fused pass (each gradient and state byte
 * crossing HBM once, as in zero_step) reads the optimizer state from the *_in buffers and
 * writes the updated state to the *_out buffers and the fp16 parameters to p16_out; the
 * per-bucket non-finite counts are copied back (the stream is synchronised) and decide:
 *   *applied = 1: every count is zero; the *_out buffers and p16_out hold the step (for
 *     stage 3, p16_out is the shard-written buffer and every unit has been gathered from
 *     it into p16_full).  The caller makes the out set its current state.
 *   *applied = 0: the *_out buffers and p16_out hold values of a discarded update; the
 *     *_in buffers, the caller's current fp16 parameters and p16_full are untouched.
 * The scaler advances as in zero_step_dynamic; loss_scale and step come from it.
 * Stage 0-2: p16_out is a full fp16 parameter buffer [P] (p16_full unused, may be NULL);
 * stage 3: p16_out [P] receives the owners' shards, p16_full [P] the gathered result.
 * Costs the fused step's bytes instead of the reduce-then-update pair of
 * zero_step_dynamic, for a second state set (12 bytes and 2 for fp16 per parameter).
 * No in buffer may overlap an out buffer (ZERO_ERR_INVALID).  Either implementation
 * (zero_set_impl).  nonfinite: device int32 [n_buckets],
 * required, zeroed here.  The pages name
 * no overflow handling; this is the two-phase form of the skip described above. */
zero_status zero_step_dynamic_commit(const zero_layout *layout, const uint16_t *grads, int64_t rank_stride,
                                     const float *master_in, const float *m_in, const float *v_in,
                                     float *master_out, float *m_out, float *v_out, uint16_t *p16_out,
                                     uint16_t *p16_full, const zero_adamw_hparams *hp,
                                     zero_loss_scaler *scaler, int32_t *nonfinite, int32_t *applied,
                                     void *stream);

/* ---- one GPU per rank (the step over NVLink peers) --------------------------------- */

/* zero_step with each rank's gradients in a buffer of its own: rank r's gradient of flat
 * element i is rank_grads[r][i] (host array of N device pointers, each 16-byte aligned,
 * each >= P elements; they may point into this GPU's memory or into other GPUs' memory
 * mapped with zero_ipc_open).  Uses the bulk-copy pipeline; N <= 64.  Same result as
 * zero_step on the same values. */
zero_status zero_step_ranks(const zero_layout *layout, const uint16_t *const *rank_grads, float *master,
                            float *m, float *v, uint16_t *p16_shard, uint16_t *p16_full,
                            const zero_adamw_hparams *hp, int32_t *nonfinite, void *stream);

/* The fused reduce-scatter + update of shard `shard` alone, with that shard's optimizer
 * state only: what the GPU owning shard k runs when every rank sits on its own GPU (P1
 * Deepspeed ZeRO-1: each GPU updates the optimizer state of its own part).  The shard's
 * N gradient slices are read from rank_grads (peers' buffers mapped with zero_ipc_open,
 * this GPU's own for its rank) and folded in the ring order k, k+1, ..., k+N-1, so the
 * result equals the single-GPU simulation bit for bit.
 *   master_k, m_k, v_k: fp32 [S], element i of the flat buffer at [i - kS];
 *   p16_out: fp16, full [P] (stages 0-2: element i at [i]) or, for stage 3, the shard's
 *   own [S] (element i at [i - kS]).  Requires S % 8 == 0 and N <= 64.
 * The caller makes sure the peers' gradients are complete before the call (a host
 * barrier between ranks): the kernel reads peer memory but never waits on another GPU. */
zero_status zero_step_shard(const zero_layout *layout, int32_t shard, const uint16_t *const *rank_grads,
                            float *master_k, float *m_k, float *v_k, uint16_t *p16_out,
                            const zero_adamw_hparams *hp, int32_t *nonfinite, void *stream);

/* zero_step_shard as the first phase of a two-phase commit under dynamic loss scaling
 * (see zero_step_dynamic_commit): the shard's state is read from *_in and the step
 * written to *_out (each [S], no in buffer overlapping an out buffer) and the fp16
 * parameters to p16_out (laid out as for zero_step_shard; the caller keeps a second
 * parameter buffer for it); loss_scale and step come from the scaler, which is NOT
 * advanced.  Clears and fills nonfinite (device int32 [n_buckets], required), synchronises
 * the stream and stores the shard's count of non-finite reduced gradients in
 * *nonfinite_total (host).  The step must be kept or dropped on every rank alike: the
 * caller sums the ranks' counts (one all-reduce of an integer), then advances every
 * rank's scaler with zero_loss_scaler_advance and, if the sum is zero, makes the out
 * buffers current everywhere.  N <= 64, S % 8 == 0. */
zero_status zero_step_shard_commit(const zero_layout *layout, int32_t shard, const uint16_t *const *rank_grads,
                                   const float *master_in, const float *m_in, const float *v_in,
                                   float *master_out, float *m_out, float *v_out, uint16_t *p16_out,
                                   const zero_adamw_hparams *hp, const zero_loss_scaler *scaler,
                                   int32_t *nonfinite, int64_t *nonfinite_total, void *stream);

/* Advance the scaler after a step: applied = 1 counts towards the growth window, 0 backs
 * the scale off (the rules of zero_loss_scaler).  For callers that decide the step
 * themselves (zero_step_shard_commit on several ranks). */
zero_status zero_loss_scaler_advance(zero_loss_scaler *scaler, int32_t applied);

/* dst[i] = src[i] for i in shard `shard`'s range [kS, (k+1)S): the all-gather of the
 * fp16 parameters when src is the owning GPU's full buffer, mapped with zero_ipc_open
 * (P1 ZeRO-1 broadcast step).  Both flat-indexed fp16 [P], 16-byte aligned. */
zero_status zero_copy_shard(const zero_layout *layout, int32_t shard, const uint16_t *src, uint16_t *dst,
                            void *stream);

/* CUDA IPC.  zero_ipc_get_handle exports the allocation dev_ptr lies in as a 64-byte
 * handle plus dev_ptr's byte offset within it (pointers from a caching allocator lie
 * inside larger allocations).  zero_ipc_open maps such a handle into this process (peer
 * access enabled) and returns the address of the same byte; zero_ipc_close unmaps it,
 * given the same offset. */
zero_status zero_ipc_get_handle(const void *dev_ptr, void *handle_out, int64_t *offset_out);
zero_status zero_ipc_open(const void *handle, int64_t offset, void **dev_ptr_out);
zero_status zero_ipc_close(void *dev_ptr, int64_t offset);

/* Select the implementation of the fused step and of zero_reduce_scatter (and the
 * reduce pass of zero_step_dynamic): 0 = automatic (for the fused step the bulk-copy
 * pipeline for N <= 16, where it has an instance per rank count, register streaming
 * above, where it runs at the copy bandwidth; for the reduce-scatter alone the pipeline
 * for 5 <= N <= 16 and register streaming otherwise, as measured), 1 = register streaming (vectorised 16-byte loads held in
 * registers; any N), 2 = bulk-copy pipeline (cp.async.bulk into a shared-memory ring,
 * warp-specialised; one runtime-N instance serves 17 <= N <= 64; register streaming
 * above).  The per-rank-pointer calls (zero_step_ranks, zero_step_shard*) always use the
 * pipeline.  Results are bit-identical. */
zero_status zero_set_impl(zero_layout *layout, int32_t impl);

/* Cap on the number of CTAs of the tile-walking kernels (the fused step in both
 * implementations, and the reduce-scatter): 0 (the default) = as many as the GPU holds
 * (one per SM for the pipeline), k > 0 = at most k.  Every grid size gives bit-identical
 * results: tiles are dealt to CTAs by a fixed stride.  A capped step leaves the other
 * SMs to concurrent work (a backward pass whose gradients the step consumes bucket by
 * bucket, as in [P1] "DDP": the first finished group is synchronised while the next is
 * computed); it is slower alone, since each SM moves at most ~60 GB/s through the
 * step's arithmetic.  A cap set here also replaces the overlapped steps' own choice
 * (see zero_step_overlapped).  Negative k: ZERO_ERR_INVALID.  No counterpart on the
 * pages. */
zero_status zero_set_max_ctas(zero_layout *layout, int32_t max_ctas);

/* Grid of the all-gather copies (zero_allgather, zero_gather_unit, zero_gather_unit_ranks
 * and the gather inside the stage-3 steps): 0 (the default) = a grid of short blocks over
 * the whole range, the fastest when a gather has the GPU to itself; k > 0 = k persistent
 * CTAs, so that a gather occupies at most k SMs and can run beside a layer's compute that
 * leaves those SMs free (P1 ZeRO-3: the next layer's parameters are gathered while the
 * current layer computes).  The copies of this GPU's memory then move 48 KB chunks
 * global -> shared -> global with bulk copies (~144 KB of loads in flight; bounded waits
 * report ZERO_ERR_TIMEOUT through zero_get_error); the gather from the ranks' shards
 * (zero_gather_unit_ranks, possibly peers' memory) deals its blocks of 16-byte loads to
 * the k CTAs by a grid stride.  Results are identical for every k.  Negative k:
 * ZERO_ERR_INVALID.  No counterpart on the pages. */
zero_status zero_set_gather_ctas(zero_layout *layout, int32_t max_ctas);

/* Test hook of the bulk-copy pipeline's bounded waits: every in-kernel wait gives up
 * after wait_limit_ns nanoseconds (default 2e9) and records ZERO_ERR_TIMEOUT.  With
 * skip_first_fill = 1 the pipeline never posts its first chunk, so the consumers' wait
 * for it expires: the kernel then drains its own copies and returns, and
 * zero_get_error() reports ZERO_ERR_TIMEOUT (the GPU context stays usable).  Set
 * skip_first_fill back to 0 for normal use.  Requires an uploaded layout. */
zero_status zero_debug_set_wait(zero_layout *layout, int64_t wait_limit_ns, int32_t skip_first_fill);

/* Synchronise `stream`, read and clear the layout's device error word. */
zero_status zero_get_error(const zero_layout *layout, void *stream);

const char *zero_status_string(zero_status status);

#ifdef __cplusplus
}
#endif

#endif /* ZERO_H */
