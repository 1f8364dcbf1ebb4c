/*
 * oracle/oracle.c -- the CPU oracle's arithmetic.  TEST INFRASTRUCTURE ONLY.
 *
 * Only tests/, __graft_entry__.smoke() and bench.py's CPU-baseline / reference arm
 * may load this library.  It shares no code with the CUDA library: its own fp16
 * conversions, its own ring, its own optimizer update.  Plain single-threaded C,
 * compiled with -O2 -ffp-contract=off (no FMA contraction, no fast-math): every
 * float operation below is one IEEE-754 binary32 operation, rounded to nearest even.
 *
 * What it follows (page = source address of the text, then its section):
 *  - ring scatter-reduce and all-gather: en.pswp.cn/web/84187 "DDP" (the three-GPU
 *    a/b/c Ring-AllReduce walk-through) and rkmt.cn/news/44736 "DDP" (two phases:
 *    scatter-reduce passes and adds, all-gather passes and overwrites);
 *  - the shard update order: rkmt.cn/news/44736 "Deepspeed ZeRO-1", update step
 *    (fp16 gradient to fp32 without storing it, scale, update the fp32 first and
 *    second moments, update the fp32 master weights, update the fp16 parameters);
 *  - the Adam state per parameter (one first and one second moment, fp32 master):
 *    rkmt.cn/news/44736 preamble and "Deepspeed ZeRO" memory paragraph.
 * The AdamW formula itself is not printed on the pages; the oracle uses Adam's
 * bias-corrected moments with decoupled weight decay, in the operation order of
 * PyTorch's AdamW (weight decay first; denominator sqrt(v)/sqrt(1-beta2^t) + eps).
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

#define ORACLE_API __attribute__((visibility("default")))

/* ------------------------------------------------------------------ fp16
 * IEEE 754 binary16: 1 sign bit, 5 exponent bits (bias 15), 10 fraction bits.
 * Decoding is exact in double; encoding picks the nearest representable half by
 * working out the spacing of halfs at the value's magnitude and rounding the
 * quotient with rint() (round half to even in the default rounding mode).
 */
ORACLE_API float oracle_half_to_float(uint16_t h)
{
    const int sign = (h >> 15) & 1;
    const int e = (h >> 10) & 0x1f;
    const int f = h & 0x3ff;
    double mag;
    if (e == 0x1f)
        mag = f ? NAN : INFINITY;
    else if (e == 0)
        mag = ldexp((double)f, -24);                 /* subnormal: f * 2^-24 */
    else
        mag = ldexp((double)(1024 + f), e - 25);     /* (1 + f/1024) * 2^(e-15) */
    return (float)(sign ? -mag : mag);
}

ORACLE_API uint16_t oracle_double_to_half(double x)
{
    const uint16_t sign = signbit(x) ? 0x8000 : 0;
    const double a = fabs(x);
    if (isnan(x)) return (uint16_t)(sign | 0x7e00);
    if (a == 0.0) return sign;
    /* spacing of halfs at |x|: 2^-24 below 2^-14, else 2^(floor(log2|x|) - 10) */
    int ex;
    frexp(a, &ex);                                    /* a = frac * 2^ex, frac in [0.5,1) */
    const int e = ex - 1;                             /* floor(log2 a) */
    const double ulp = e < -14 ? ldexp(1.0, -24) : ldexp(1.0, e - 10);
    const double q = rint(a / ulp);                   /* exact division by a power of 2 */
    const double r = q * ulp;
    if (r >= 65536.0 || isinf(a)) return (uint16_t)(sign | 0x7c00);   /* overflow: inf */
    /* re-encode the (exactly representable) rounded magnitude r */
    if (r < ldexp(1.0, -14))
        return (uint16_t)(sign | (uint16_t)(r / ldexp(1.0, -24)));   /* subnormal */
    frexp(r, &ex);
    const int er = ex - 1;
    const uint16_t frac = (uint16_t)(r / ldexp(1.0, er - 10) - 1024.0);
    return (uint16_t)(sign | (uint16_t)((er + 15) << 10) | frac);
}

/* fp32 -> fp16: the fp32 value is exact in double, so one rounding, as above. */
ORACLE_API uint16_t oracle_float_to_half(float x)
{
    return oracle_double_to_half((double)x);
}

/* One hop of the fp16 wire: the receiver adds its own fp16 gradient to the fp16 partial
 * it received and sends the sum on as fp16.  Two fp16 values have at most 11 significant
 * bits each within exponents -24..15, so their sum is exact in double; rounding it once
 * gives the correctly rounded fp16 sum. */
static float wire16_add(float incoming, float own)
{
    return oracle_half_to_float(oracle_double_to_half((double)incoming + (double)own));
}

ORACLE_API void oracle_halfs_to_floats(const uint16_t *in, float *out, int64_t n)
{
    for (int64_t i = 0; i < n; ++i) out[i] = oracle_half_to_float(in[i]);
}

ORACLE_API void oracle_floats_to_halfs(const float *in, uint16_t *out, int64_t n)
{
    for (int64_t i = 0; i < n; ++i) out[i] = oracle_float_to_half(in[i]);
}

/* ------------------------------------------------------------------ ring
 * Ranks are numbered 0..N-1 around the ring; rank r sends to rank (r+1) mod N.
 * Chunk k of a bucket [blo, bhi) is the part of it inside shard k, [kS, (k+1)S).
 */
static int64_t imod(int64_t a, int64_t n) { int64_t r = a % n; return r < 0 ? r + n : r; }

static void chunk_range(int64_t k, int64_t shard, int64_t lo, int64_t hi, int64_t *clo, int64_t *chi)
{
    int64_t a = k * shard, b = (k + 1) * shard;
    if (a < lo) a = lo;
    if (b > hi) b = hi;
    if (b < a) b = a;
    *clo = a;
    *chi = b;
}

/*
 * Scatter-reduce of one bucket, simulated hop by hop.
 *   grads    fp16 bits, rank r's copy at grads[r * rank_stride + i]
 *   work     n_ranks * (bhi - blo) floats: rank r's running partials of the bucket
 *   hops     how many hops to run (N-1 for the full phase; fewer to inspect a prefix)
 *   reduced  if not NULL, receives the completed sum of every chunk (fp32, flat index)
 *   log      if not NULL, 4 int64 per send: hop, sender, receiver, chunk
 *   sent, recv  if not NULL, per-rank element counters (incremented)
 * Each rank first converts its own fp16 gradients to fp32 (exact).  At hop h rank r
 * passes its running partial of chunk (r - h) mod N to rank r+1, and the receiver adds
 * its own partial to it (page 3's trace: a0 goes to GPU1, which forms a0+a1, ...).
 * After N-1 hops chunk k's full sum, folded in the order k, k+1, ..., k+N-1, sits at
 * rank (k - 1) mod N.  Returns the number of log records written.
 *   wire16   0: partials travel as fp32 (every add one fp32 rounding); 1: partials travel
 *            as fp16, every hop's sum rounded to fp16 (rkmt.cn/news/44736 "Deepspeed
 *            ZeRO-1": each GPU ends up with its part's gradient mean in fp16).
 */
ORACLE_API int64_t oracle_ring_reduce_scatter(const uint16_t *grads, int32_t n_ranks,
                                              int64_t rank_stride, int64_t shard,
                                              int64_t blo, int64_t bhi, int32_t hops, int32_t wire16,
                                              float *work, float *reduced, int64_t *log,
                                              int64_t *sent, int64_t *recv)
{
    const int64_t n = bhi - blo;
    int64_t nlog = 0;
    for (int32_t r = 0; r < n_ranks; ++r)
        for (int64_t i = 0; i < n; ++i)
            work[r * n + i] = oracle_half_to_float(grads[r * rank_stride + blo + i]);

    for (int32_t h = 0; h < hops; ++h) {
        for (int32_t r = 0; r < n_ranks; ++r) {
            const int64_t k = imod(r - h, n_ranks);
            const int32_t dst = (int32_t)imod(r + 1, n_ranks);
            int64_t clo, chi;
            chunk_range(k, shard, blo, bhi, &clo, &chi);
            for (int64_t i = clo; i < chi; ++i) {
                const float incoming = work[r * n + (i - blo)];
                const float own = work[dst * n + (i - blo)];
                work[dst * n + (i - blo)] = wire16 ? wire16_add(incoming, own) : incoming + own;
            }
            if (log) {
                log[4 * nlog + 0] = h;
                log[4 * nlog + 1] = r;
                log[4 * nlog + 2] = dst;
                log[4 * nlog + 3] = k;
                ++nlog;
            }
            if (sent) sent[r] += chi - clo;
            if (recv) recv[dst] += chi - clo;
        }
    }
    if (reduced) {
        for (int64_t k = 0; k < n_ranks; ++k) {
            const int64_t holder = imod(k - 1, n_ranks);
            int64_t clo, chi;
            chunk_range(k, shard, blo, bhi, &clo, &chi);
            for (int64_t i = clo; i < chi; ++i) reduced[i] = work[holder * n + (i - blo)];
        }
    }
    return nlog;
}

/*
 * All-gather of the range [lo, hi) over N replicas, simulated hop by hop.
 *   rep      n_ranks replicas of elem_size-byte elements, replica r at rep + r*rep_stride elements
 * Before the call, chunk k is valid only in the replica of rank (k - 1) mod N (where
 * the scatter-reduce completed it and where its shard was updated).  At hop h rank r
 * passes chunk (r + 1 - h) mod N to rank r+1, which overwrites its copy (page 1: in
 * the all-gather phase values are passed on and directly overwrite).  After N-1 hops
 * every replica holds every chunk.  Returns the number of log records written.
 */
ORACLE_API int64_t oracle_ring_allgather(void *rep, int32_t elem_size, int32_t n_ranks,
                                         int64_t rep_stride, int64_t shard, int64_t lo, int64_t hi,
                                         int64_t *log, int64_t *sent, int64_t *recv)
{
    unsigned char *base = (unsigned char *)rep;
    int64_t nlog = 0;
    for (int32_t h = 0; h < n_ranks - 1; ++h) {
        for (int32_t r = 0; r < n_ranks; ++r) {
            const int64_t k = imod(r + 1 - h, n_ranks);
            const int32_t dst = (int32_t)imod(r + 1, n_ranks);
            int64_t clo, chi;
            chunk_range(k, shard, lo, hi, &clo, &chi);
            if (chi > clo)
                memcpy(base + ((int64_t)dst * rep_stride + clo) * elem_size,
                       base + ((int64_t)r * rep_stride + clo) * elem_size,
                       (size_t)((chi - clo) * elem_size));
            if (log) {
                log[4 * nlog + 0] = h;
                log[4 * nlog + 1] = r;
                log[4 * nlog + 2] = dst;
                log[4 * nlog + 3] = k;
                ++nlog;
            }
            if (sent) sent[r] += chi - clo;
            if (recv) recv[dst] += chi - clo;
        }
    }
    return nlog;
}

/* ------------------------------------------------------------------ update
 * Scalars of step t, each computed in double from the hyper-parameters and rounded
 * once to fp32:
 *   s[0] inv_scale = 1/(N*L)      (mean over N ranks of loss-scaled gradients)
 *   s[1] decay     = 1 - lr*wd    (decoupled weight decay)
 *   s[2] beta1, s[3] 1-beta1, s[4] beta2, s[5] 1-beta2
 *   s[6] step_size = lr / (1 - beta1^t)
 *   s[7] sqrt_bc2  = sqrt(1 - beta2^t)
 *   s[8] eps
 */
ORACLE_API void oracle_adamw_scalars(float *s, int32_t n_ranks, double loss_scale, double lr,
                                     double beta1, double beta2, double eps, double weight_decay,
                                     int64_t t)
{
    s[0] = (float)(1.0 / ((double)n_ranks * loss_scale));
    s[1] = (float)(1.0 - lr * weight_decay);
    s[2] = (float)beta1;
    s[3] = (float)(1.0 - beta1);
    s[4] = (float)beta2;
    s[5] = (float)(1.0 - beta2);
    s[6] = (float)(lr / (1.0 - pow(beta1, (double)t)));
    s[7] = (float)sqrt(1.0 - pow(beta2, (double)t));
    s[8] = (float)eps;
}

/*
 * One element of the shard update, in the pages' order:
 *   fp16 -> fp32 happened in the ring; sum s is scaled: g = s * inv_scale
 *   p = p * decay                           (decoupled weight decay)
 *   m = beta1*m + (1-beta1)*g               (first moment)
 *   v = beta2*v + (1-beta2)*(g*g)           (second moment)
 *   p = p - step_size * (m / (sqrt(v)/sqrt_bc2 + eps))   (fp32 master weight)
 *   p16 = fp16(p)                           (fp16 parameter)
 */
static void adamw_one(float sum, const float *s, float *p, float *m, float *v, uint16_t *p16)
{
    const float g = sum * s[0];
    float pp = *p * s[1];
    const float mm = *m * s[2] + g * s[3];
    const float gg = g * g;
    const float vv = *v * s[4] + gg * s[5];
    const float root = sqrtf(vv);
    const float denom = root / s[7] + s[8];
    const float ratio = mm / denom;
    pp = pp - s[6] * ratio;
    *p = pp;
    *m = mm;
    *v = vv;
    *p16 = oracle_float_to_half(pp);
}

/* The update over elements [lo, hi) of flat buffers; p16 receives the fp16 params. */
ORACLE_API void oracle_adamw(int64_t lo, int64_t hi, const float *reduced, float *master,
                             float *m, float *v, uint16_t *p16, const float *s)
{
    for (int64_t i = lo; i < hi; ++i)
        adamw_one(reduced[i], s, &master[i], &m[i], &v[i], &p16[i]);
}

/* Count of non-finite values among reduced[lo, hi). */
ORACLE_API int64_t oracle_count_nonfinite(const float *reduced, int64_t lo, int64_t hi)
{
    int64_t c = 0;
    for (int64_t i = lo; i < hi; ++i)
        if (!isfinite(reduced[i])) ++c;
    return c;
}

/*
 * The same computation for a sample of single elements (checks at full size, where
 * whole buffers would not fit the oracle's time budget).  Element j lies in shard
 * shard_of[j]; its gradients on the N ranks are g[j*N + r].  The ring carries the
 * element's partial from rank k = shard_of[j] around the ring, each rank adding its
 * own value, exactly as the bucket simulation does for the element's chunk.  Then
 * `steps` updates with the scalars of steps 1..steps (scalars[t-1][9]); the gradients
 * are the same at every step.  reduced[j] receives the ring sum.
 */
ORACLE_API void oracle_sampled(int64_t n, int32_t n_ranks, const uint16_t *g, const int64_t *shard_of,
                               int32_t wire16, int32_t steps, const float *scalars, float *reduced,
                               float *master, float *m, float *v, uint16_t *p16)
{
    for (int64_t j = 0; j < n; ++j) {
        const int64_t k = shard_of[j];
        float partial = oracle_half_to_float(g[j * n_ranks + k]);      /* starts at rank k */
        for (int32_t h = 0; h < n_ranks - 1; ++h) {
            const int64_t receiver = imod(k + h + 1, n_ranks);
            const float own = oracle_half_to_float(g[j * n_ranks + receiver]);
            partial = wire16 ? wire16_add(partial, own) : partial + own;
        }
        reduced[j] = partial;
        for (int32_t t = 0; t < steps; ++t)
            adamw_one(partial, scalars + 9 * t, &master[j], &m[j], &v[j], &p16[j]);
    }
}
