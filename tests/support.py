"""Helpers shared by the GPU parity tests: seeded inputs for both sides, the oracle's
answers, and the comparison rules.

Both sides get their inputs from seeded_inputs (host fill for the oracle, device fill
for the CUDA path; the two fills are checked bit-identical in test_inputs_gen.py).
Nothing the CUDA path computes ever feeds the oracle.

Comparison bar: ring sums bit-exact; fp32 master / moments within 1e-6 relative;
fp16 parameters within 1 ulp.  The arithmetic on both sides is the same sequence of
correctly rounded IEEE operations, so bit-exact agreement is also checked separately.
"""
import numpy as np

import oracle
import seeded_inputs as si
from oracle.layout import make_layout

F32_REL = 1e-6
F16_ULPS = 1


def oracle_layout(wl):
    return make_layout(list(wl.tensors), wl.n_ranks, wl.bucket_elems, wl.pad_align, list(wl.units))


def hyper(wl):
    return oracle.Hyper(wl.lr, wl.beta1, wl.beta2, wl.eps, wl.weight_decay, wl.loss_scale)


def host_inputs(wl, P):
    """grads uint16 [N, P]; master, m, v float32 [P] (zero tail padding)."""
    psi = wl.psi
    g = si.fill_grads(wl.n_ranks, P, psi, wl.seed, wl.grad_sigma, wl.loss_scale, wl.heavy_frac, wl.heavy_mult)
    master = si.fill_f32(P, psi, wl.seed, si.STREAM_MASTER, wl.master_sigma)
    m = si.fill_f32(P, psi, wl.seed, si.STREAM_M, wl.m_sigma) if wl.m_sigma else np.zeros(P, np.float32)
    v = si.fill_f32(P, psi, wl.seed, si.STREAM_V, wl.v_sigma, True) if wl.v_sigma else np.zeros(P, np.float32)
    return g, master, m, v


def device_inputs(wl, P, rank_stride=None):
    """The same inputs generated directly in device memory (torch tensors).  The rank
    stride defaults to P rounded up to a multiple of 8 (the ABI's 16-byte rule)."""
    import torch
    stride = rank_stride or (P + 7) // 8 * 8
    psi = wl.psi
    g = torch.empty((wl.n_ranks, stride), dtype=torch.int16, device="cuda")
    si.fill_grads_cuda(g, psi, wl.seed, wl.grad_sigma, wl.loss_scale, wl.heavy_frac, wl.heavy_mult)
    master = torch.empty(P, dtype=torch.float32, device="cuda")
    si.fill_f32_cuda(master, psi, wl.seed, si.STREAM_MASTER, wl.master_sigma)
    m = torch.zeros(P, dtype=torch.float32, device="cuda")
    v = torch.zeros(P, dtype=torch.float32, device="cuda")
    if wl.m_sigma:
        si.fill_f32_cuda(m, psi, wl.seed, si.STREAM_M, wl.m_sigma)
    if wl.v_sigma:
        si.fill_f32_cuda(v, psi, wl.seed, si.STREAM_V, wl.v_sigma, absval=True)
    return g, master, m, v


def sampled_oracle(wl, lay, idx, steps):
    """Oracle values at flat indices idx after `steps` steps (per-element path)."""
    psi = wl.psi
    g = si.gather_grads(idx, wl.n_ranks, psi, wl.seed, wl.grad_sigma, wl.loss_scale, wl.heavy_frac,
                        wl.heavy_mult)
    master = si.gather_f32(idx, psi, wl.seed, si.STREAM_MASTER, wl.master_sigma)
    m = si.gather_f32(idx, psi, wl.seed, si.STREAM_M, wl.m_sigma) if wl.m_sigma else np.zeros(len(idx), np.float32)
    v = (si.gather_f32(idx, psi, wl.seed, si.STREAM_V, wl.v_sigma, True) if wl.v_sigma
         else np.zeros(len(idx), np.float32))
    sc = np.stack([oracle.adamw_scalars(wl.n_ranks, hyper(wl), t) for t in range(1, steps + 1)])
    reduced, p16 = oracle.sampled(g, idx // lay.shard, steps, sc, master, m, v)
    return reduced, master, m, v, p16


def sample_indices(lay, n_random=16384, seed=0):
    """Random indices plus every segment, shard, bucket and unit edge, and the tail."""
    P = lay.padded
    rng = np.random.default_rng(seed)
    pts = [rng.integers(0, P, n_random)]
    edges = []
    for _, _, lo, hi in lay.segments:
        edges += [lo, lo + 1, lo + 7, lo + 8, hi - 1, hi - 2, hi - 8, hi - 9]
    for lo, hi in lay.units:
        edges += [lo, lo + 1, hi - 1]
    edges += [lay.psi - 1, lay.psi, P - 1, 0]
    pts.append(np.array(edges, dtype=np.int64))
    idx = np.unique(np.concatenate(pts))
    return idx[(idx >= 0) & (idx < P)]


def f16_ordered(bits):
    """Map fp16 bit patterns to integers that preserve numeric order (ulp distance)."""
    b = bits.astype(np.int32)
    return np.where(b & 0x8000, -(b & 0x7FFF), b)


def assert_f32_close(got, want, what, rel=F32_REL):
    got = np.asarray(got, np.float32)
    want = np.asarray(want, np.float32)
    same = (got.view(np.uint32) == want.view(np.uint32)) | (np.isnan(got) & np.isnan(want))
    bad = ~same & ~(np.abs(got.astype(np.float64) - want) <= rel * np.abs(want.astype(np.float64)))
    assert not bad.any(), f"{what}: {bad.sum()} elements beyond {rel} relative, first at {np.flatnonzero(bad)[:5]}"


def f16_isnan(bits):
    return ((bits & 0x7C00) == 0x7C00) & ((bits & 0x03FF) != 0)


def assert_f16_ulp(got, want, what, ulps=F16_ULPS):
    """Within `ulps` units in the last place; any NaN matches any NaN (the payload
    of a NaN carries no value: CUDA's conversion writes 0x7FFF, the oracle 0x7E00)."""
    got = np.asarray(got, np.uint16)
    want = np.asarray(want, np.uint16)
    nan_g, nan_w = f16_isnan(got), f16_isnan(want)
    assert np.array_equal(nan_g, nan_w), f"{what}: NaN positions differ"
    d = np.abs(f16_ordered(got[~nan_g]) - f16_ordered(want[~nan_w]))
    assert d.max(initial=0) <= ulps, f"{what}: max {d.max()} ulp"


def assert_bits_equal(got, want, what, any_nan=False):
    """Bit for bit.  any_nan: a NaN matches any NaN (float32, or fp16 bits as uint16) —
    IEEE 754 leaves the payload of an invalid operation's NaN open: x86 gives 0xFFC00000
    for 0/0, CUDA 0x7FFFFFFF — while NaN positions must still agree."""
    got = np.ascontiguousarray(got)
    want = np.ascontiguousarray(want)
    diff = (got.view(np.uint8).reshape(got.size, -1) != want.view(np.uint8).reshape(want.size, -1)).any(axis=1)
    if any_nan:
        isnan = f16_isnan if got.dtype == np.uint16 else np.isnan
        nan_g, nan_w = isnan(got).reshape(-1), isnan(want).reshape(-1)
        assert np.array_equal(nan_g, nan_w), f"{what}: NaN positions differ"
        diff &= ~(nan_g & nan_w)
    n = int(diff.sum())
    assert n == 0, f"{what}: {n} elements differ bitwise"


def oracle_run(wl, steps=None):
    """The oracle's result after `steps` (default: the workload's) optimizer steps on the
    workload's seeded inputs, and the oracle's layout."""
    lay = oracle_layout(wl)
    g, master, m, v = host_inputs(wl, lay.padded)
    return oracle.run_steps(lay, wl.stage, g, master, m, v, hyper(wl), steps or wl.steps), lay


def to_np(t):
    """A device tensor as a host array; int16 tensors (fp16 bit patterns) as uint16."""
    a = t.cpu().numpy()
    return a.view(np.uint16) if a.dtype == np.int16 else a


def assert_state_matches_oracle(wl, got, ref, what=""):
    """got: dict with device tensors master, m, v, p16_full (and p16_shard for stage 3).
    Within the parity tolerance first (fp32 1e-6 relative, fp16 1 ulp), then bit for bit:
    both sides run the same sequence of correctly rounded operations."""
    S_f32 = (("master", ref.master), ("m", ref.m), ("v", ref.v))
    for name, want in S_f32:
        assert_f32_close(to_np(got[name]), want, what + name)
    f16 = [("p16_full", ref.p16_full)] + ([("p16_shard", ref.p16_shard)] if wl.stage == 3 else [])
    for name, want in f16:
        assert_f16_ulp(to_np(got[name]), want, what + name)
    for name, want in S_f32 + tuple(f16):
        assert_bits_equal(to_np(got[name]), want, what + name + " (bits)")


# ---------------------------------------------------------------- guard regions
# compute-sanitizer is not available to these tests, so writes past a buffer are caught
# the old way: every output buffer sits between two guard regions of a fixed byte
# pattern, and the guards are compared after each step.

GUARD_BYTES = 4096          # a multiple of 16, so the guarded buffer keeps 16-byte alignment
GUARD_BYTE = 0x5A


class Guarded:
    """A device tensor of `n` elements with a guard region before and after it."""

    def __init__(self, n, dtype, fill=None):
        import torch
        item = torch.empty((), dtype=dtype).element_size()
        self.g = GUARD_BYTES // item
        self.raw = torch.empty(n + 2 * self.g, dtype=dtype, device="cuda")
        self.raw.view(torch.uint8).fill_(GUARD_BYTE)
        self.t = self.raw[self.g:self.g + n]
        if fill is not None:
            self.t.copy_(fill)

    def intact(self):
        import torch
        b = self.raw.view(torch.uint8)
        return bool((b[:GUARD_BYTES] == GUARD_BYTE).all()) and bool((b[-GUARD_BYTES:] == GUARD_BYTE).all())


def guard_outputs(bufs, names=("master", "m", "v", "p16_shard", "p16_full", "nonfinite")):
    """Move the named tensors of a buffer dict into guarded allocations (same values);
    returns the guards."""
    guards = {}
    for k in names:
        if bufs.get(k) is None:
            continue
        gd = Guarded(bufs[k].numel(), bufs[k].dtype, fill=bufs[k])
        bufs[k] = gd.t
        guards[k] = gd
    return guards


def assert_guards_intact(guards, what=""):
    import torch
    torch.cuda.synchronize()
    broken = [k for k, gd in guards.items() if not gd.intact()]
    assert not broken, f"{what}: guard regions overwritten around {broken}"
