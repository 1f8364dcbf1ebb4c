"""The allocation-free entry point, zero_step_noalloc, against zero_step and the oracle.

Some callers cannot let a library allocate device memory (their GPU memory belongs to
another allocator or a reserved pool, or they cannot take the synchronisation an
allocation may cause); zero_step_noalloc serves them by keeping the step's scratch (the
segment table and its tile index) in a static device array.  These tests call it through
the C ABI on a layout that was never uploaded (so no library allocation exists at all)
and check its outputs against zero_step's, within the tolerance of the other parity
tests and then bit for bit (both kernels follow the same rounded operations), on two
calls in a row (the second call runs on the array the first one left), and the final
state against the oracle's two steps.

This file is collected last on purpose: if it fails, every other test has already run.
"""
import numpy as np
import pytest

from seeded_inputs.workloads import reduced_workloads
import zero_sharded_optimizer_ring_b200 as zs
from zero_sharded_optimizer_ring_b200 import _abi
import support as S

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


def _hp(wl, t):
    return zs.AdamW(wl.lr, wl.beta1, wl.beta2, wl.eps, wl.weight_decay, wl.loss_scale, t)


def _bufs(P, wl):
    g, master, m, v = S.device_inputs(wl, P)
    return dict(g=g, master=master, m=m, v=v,
                p16_shard=torch.zeros(P, dtype=torch.int16, device="cuda"),
                p16_full=torch.zeros(P, dtype=torch.int16, device="cuda"),
                nonfinite=torch.zeros(64, dtype=torch.int32, device="cuda"))


def _np(t):
    a = t.cpu().numpy()
    return a.view(np.uint16) if a.dtype == np.int16 else a


@pytest.mark.parametrize("key", ["flat1p3b_n4_zero1", "llama3b_n8_zero3", "ragged2000_n16_zero2",
                                 "ring3_psi1m_zero1"])
def test_noalloc_matches_step_on_two_calls(key):
    wl = reduced_workloads()[key]
    args = (list(wl.tensors), wl.n_ranks, wl.stage, wl.bucket_elems, wl.pad_align, list(wl.units))
    uploaded = zs.Layout(*args).to_device()
    host_only = zs.Layout(*args)                  # never uploaded: nothing allocated for it
    assert host_only.n_segments <= _abi.NOALLOC_MAX_SEGMENTS
    ref, _ = S.oracle_run(wl, 2)
    a = _bufs(uploaded.padded, wl)
    b = _bufs(uploaded.padded, wl)
    guards = S.guard_outputs(b)            # a write past any output buffer shows up here
    for t in (1, 2):
        zs.step(uploaded, a["g"], a["master"], a["m"], a["v"], a["p16_shard"], a["p16_full"], _hp(wl, t),
                nonfinite=a["nonfinite"])
        zs.step_noalloc(host_only, b["g"], b["master"], b["m"], b["v"], b["p16_shard"], b["p16_full"],
                        _hp(wl, t), nonfinite=b["nonfinite"])
        torch.cuda.synchronize()
        S.assert_guards_intact(guards, f"call {t}")
        S.assert_f32_close(_np(b["master"]), _np(a["master"]), f"master after call {t}")
        S.assert_f32_close(_np(b["m"]), _np(a["m"]), f"m after call {t}")
        S.assert_f32_close(_np(b["v"]), _np(a["v"]), f"v after call {t}")
        S.assert_f16_ulp(_np(b["p16_full"]), _np(a["p16_full"]), f"p16_full after call {t}")
        if wl.stage == 3:
            S.assert_f16_ulp(_np(b["p16_shard"]), _np(a["p16_shard"]), f"p16_shard after call {t}")
        assert np.array_equal(_np(b["nonfinite"]), _np(a["nonfinite"]))
        # the header promises more than the tolerance: the same bits as zero_step
        names = ("master", "m", "v", "p16_full") + (("p16_shard",) if wl.stage == 3 else ())
        for name in names:
            S.assert_bits_equal(_np(b[name]), _np(a[name]), f"{name} after call {t} (bits)")
    # and both equal the oracle's two steps
    S.assert_state_matches_oracle(wl, b, ref, "zero_step_noalloc: ")


def test_noalloc_rejects_layouts_beyond_its_table():
    # one rank, 8-element buckets: 12,500 segments, more than the static table holds
    lay = zs.Layout([100_000], 1, 1, 8, 8)
    assert lay.n_segments > _abi.NOALLOC_MAX_SEGMENTS
    g = torch.zeros((1, lay.padded), dtype=torch.int16, device="cuda")
    st = [torch.zeros(lay.padded, dtype=torch.float32, device="cuda") for _ in range(3)]
    p16 = torch.zeros(lay.padded, dtype=torch.int16, device="cuda")
    with pytest.raises(zs.ZeroError) as e:
        zs.step_noalloc(lay, g, *st, None, p16, zs.AdamW())
    assert e.value.status == 1
