"""Pins of the oracle's fp16-wire ring and its dynamic loss scaling.

- one hop of the fp16 wire is the correctly rounded fp16 sum (numpy's double -> half
  conversion of the exact double sum);
- hand-computed three-rank cases where the wire and fp32 accumulation differ (rounding
  at every hop; overflow of a partial sum, which depends on the ring order);
- the scaler's state machine against a hand-derived trace (golden fixture);
- skipped steps change no state; applied steps equal a plain step at the scale used.
"""
import json
import os

import numpy as np

import oracle
from oracle.layout import make_layout

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _ring(g16, wire16, shard=None):
    g = np.ascontiguousarray(np.asarray(g16, dtype=np.float16).view(np.uint16))
    N, P = g.shape
    red = np.zeros(P, np.float32)
    oracle.ring_reduce_scatter(g, shard or P // N, 0, P, reduced=red, wire16=wire16)
    return red


def test_one_wire_hop_is_the_rounded_fp16_sum():
    rng = np.random.default_rng(31)
    bits = rng.integers(0, 1 << 16, (2, 200_000), dtype=np.uint32).astype(np.uint16)
    bits[(bits & 0x7C00) == 0x7C00] = 0x3C00                         # no inf / nan inputs
    a = bits.view(np.float16)
    red = _ring(a, True, shard=a.shape[1])                          # one shard: fold from rank 0
    with np.errstate(over="ignore"):
        want = (a[0].astype(np.float64) + a[1].astype(np.float64)).astype(np.float16)
        got = red.astype(np.float16)
    assert np.array_equal(got.view(np.uint16), want.view(np.uint16))


def test_wire_rounds_at_every_hop():
    # ranks 0, 1, 2 hold 1, 2^-11, 2^-11 for an element of shard 0
    g = np.zeros((3, 3), np.float16)
    g[:, 0] = [1.0, 2.0 ** -11, 2.0 ** -11]
    assert _ring(g, False)[0] == np.float32(1 + 2.0 ** -10)         # fp32: exact
    assert _ring(g, True)[0] == np.float32(1.0)                     # each 1 + 2^-11 ties to 1


def test_wire_overflow_depends_on_ring_order():
    # shard 0 folds ranks 0, 1, 2; shard 1 folds 1, 2, 0
    g = np.zeros((3, 2), np.float16)
    g[:, 0] = [40000.0, 40000.0, -40000.0]        # 80000 overflows fp16 at the first hop
    g[:, 1] = [40000.0, -40000.0, 40000.0]        # from rank 1: -40000 + 40000 = 0, then 40000
    red = _ring(g, True, shard=1)
    assert np.isinf(red[0]) and red[1] == np.float32(40000.0)
    red32 = _ring(g, False, shard=1)
    assert red32[0] == np.float32(40000.0) and red32[1] == np.float32(40000.0)


def test_scaler_follows_hand_trace():
    gold = json.load(open(os.path.join(GOLDEN, "loss_scaler_trace.json")))
    sc = oracle.LossScaler(gold["scale"], gold["factor"], gold["window"], gold["min_scale"])
    for overflow, want in zip(gold["overflow"], gold["expect"]):
        used = sc.scale
        sc.update(overflow)
        assert used == want["scale_used"]
        assert (0 if overflow else sc.step) == want["applied_step"]
    f = gold["final"]
    assert (sc.scale, sc.clean_steps, sc.step, sc.skipped) == (f["scale"], f["clean_steps"], f["step"], f["skipped"])


def test_dynamic_run_skips_overflowing_steps():
    N, n = 4, 4096
    lay = make_layout([n], N, 1000, 8)
    P = lay.padded
    rng = np.random.default_rng(5)
    z = rng.standard_normal((N, P))
    z[:, n:] = 0

    def grads_at(scale, i):
        with np.errstate(over="ignore"):
            return np.ascontiguousarray((z * 1e-3 * scale).astype(np.float16).view(np.uint16))

    master = (rng.standard_normal(P) * 0.02).astype(np.float32)
    master[n:] = 0
    zero = np.zeros(P, np.float32)
    hp = oracle.Hyper()
    for wire in (False, True):
        sc = oracle.LossScaler(2.0 ** 26, window=2)
        last, trace = oracle.run_steps_dynamic(lay, 1, grads_at, master, zero, zero, hp, 8, sc, wire16=wire)
        assert any(o for _, o, _ in trace) and not all(o for _, o, _ in trace)
        # replay: applied steps equal plain single steps at the scale each one used
        st = [master.copy(), zero.copy(), zero.copy()]
        t = 0
        for i, (used, overflow, step) in enumerate(trace):
            if overflow:
                continue
            t += 1
            assert step == t
            h = oracle.Hyper(loss_scale=used)
            r = oracle.run_steps(lay, 1, grads_at(used, i), *st, h, 1, wire16=wire, first_step=t)
            st = [r.master, r.m, r.v]
        assert np.array_equal(st[0].view(np.uint32), last.master.view(np.uint32))
        assert sc.step == t and sc.skipped == sum(o for _, o, _ in trace)
