"""Pins of the oracle's ring scatter-reduce / all-gather.

- the pages' three-GPU a/b/c walk-through, hop by hop (golden fixture);
- an order probe whose result differs for any other starting rank or direction;
- brute force on tiny inputs: exact inputs give the exact sum, general inputs stay
  within the recursive-summation error bound of the exact (float64) sum.
"""
import json
import os

import numpy as np
import pytest

import oracle
from oracle.layout import make_layout

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
CHUNK = {"a": 0, "b": 1, "c": 2}


def _trace_grads():
    # GPU r's copy of chunk c is 2^r * 8^c: a partial sum's value names its terms
    g = np.zeros((3, 3), dtype=np.float16)
    for r in range(3):
        for c in range(3):
            g[r, c] = 2.0 ** r * 8.0 ** c
    return g.view(np.uint16).copy()


def _value(chunk, terms):
    return sum(2.0 ** r * 8.0 ** chunk for r in terms)


def test_three_gpu_walkthrough_scatter_reduce():
    trace = json.load(open(os.path.join(GOLDEN, "ring3_trace.json")))["scatter_reduce"]
    g = _trace_grads()
    _, log = oracle.ring_reduce_scatter(g, 1, 0, 3, want_log=True)
    sends = [{"hop": int(h) + 1, "from": int(s), "to": int(d), "chunk": "abc"[int(k)]}
             for h, s, d, k in log]
    assert sorted(sends, key=str) == sorted(trace["sends"], key=str)
    for hop, holders in trace["after_hop"].items():
        work, _ = oracle.ring_reduce_scatter(g, 1, 0, 3, hops=int(hop))
        for e in holders:
            c = CHUNK[e["chunk"]]
            assert work[e["gpu"], c] == _value(c, e["terms"]), (hop, e)


def test_three_gpu_walkthrough_all_gather():
    trace = json.load(open(os.path.join(GOLDEN, "ring3_trace.json")))["all_gather"]
    g = _trace_grads()
    work, _ = oracle.ring_reduce_scatter(g, 1, 0, 3)
    rep = work.copy()                       # every rank's partial buffer becomes its replica
    log = oracle.ring_allgather(rep, 1, 0, 3, want_log=True)
    first = [tuple(x) for x in log if x[0] == 0]
    fs = trace["first_send"]
    assert (0, fs["from"], fs["to"], CHUNK[fs["chunk"]]) in first
    full = [_value(c, [0, 1, 2]) for c in range(3)]
    for r in range(3):
        assert list(rep[r]) == full


@pytest.mark.parametrize("k", [0, 1, 2])
def test_order_probe(k):
    # chunk k: ranks k and k+1 hold 2^-24 (smallest fp16 subnormal), rank k+2 holds 1.
    # Folding from rank k: (2^-24 + 2^-24) + 1 = 1 + 2^-23.  Starting at k+1 or k+2
    # (or going the other way round) adds a lone 2^-24 to 1 first: a tie, rounded to 1.
    g = np.zeros((3, 3), dtype=np.uint16)
    g[k, k] = 0x0001
    g[(k + 1) % 3, k] = 0x0001
    g[(k + 2) % 3, k] = 0x3C00
    red = np.zeros(3, dtype=np.float32)
    oracle.ring_reduce_scatter(g, 1, 0, 3, reduced=red)
    assert red[k] == np.float32(1.0) + np.float32(2.0 ** -23)


def _random_case(rng, exact):
    N = int(rng.integers(2, 5))
    psi = int(rng.integers(1, 65))
    A = int(rng.choice([1, 2, 4]))
    lay = make_layout([psi], N, int(rng.integers(-1, 20)), A)
    if exact:   # multiples of 2^-10 below 2 in magnitude: every partial sum is exact in fp32
        vals = rng.integers(-2047, 2048, (N, lay.padded)).astype(np.float64) / 1024.0
    else:
        vals = rng.standard_normal((N, lay.padded)) * np.exp(rng.uniform(-8, 8, (N, lay.padded)))
    g = vals.astype(np.float16)
    g[:, psi:] = 0
    return lay, g.view(np.uint16).copy(), g.astype(np.float64)


def _ring_all(lay, g):
    red = np.zeros(lay.padded, dtype=np.float32)
    for lo, hi in lay.buckets:
        oracle.ring_reduce_scatter(g, lay.shard, lo, hi, reduced=red)
    return red


def test_brute_force_exact_inputs_equal_direct_sum():
    rng = np.random.default_rng(7)
    for _ in range(300):
        lay, g, x = _random_case(rng, exact=True)
        red = _ring_all(lay, g)
        assert np.array_equal(red.astype(np.float64), x.sum(axis=0))


def test_brute_force_general_inputs_within_summation_bound():
    rng = np.random.default_rng(8)
    u = 2.0 ** -24
    for _ in range(300):
        lay, g, x = _random_case(rng, exact=False)
        red = _ring_all(lay, g).astype(np.float64)
        n = lay.n_ranks - 1
        bound = n * u / (1 - n * u) * np.abs(x).sum(axis=0)
        assert np.all(np.abs(red - x.sum(axis=0)) <= bound)


def test_two_ranks_is_a_single_rounded_add():
    rng = np.random.default_rng(9)
    g = (rng.standard_normal((2, 1000)) * 10).astype(np.float16)
    lay = make_layout([1000], 2, 300, 4)
    red = _ring_all(lay, g.view(np.uint16).copy())
    assert np.array_equal(red, g[0].astype(np.float32) + g[1].astype(np.float32))


def test_single_rank_is_conversion():
    g = np.arange(0, 5000, dtype=np.uint16).reshape(1, -1) * 13
    lay = make_layout([5000], 1, 999, 1)
    red = _ring_all(lay, g)
    assert np.array_equal(red.view(np.uint32), oracle.half_to_float(g[0]).view(np.uint32))


def test_sampled_path_equals_bucket_simulation():
    rng = np.random.default_rng(10)
    for _ in range(40):
        lay, g, _ = _random_case(rng, exact=False)
        red = _ring_all(lay, g)
        idx = np.arange(lay.padded)
        hp = oracle.Hyper(loss_scale=3.0)
        sc = np.stack([oracle.adamw_scalars(lay.n_ranks, hp, t) for t in (1, 2)])
        master = rng.standard_normal(lay.padded).astype(np.float32)
        zeros = np.zeros(lay.padded, dtype=np.float32)
        r2, p16 = oracle.sampled(g.T.copy(), idx // lay.shard, 2, sc, master.copy(), zeros.copy(), zeros.copy())
        assert np.array_equal(r2.view(np.uint32), red.view(np.uint32))
        full = oracle.run_steps(lay, 1, g, master, zeros, zeros, hp, 2)
        assert np.array_equal(p16, full.p16_full)


@pytest.mark.parametrize("N", [3, 4, 5])
def test_a_dropped_or_duplicated_hop_is_caught(N):
    """Fault injection into the literal ring: one hop fewer leaves every chunk's sum
    without one rank's value, which the exact-sum invariant and the send counts both
    catch; one hop more adds a rank twice into a partial that nobody reads (each sum is
    read from the rank that completed it, which a further send does not change), which
    only the send counts catch.  The counts are the pages' closed form: (N-1)*S
    elements sent and received per rank in one scatter-reduce."""
    S = 8
    rng = np.random.default_rng(40 + N)
    # fp16 values on a 2^-10 grid, |x| < 2 (exactly representable): every partial sum
    # is exact in fp32
    vals = rng.integers(-2047, 2048, size=(N, N * S)) / 1024.0
    g = vals.astype(np.float16).view(np.uint16).copy()
    assert np.all(g.view(np.float16).astype(np.float64) == vals)
    exact = vals.sum(axis=0)
    for hops in (N - 1, N - 2, N):
        red = np.zeros(N * S, dtype=np.float32)
        sent = np.zeros(N, dtype=np.int64)
        recv = np.zeros(N, dtype=np.int64)
        oracle.ring_reduce_scatter(g, S, 0, N * S, hops=hops, reduced=red, sent=sent, recv=recv)
        sums_exact = bool(np.all(red.astype(np.float64) == exact))
        counts_closed_form = bool(np.all(sent == (N - 1) * S) and np.all(recv == (N - 1) * S))
        assert sums_exact == (hops != N - 2), hops
        assert counts_closed_form == (hops == N - 1), hops
