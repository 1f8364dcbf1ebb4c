"""Pins of the oracle's layout, stage composition and per-rank accounting.

- layout: brute-force membership on tiny sizes; the 3-GPU "thirds" split;
- stages 0 (DDP), 1, 2, 3 and any bucket split give bit-identical results, with every
  rank's replica identical after the all-gathers;
- all-gather = concatenation of the ranks' partitions;
- literal ring send counts equal the closed-form counters; the closed forms reproduce
  the pages' 16 psi, ~4x / ~8x / N x savings and the 1.5x ZeRO-3 communication.
"""
import json
import os

import numpy as np
import pytest

import oracle
from oracle.layout import ceil_div, counters, make_layout

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def test_layout_brute_force():
    rng = np.random.default_rng(11)
    for _ in range(400):
        N = int(rng.integers(1, 7))
        tensors = [int(x) for x in rng.integers(0, 30, int(rng.integers(0, 6)))]
        A = int(rng.choice([1, 2, 8, 128]))
        B = int(rng.integers(-2, 60))
        lay = make_layout(tensors, N, B, A)
        psi = sum(tensors)
        assert lay.psi == psi
        if psi == 0:
            assert lay.padded == 0 and lay.buckets == [] and lay.segments == []
            continue
        S, P = lay.shard, lay.padded
        assert S % A == 0 and S >= ceil_div(psi, N) and S - A < ceil_div(psi, N)
        assert P == N * S >= psi
        assert lay.tensor_off == list(np.cumsum([0] + tensors)[:-1])
        owner_b = np.full(P, -1)
        for b, (lo, hi) in enumerate(lay.buckets):
            assert 0 <= lo < hi <= P and (B <= 0 or hi - lo <= B)
            assert np.all(owner_b[lo:hi] == -1)
            owner_b[lo:hi] = b
        assert np.all(owner_b >= 0)
        assert lay.buckets[0][1] == P                  # the last gradients form bucket 0
        assert all(lay.buckets[b][0] == lay.buckets[b + 1][1] for b in range(len(lay.buckets) - 1))
        seen = np.zeros(P, int)
        for b, k, lo, hi in lay.segments:
            assert lay.buckets[b][0] <= lo < hi <= lay.buckets[b][1]
            assert k * S <= lo and hi <= (k + 1) * S
            seen[lo:hi] += 1
        assert np.all(seen == 1)


def test_three_gpu_thirds():
    lay = make_layout([3 * 1000], 3, 0, 1)
    assert lay.shard == 1000
    assert [(k * lay.shard, (k + 1) * lay.shard) for k in range(3)] == [(0, 1000), (1000, 2000), (2000, 3000)]


def _tiny(rng):
    N = int(rng.integers(1, 6))
    tensors = [int(x) for x in rng.integers(1, 40, int(rng.integers(1, 7)))]
    A = int(rng.choice([1, 4, 8]))
    lay0 = make_layout(tensors, N, 0, A)
    P = lay0.padded
    psi = lay0.psi
    g = (rng.standard_normal((N, P)) * 3).astype(np.float16)
    g[:, psi:] = 0
    master = np.zeros(P, np.float32)
    master[:psi] = rng.standard_normal(psi) * 0.02
    m = np.zeros(P, np.float32)
    v = np.zeros(P, np.float32)
    m[:psi] = rng.standard_normal(psi) * 1e-3
    v[:psi] = np.abs(rng.standard_normal(psi)) * 1e-5
    units = sorted({0} | {int(x) for x in rng.integers(0, len(tensors), 2)})
    return N, tensors, A, g.view(np.uint16).copy(), master, m, v, units


def test_stages_and_bucket_splits_are_bit_identical():
    rng = np.random.default_rng(12)
    hp = oracle.Hyper(loss_scale=16.0)
    for _ in range(40):
        N, tensors, A, g, master, m, v, units = _tiny(rng)
        ref = None
        for stage in (0, 1, 2, 3):
            for B in (0, 1, 7, 33):
                lay = make_layout(tensors, N, B, A, units)
                r = oracle.run_steps(lay, stage, g, master, m, v, hp, 3, replicas=True)
                assert r.replicas_identical
                got = [r.master, r.m, r.v, r.p16_full, r.reduced]
                if ref is None:
                    ref = got
                for a, b in zip(got, ref):
                    assert np.array_equal(a.view(np.uint8), b.view(np.uint8)), (stage, B)


def test_allgather_is_concatenation_of_partitions():
    rng = np.random.default_rng(13)
    for _ in range(20):
        N, tensors, A, g, master, m, v, units = _tiny(rng)
        lay = make_layout(tensors, N, 5, A, units)
        for stage in (1, 3):
            r = oracle.run_steps(lay, stage, g, master, m, v, oracle.Hyper(), 1, replicas=True)
            parts = [r.p16_shard[k * lay.shard:(k + 1) * lay.shard] for k in range(N)]
            assert np.array_equal(r.p16_full, np.concatenate(parts))


def test_literal_send_counts_match_closed_form():
    rng = np.random.default_rng(14)
    for _ in range(20):
        N, tensors, A, g, master, m, v, units = _tiny(rng)
        lay = make_layout(tensors, N, int(rng.integers(1, 30)), A, units)
        S = lay.shard
        for stage in (0, 1, 2, 3):
            r = oracle.run_steps(lay, stage, g, master, m, v, oracle.Hyper(), 1, replicas=True)
            c = counters(lay, stage)
            one_phase = (N - 1) * S
            literal = r.sent
            if stage == 3:
                # the step runs the scatter-reduce and one gather pass; the backward pass
                # gathers the same units once more
                literal = literal + one_phase
            assert np.all(literal == c.sent_elems) and np.all(r.recv + (literal - r.sent) == c.recv_elems)


def test_memory_and_comm_closed_forms_match_pages():
    gold = json.load(open(os.path.join(GOLDEN, "memory_comm.json")))
    psi = 10 ** 12 + 7
    for N in (4, 64, 4096, 10 ** 6):
        lay = make_layout([psi], N, 0, 1)
        ddp = counters(lay, 0)
        d = gold["ddp_bytes_per_param"]
        assert (ddp.mem_p16, ddp.mem_g16, ddp.mem_os, ddp.mem_total) == \
            (d["p16"] * psi, d["g16"] * psi, d["os"] * psi, d["total"] * psi)
        z1, z2, z3 = (counters(lay, s) for s in (1, 2, 3))
        assert z1.sent_elems == z2.sent_elems == ddp.sent_elems
        assert z3.sent_elems * 2 == ddp.sent_elems * 3          # 1.5x
        # S = ceil(psi/N) pads each shard by < 1 element, hence rel = 2N/psi below
        assert z3.sent_elems / psi == pytest.approx(gold["comm_stage3_in_units_of_psi"] * (N - 1) / N, rel=2 * N / psi)
        assert ddp.sent_elems / psi == pytest.approx(gold["comm_ddp_in_units_of_psi"] * (N - 1) / N, rel=2 * N / psi)
        assert ddp.mem_total / z3.mem_total == pytest.approx(N, rel=1e-5)
    # the ~4x and ~8x savings are the large-N limits
    lay = make_layout([psi], 10 ** 6, 0, 1)
    for stage, want in gold["saving_vs_ddp_large_n"].items():
        ratio = counters(lay, 0).mem_total / counters(lay, int(stage)).mem_total
        assert ratio == pytest.approx(want, rel=1e-4)
