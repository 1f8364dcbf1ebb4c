"""CPU checks of the ZeRO-3 schedule's gather-width tuner (schedule.GatherWidth): it
times whole passes through their events and keeps the width with the lowest mean.  The
events are stand-ins with host timestamps, so no GPU is needed; each pass goes through
begin_pass / end_pass as zero3_pass drives them."""
import pytest

from zero_sharded_optimizer_ring_b200.schedule import GatherWidth, layer_breakdown


class FakeEvent:
    def __init__(self, t, done=True):
        self.t, self.done = t, done

    def elapsed_time(self, other):
        return other.t - self.t

    def query(self):
        return self.done


def fake_pass(total_ms, units=4, done=True):
    """A pass of `units` layers ending total_ms after its start event."""
    start = FakeEvent(0.0)
    step = total_ms / units
    marks = [(FakeEvent(j * step), FakeEvent(j * step + 0.1), FakeEvent((j + 1) * step, done))
             for j in range(units)]
    return marks, start


def run_pass(w, pass_ms, done=True):
    """One pass through the tuner's protocol, as zero3_pass drives it.  pass_ms(ctas) ->
    the pass time at that width."""
    ctas = w.begin_pass()
    marks, start = fake_pass(pass_ms(ctas), done=done)
    w.end_pass(marks, start)
    return ctas, marks


def test_layer_breakdown_reads_the_fake_events():
    marks, start = fake_pass(4.0, units=4)
    bd = layer_breakdown(marks, start)
    assert bd["wait_ms"] == pytest.approx([0.1, 0.1, 0.1, 0.1])
    assert bd["sum_compute_ms"] == pytest.approx(3.6)


def test_candidates_in_alternating_rounds_then_the_fastest_kept():
    w = GatherWidth(candidates=(14, 16, 18, 20), trials=3)
    times = {14: 12.0, 16: 11.5, 18: 11.0, 20: 11.8}
    seen = [run_pass(w, times.get)[0] for _ in range(17)]
    assert seen[0] == 14                             # the untimed warm-up
    assert seen[1:13] == [14, 16, 18, 20, 20, 18, 16, 14, 14, 16, 18, 20]
    assert seen[14:] == [18, 18, 18]                 # the 14th pass read the 13th; 18 kept
    assert w.chosen == 2 and w.ctas == 18
    assert w.means() == pytest.approx([12.0, 11.5, 11.0, 11.8])


def test_a_steady_drift_does_not_pick_the_wrong_width():
    """Every pass 0.1 ms slower than the one before: alternating rounds add the same
    drift to every candidate, so the truly fastest still wins."""
    w = GatherWidth(candidates=(14, 16, 18, 20), trials=2)
    base = {14: 10.6, 16: 10.3, 18: 10.0, 20: 10.45}
    n = [0]

    def pass_ms(c):
        n[0] += 1
        return base[c] + 0.1 * n[0]

    for _ in range(11):
        run_pass(w, pass_ms)
    assert w.candidates[w.chosen] == 18


def test_first_pass_is_not_timed():
    w = GatherWidth(candidates=(14, 16), trials=1)
    run_pass(w, lambda c: 500.0)                      # a slow first pass (start-up costs)
    run_pass(w, lambda c: 5.0 if c == 14 else 6.0)
    run_pass(w, lambda c: 5.0 if c == 14 else 6.0)
    run_pass(w, lambda c: 5.0)
    assert w.means() == pytest.approx([5.0, 6.0]) and w.candidates[w.chosen] == 14


def test_unfinished_pass_is_read_later_or_skipped():
    w = GatherWidth(candidates=(14, 16), trials=1)
    run_pass(w, lambda c: 5.0)                        # warm-up
    c0, marks0 = run_pass(w, lambda c: 5.0, done=False)
    assert c0 == 14
    c1, _ = run_pass(w, lambda c: 5.0)                # the first is not finished: not read,
    assert c1 == 14 and w.count == [0, 0]             # the same width is timed again
    run_pass(w, lambda c: 5.0)
    assert w.count == [1, 0]


def test_single_candidate_is_fixed():
    w = GatherWidth(candidates=(16,), trials=2)
    assert [run_pass(w, lambda c: 1.0)[0] for _ in range(5)] == [16] * 5
    assert w.chosen == 0


def test_rejects_bad_arguments():
    with pytest.raises(ValueError):
        GatherWidth(candidates=())
    with pytest.raises(ValueError):
        GatherWidth(candidates=(0, 16))
    with pytest.raises(ValueError):
        GatherWidth(trials=0)
