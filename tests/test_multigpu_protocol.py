"""The multi-GPU step's protocol on CPU (gloo, 2 and 3 ranks, no GPU): every shard is
updated exactly once per step by its owner, every rank gathers every other shard from
its owner, every read of a peer's buffer is enqueued after the host barrier that makes
that buffer complete, and, in each rank's own stream order, after a wait on that peer's
event for the phase that completed the buffer."""
import os
import socket
import sys
import time

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


class FakeLayout:
    def __init__(self, n, stage=1, n_units=3):
        self.n_ranks, self.stage, self.n_units = n, stage, n_units


class RecordingOps:
    """Stands in for the device: records what would run, and when."""

    def __init__(self, rank):
        self.rank, self.log = rank, []

    def _rec(self, *what):
        self.log.append((time.monotonic(), self.rank) + what)

    def export(self, t):
        return f"{t}@{self.rank}".encode()

    def open(self, handle):
        self._rec("open", handle.decode())
        return "mapped:" + handle.decode()

    def close(self, ptr):
        self._rec("close", ptr)

    def step_shard(self, layout, shard, rank_grads, master_k, m_k, v_k, p16_full, hp, nonfinite):
        self._rec("update", shard, tuple(rank_grads), hp)

    def copy_shard(self, layout, shard, src, dst):
        self._rec("gather", shard, src, dst)

    def gather_unit_ranks(self, layout, unit, shards, dst, stream=None):
        self._rec("unit", unit, tuple(shards), dst)

    def sync(self):
        self._rec("barrier")

    def new_fence(self):
        self.n_fences = getattr(self, "n_fences", 0) + 1
        return f"fence{self.n_fences}@{self.rank}"

    def fence_handle(self, ev):
        return ev.encode()

    def open_fence(self, handle):
        return "mapped:" + handle.decode()

    def record(self, ev, name):
        self._rec("record", name)

    def wait(self, ev, name, stream=None):
        self._rec("wait", name[0], name[1])


def _check_stream_order(log, world, stage=1):
    """In one rank's log (its stream order): every device op that reads a peer's buffer
    comes after a wait on that peer's event of the phase that completed the buffer, and a
    rank rewrites its own parameters only after waiting for every peer to finish reading
    them."""
    rank = log[0][1]
    peers = [r for r in range(world) if r != rank]
    waited = set()                      # (phase, peer) waited on since that phase's last record
    n_updates = 0
    for e in log:
        what = e[2]
        if what == "record":
            waited = {w for w in waited if w[0] != e[3]}
        elif what == "wait":
            waited.add((e[3], e[4]))
        elif what == "update":
            assert all(("grads", j) in waited for j in peers), (rank, "update before every peer's grads")
            if n_updates and stage != 3:
                assert all(("gathered", j) in waited for j in peers), (rank, "rewrites p16 still being read")
            n_updates += 1
        elif what == "gather":
            assert ("updated", e[3]) in waited, (rank, "copies a shard before its owner's update")
        elif what == "unit":
            assert all(("updated", j) in waited for j in peers), (rank, "gathers a layer before its owners' update")


def _worker(rank, world, port, steps, out, stage=1):
    import datetime
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    from zero_sharded_optimizer_ring_b200.multigpu import RankStep
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    ops = RecordingOps(rank)
    lay = FakeLayout(world, stage)
    rs = RankStep(lay, rank, world, "grads", "m0", "m1", "m2", "p16", ops=ops)
    for t in range(steps):
        ops._rec("grads_written", t)
        rs.step(hp=t)
        if stage == 3:                  # the next forward and backward fetch every layer twice
            for u in list(range(lay.n_units)) + list(range(lay.n_units))[::-1]:
                rs.gather_unit(u, f"slot{u % 2}")
    rs.close()
    out.put(ops.log)
    dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_multigpu_step_protocol(world):
    steps = 3
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, steps, q)) for r in range(world)]
    for p in procs:
        p.start()
    logs = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(60)
        assert p.exitcode == 0
    ev = sorted(e for log in logs for e in log)

    for t in range(steps):
        updates = [e for e in ev if e[2] == "update" and e[5] == t]
        assert sorted((e[1], e[3]) for e in updates) == [(r, r) for r in range(world)]   # owner updates own shard
        for e in updates:                                   # reads the right buffers
            assert e[4] == tuple("grads" if r == e[1] else f"mapped:grads@{r}" for r in range(world))
        written = max(e[0] for e in ev if e[2] == "grads_written" and e[3] == t)
        assert min(e[0] for e in updates) > written         # nobody reads gradients still being written
        done = max(e[0] for e in updates)
        step_gathers = [e for e in ev if e[2] == "gather"][t * world * (world - 1):(t + 1) * world * (world - 1)]
        assert all(done < e[0] for e in step_gathers)       # nobody reads parameters before their update
        assert sorted((e[1], e[3]) for e in step_gathers) == \
            sorted((r, j) for r in range(world) for j in range(world) if j != r)
        for e in step_gathers:
            assert e[4] == f"mapped:p16@{e[3]}" and e[5] == "p16"
        if t + 1 < steps:                                   # next step's gradients after this step's reads
            nxt = min(e[0] for e in ev if e[2] == "grads_written" and e[3] == t + 1)
            assert nxt > max(e[0] for e in step_gathers)
    closes = [e for e in ev if e[2] == "close"]
    assert len(closes) == world * 2 * (world - 1)
    for log in logs:
        _check_stream_order(log, world)


@pytest.mark.parametrize("world", [2, 3])
def test_multigpu_zero3_protocol(world):
    """ZeRO-3: no third phase; every layer is gathered from all owners' shards, after every
    owner has written its shard for the step and before any owner writes it again."""
    steps = 3
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, steps, q, 3)) for r in range(world)]
    for p in procs:
        p.start()
    logs = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(60)
        assert p.exitcode == 0
    ev = sorted(e for log in logs for e in log)
    assert not [e for e in ev if e[2] == "gather"]                   # no full-buffer copies
    units = [e for e in ev if e[2] == "unit"]
    assert len(units) == steps * world * 2 * 3
    for e in units:                                                   # every owner's shard, mapped
        assert e[4] == tuple("p16" if r == e[1] else f"mapped:p16@{r}" for r in range(world))
    for t in range(steps):
        updates = [e for e in ev if e[2] == "update" and e[5] == t]
        assert sorted((e[1], e[3]) for e in updates) == [(r, r) for r in range(world)]
        step_units = units[t * world * 6:(t + 1) * world * 6]
        assert min(e[0] for e in step_units) > max(e[0] for e in updates)   # after every shard is written
        if t + 1 < steps:
            nxt = [e for e in ev if e[2] == "update" and e[5] == t + 1]
            assert max(e[0] for e in step_units) < min(e[0] for e in nxt)   # before any is rewritten
    for log in logs:
        _check_stream_order(log, world, stage=3)


class DynamicOps(RecordingOps):
    """RecordingOps plus the commit step: shard `bad_at[0]` reports an overflow at step
    `bad_at[1]`; the all-reduce is a real one over the gloo group."""

    def __init__(self, rank, bad_at):
        super().__init__(rank)
        self.bad_at = bad_at
        self.t = 0

    def step_shard_commit(self, layout, shard, rank_grads, state_in, state_out, p16_out, hp, scaler, nonfinite):
        self._rec("commit", shard, state_in, state_out, p16_out)
        return 5 if (shard, self.t) == self.bad_at else 0

    def all_reduce_sum(self, x, group=None):
        import torch
        import torch.distributed as dist
        t = torch.tensor([x], dtype=torch.int64)
        dist.all_reduce(t, group=group)
        self._rec("allreduce", int(t.item()))
        return int(t.item())

    def advance(self, scaler, applied):
        scaler.append(applied)
        self._rec("advance", applied)


def _dyn_worker(rank, world, port, steps, bad_at, out):
    import datetime
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    from zero_sharded_optimizer_ring_b200.multigpu import RankStep
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    ops = DynamicOps(rank, bad_at)
    rs = RankStep(FakeLayout(world), rank, world, "grads", "a0", "a1", "a2", "p16a", ops=ops,
                  spare=("b0", "b1", "b2", "p16b"))
    decisions = []
    for t in range(steps):
        ops.t = t
        ops._rec("grads_written", t)
        rs.step_dynamic(hp=t, scaler=decisions, nonfinite="nf")
        ops._rec("current", rs.state, rs.p16)
    rs.close()
    out.put((rank, decisions, ops.log))
    dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_multigpu_dynamic_commit_protocol(world):
    """One shard overflows at step 1: every rank skips that step (same decision, no
    gathers, the current set unchanged); every applied step reads the current set, writes
    the other one, swaps everywhere and gathers the owners' new buffers."""
    steps, bad_at = 4, (world - 1, 1)
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_dyn_worker, args=(r, world, port, steps, bad_at, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted([q.get(timeout=120) for _ in range(world)], key=lambda x: x[0])
    for p in procs:
        p.join(60)
        assert p.exitcode == 0
    want = [True, False, True, True]
    for rank, decisions, log in res:
        assert decisions == want                                      # the same decision everywhere
        commits = [e for e in log if e[2] == "commit"]
        currents = [e for e in log if e[2] == "current"]
        cur = ("a0", "a1", "a2"), "p16a"
        other = {"a": (("b0", "b1", "b2"), "p16b"), "b": (("a0", "a1", "a2"), "p16a")}
        for t, applied in enumerate(want):
            c = commits[t]
            assert c[3] == rank and c[4] == cur[0]                   # reads the current set
            nxt = other[cur[1][-1]]
            assert (c[5], c[6]) == nxt                                # writes the other one
            if applied:
                cur = nxt
            assert (currents[t][3], currents[t][4]) == cur
        gathers = [e for e in log if e[2] == "gather"]
        assert len(gathers) == (world - 1) * sum(want)                # none for the skipped step
        for e in gathers:
            assert e[4].startswith("mapped:p16") and e[5] in ("p16a", "p16b") and e[4].endswith(f"@{e[3]}")
            assert e[4][len("mapped:"):].split("@")[0] == e[5]        # from the owners' current buffer


def _dying_worker(rank, world, port, out):
    import datetime
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    from zero_sharded_optimizer_ring_b200.multigpu import RankStep
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=10))
    ops = RecordingOps(rank)
    rs = RankStep(FakeLayout(world), rank, world, "grads", "m0", "m1", "m2", "p16", ops=ops)
    rs.step(hp=0)                                       # one good step on every rank
    if rank == world - 1:
        os._exit(3)                                     # this rank dies between steps
    t0 = time.monotonic()
    try:
        rs.step(hp=1)
        out.put((rank, "no error", time.monotonic() - t0, ops.log))
    except Exception as e:                              # the barrier reports the dead peer
        out.put((rank, type(e).__name__, time.monotonic() - t0, ops.log))


def test_dead_rank_stops_the_others_at_the_first_barrier():
    """A rank that dies between steps is noticed by the others at their next host barrier
    (the process group ends it with an error within its timeout): no surviving rank starts
    the update that would read the dead rank's gradients."""
    world = 3
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_dying_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(world - 1)]
    for p in procs:
        p.join(60)
    assert procs[-1].exitcode == 3
    for rank, what, seconds, log in res:
        assert what != "no error" and seconds < 60, (rank, what, seconds)
        updates = [e for e in log if e[2] == "update"]
        assert [e[5] for e in updates] == [0]           # step 1's update never started
