"""The step with one process per GPU (host orchestration only).

Rank r holds its own fp16 gradients [P], the optimizer state of shard r (master, m, v:
[S] each, rank r owning shard r as in rkmt.cn/news/44736 "Deepspeed ZeRO-1", where GPU0
is responsible for the first third) and, for ZeRO stages 0-2, the full fp16 parameters
[P]; for ZeRO-3 only its own shard of them [S] ("Deepspeed ZeRO-3": every GPU keeps its
part of the parameters and fetches the rest layer by layer when it needs them).
Every rank maps the other ranks' gradient and parameter buffers, and three
interprocess CUDA events of theirs (one per phase), with CUDA IPC once; a step then runs
three phases, each closed by a fence:

  1. every rank's gradients are complete (fence "grads");
  2. rank r runs zero_step_shard for shard r: the fused kernel pulls the shard's slices
     from all N gradient buffers over NVLink and folds them in the ring order r, r+1, ...,
     r+N-1, which equals the single-GPU simulation bit for bit (fence "updated");
  3. stages 0-2: rank r copies every other shard's new fp16 parameters from its owner's
     buffer into its own (the all-gather; fence "gathered", before anyone writes those
     buffers again).  Stage 3 has no third phase: gather_unit() later fetches one layer
     from all owners' shards, on a stream that first waits for every owner's "updated"
     mark; the shards stay unchanged until the owners' next phase 2, which waits for
     every rank's next "grads" mark, i.e. for the end of its forward and backward.

A fence is stream-ordered, not a device synchronisation: each rank records its phase
event on its stream, a host barrier makes sure every rank's record is enqueued, and each
rank's stream then waits for every peer's event.  The GPU never drains between phases,
and no kernel waits on another GPU: the waits are stream dependencies resolved before a
kernel starts, so each kernel only reads peer memory that is complete and stable.

Under dynamic loss scaling (step_dynamic) every rank keeps a second state set and a
second parameter buffer.  Phase 2 becomes the first half of a two-phase commit: the
owner writes its shard's step into the spare set (zero_step_shard_commit) and counts the
non-finite reduced gradients; one all-reduce of that integer (the only exchange this
adds) gives every rank the same decision, after which all scalers advance alike and,
if no shard overflowed, every rank makes the spare set current and phase 3 follows.
"""


class CudaOps:
    """The device operations of a step, through the library's C ABI."""

    def __init__(self):
        import zero_sharded_optimizer_ring_b200 as zs
        self.zs = zs

    def export(self, t):
        return self.zs.ipc_handle(t)

    def open(self, handle):
        return self.zs.ipc_open(handle)             # (device address, offset)

    def close(self, mapped):
        self.zs.ipc_close(mapped)

    @staticmethod
    def _addr(x):
        return x[0] if isinstance(x, tuple) else x

    def step_shard(self, layout, shard, rank_grads, master_k, m_k, v_k, p16, hp, nonfinite):
        self.zs.step_shard(layout, shard, [self._addr(g) for g in rank_grads], master_k, m_k, v_k, p16, hp,
                           nonfinite)

    def copy_shard(self, layout, shard, src, dst):
        self.zs.copy_shard(layout, shard, self._addr(src), dst)

    def gather_unit_ranks(self, layout, unit, shards, dst, stream=None):
        self.zs.gather_unit_ranks(layout, unit, [self._addr(p) for p in shards], dst, stream=stream)

    def step_shard_commit(self, layout, shard, rank_grads, state_in, state_out, p16_out, hp, scaler, nonfinite):
        return self.zs.step_shard_commit(layout, shard, [self._addr(g) for g in rank_grads], state_in, state_out,
                                         p16_out, hp, scaler, nonfinite)

    def all_reduce_sum(self, x, group=None):
        import torch
        import torch.distributed as dist
        dev = "cuda" if dist.get_backend(group) == "nccl" else "cpu"
        t = torch.tensor([int(x)], dtype=torch.int64, device=dev)
        dist.all_reduce(t, group=group)
        return int(t.item())

    def advance(self, scaler, applied):
        scaler.advance(applied)

    def sync(self):
        import torch
        torch.cuda.synchronize()

    # phase fences: interprocess events (no timing), recorded and waited on streams
    def new_fence(self):
        import torch
        return torch.cuda.Event(interprocess=True)

    def fence_handle(self, ev):
        return ev.ipc_handle()

    def open_fence(self, handle):
        import torch
        return torch.cuda.Event.from_ipc_handle(torch.cuda.current_device(), handle)

    def record(self, ev, name):
        ev.record()                                       # on the current stream

    def wait(self, ev, name, stream=None):
        import torch
        (stream or torch.cuda.current_stream()).wait_event(ev)


class RankStep:
    """One rank's share of the multi-GPU step (see the module docstring)."""

    def __init__(self, layout, rank, world, grads, master_k, m_k, v_k, p16, group=None, ops=None, spare=None):
        """p16: the full fp16 parameters [P] (stages 0-2) or this rank's shard of them [S]
        (stage 3).  spare: (master_k, m_k, v_k, p16) of the same shapes, the second set
        that step_dynamic() needs.  group: the process group of the fences' host barriers;
        a gloo group keeps them on the host (an NCCL group's barrier is itself a GPU
        collective, queued behind this rank's work, so the GPU would drain at every phase)."""
        import torch.distributed as dist
        if layout.n_ranks != world:
            raise ValueError("the layout's rank count must equal the world size")
        self.dist, self.group = dist, group
        self.layout, self.rank, self.world = layout, rank, world
        self.ops = ops or CudaOps()
        self.grads = grads
        self.sets = [((master_k, m_k, v_k), p16)]
        if spare is not None:
            self.sets.append((tuple(spare[:3]), spare[3]))
        self.cur = 0
        self.fences = {ph: self.ops.new_fence() for ph in self.PHASES}
        mine = (rank, self.ops.export(grads), [self.ops.export(p) for _, p in self.sets],
                {ph: self.ops.fence_handle(ev) for ph, ev in self.fences.items()})
        everyone = [None] * world
        dist.all_gather_object(everyone, mine, group=group)
        self.opened = []
        self.peer_grads = [None] * world
        self.peer_p16 = [[None] * world for _ in self.sets]       # [set][rank]
        self.peer_fences = {ph: {} for ph in self.PHASES}         # [phase][peer rank]
        for r, hg, hps, hfs in everyone:
            if r == rank:
                self.peer_grads[r] = grads
                for s, (_, p) in enumerate(self.sets):
                    self.peer_p16[s][r] = p
            else:
                self.peer_grads[r] = self.ops.open(hg)
                self.opened.append(self.peer_grads[r])
                for s, h in enumerate(hps):
                    self.peer_p16[s][r] = self.ops.open(h)
                    self.opened.append(self.peer_p16[s][r])
                for ph, h in hfs.items():
                    self.peer_fences[ph][r] = self.ops.open_fence(h)

    @property
    def state(self):
        """The current (master, m, v) of this rank's shard."""
        return self.sets[self.cur][0]

    @property
    def p16(self):
        """The current fp16 parameters (full, or this rank's shard for stage 3)."""
        return self.sets[self.cur][1]

    PHASES = ("grads", "updated", "gathered")

    def _barrier(self):
        self.ops.sync()
        self.dist.barrier(group=self.group)

    def _fence(self, phase):
        """Everything this rank has enqueued so far is `phase`; everything it enqueues from
        now on runs after every peer's `phase` work.  Record, host barrier (all records
        are enqueued before anyone waits), one stream wait per peer."""
        self.ops.record(self.fences[phase], phase)
        self.dist.barrier(group=self.group)
        for r, ev in self.peer_fences[phase].items():
            self.ops.wait(ev, (phase, r))

    def step(self, hp, nonfinite=None):
        self._fence("grads")                                # 1: all gradients written
        self.ops.step_shard(self.layout, self.rank, self.peer_grads, *self.state, self.p16, hp, nonfinite)
        self._fence("updated")                              # 2: every shard updated
        self._gather_all()

    def step_dynamic(self, hp, scaler, nonfinite):
        """One step under dynamic loss scaling (the gradients carry scaler.scale); returns
        True if it was applied on every rank, False if some shard overflowed and every
        rank skipped it.  nonfinite: device int32 [n_buckets] scratch."""
        if len(self.sets) < 2:
            raise ValueError("step_dynamic needs the spare buffer set")
        self._fence("grads")                                # 1: all gradients written
        nxt = 1 - self.cur
        bad = self.ops.step_shard_commit(self.layout, self.rank, self.peer_grads, self.sets[self.cur][0],
                                         self.sets[nxt][0], self.sets[nxt][1], hp, scaler, nonfinite)
        self.ops.record(self.fences["updated"], "updated")  # for stage 3's gather_unit
        # the commit synchronised this rank's stream to read its count; the all-reduce
        # then means every rank's commit (and so its shard) is complete
        applied = self.ops.all_reduce_sum(bad, self.group) == 0   # 2: every rank's shard counted
        self.ops.advance(scaler, applied)
        if applied:
            self.cur = nxt
            self._gather_all()
        return applied

    def _gather_all(self):
        if self.layout.stage == 3:
            return                                          # layers are gathered when used
        for j in range(self.world):
            if j != self.rank:
                self.ops.copy_shard(self.layout, j, self.peer_p16[self.cur][j], self.p16)
        self._fence("gathered")                             # 3: parameters gathered everywhere

    def gather_unit(self, unit, dst, stream=None):
        """Stage 3: unit `unit`'s fp16 parameters into dst, pulled from every owner's shard
        (call between step() and the next step(), e.g. before a layer's forward and again
        before its backward).  `stream` (default: the current one) first waits for every
        owner's last "updated" mark, so a prefetch stream needs no other ordering."""
        if self.layout.stage != 3:
            raise ValueError("stages 0-2 keep the full parameters in p16")
        for r, ev in self.peer_fences["updated"].items():
            self.ops.wait(ev, ("updated", r), stream)
        self.ops.gather_unit_ranks(self.layout, unit, self.peer_p16[self.cur], dst, stream)

    def prefetch(self, slots, gather_stream, compute_stream, **kw):
        """Stage 3: a schedule.Zero3Prefetch whose gathers are this rank's gather_unit
        (every owner's shard; the gather width tuned per kind of pass as on one GPU)."""
        from .schedule import Zero3Prefetch
        return Zero3Prefetch(self.layout, None, slots, gather_stream, compute_stream, gather=self.gather_unit, **kw)

    def close(self):
        """Unmap the peers' buffers (before the process group or the buffers go away)."""
        self._barrier()
        for p in self.opened:
            self.ops.close(p)
        self.opened = []
