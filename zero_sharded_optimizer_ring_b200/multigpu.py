"""The step with one process per GPU (host orchestration only).

Rank r holds its own fp16 gradients [P], the optimizer state of shard r (master, m, v:
[S] each, rank r owning shard r as in rkmt.cn/news/44736 "Deepspeed ZeRO-1", where GPU0
is responsible for the first third) and, for ZeRO stages 0-2, the full fp16 parameters
[P]; for ZeRO-3 only its own shard of them [S] ("Deepspeed ZeRO-3": every GPU keeps its
part of the parameters and fetches the rest layer by layer when it needs them).
Every rank maps the other ranks' gradient and parameter buffers with CUDA IPC once; a
step then runs three phases, each closed by a host barrier:

  1. every rank's gradients are complete (barrier);
  2. rank r runs zero_step_shard for shard r: the fused kernel pulls the shard's slices
     from all N gradient buffers over NVLink and folds them in the ring order r, r+1, ...,
     r+N-1, which equals the single-GPU simulation bit for bit (barrier);
  3. stages 0-2: rank r copies every other shard's new fp16 parameters from its owner's
     buffer into its own (the all-gather; barrier before anyone writes those buffers
     again).  Stage 3 has no third phase: gather_unit() later fetches one layer from all
     owners' shards; those stay unchanged until the owners' next phase 2, which comes
     after every rank's next phase-1 barrier, i.e. after its forward and backward.

No kernel waits on another GPU: the barriers are host-side, after a device
synchronisation, so each kernel only reads peer memory that is complete and stable.
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

    def sync(self):
        import torch
        torch.cuda.synchronize()


class RankStep:
    """One rank's share of the multi-GPU step (see the module docstring)."""

    def __init__(self, layout, rank, world, grads, master_k, m_k, v_k, p16, group=None, ops=None):
        """p16: the full fp16 parameters [P] (stages 0-2) or this rank's shard of them [S]
        (stage 3)."""
        import torch.distributed as dist
        if layout.n_ranks != world:
            raise ValueError("the layout's rank count must equal the world size")
        self.dist, self.group = dist, group
        self.layout, self.rank, self.world = layout, rank, world
        self.ops = ops or CudaOps()
        self.grads, self.state, self.p16 = grads, (master_k, m_k, v_k), p16
        mine = (rank, self.ops.export(grads), self.ops.export(p16))
        everyone = [None] * world
        dist.all_gather_object(everyone, mine, group=group)
        self.opened = []
        self.peer_grads = [None] * world
        self.peer_p16 = [None] * world
        for r, hg, hp16 in everyone:
            if r == rank:
                self.peer_grads[r], self.peer_p16[r] = grads, p16
            else:
                self.peer_grads[r] = self.ops.open(hg)
                self.peer_p16[r] = self.ops.open(hp16)
                self.opened += [self.peer_grads[r], self.peer_p16[r]]

    def _barrier(self):
        self.ops.sync()
        self.dist.barrier(group=self.group)

    def step(self, hp, nonfinite=None):
        self._barrier()                                     # 1: all gradients written
        self.ops.step_shard(self.layout, self.rank, self.peer_grads, *self.state, self.p16, hp, nonfinite)
        self._barrier()                                     # 2: every shard updated
        if self.layout.stage == 3:
            return                                          # layers are gathered when used
        for j in range(self.world):
            if j != self.rank:
                self.ops.copy_shard(self.layout, j, self.peer_p16[j], self.p16)
        self._barrier()                                     # 3: parameters gathered everywhere

    def gather_unit(self, unit, dst, stream=None):
        """Stage 3: unit `unit`'s fp16 parameters into dst, pulled from every owner's shard
        (call between step() and the next step(), e.g. before a layer's forward and again
        before its backward)."""
        if self.layout.stage != 3:
            raise ValueError("stages 0-2 keep the full parameters in p16")
        self.ops.gather_unit_ranks(self.layout, unit, self.peer_p16, dst, stream)

    def close(self):
        """Unmap the peers' buffers (before the process group or the buffers go away)."""
        self._barrier()
        for p in self.opened:
            self.ops.close(p)
        self.opened = []
