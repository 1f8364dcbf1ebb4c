"""Oracle layout and per-rank accounting.  TEST INFRASTRUCTURE ONLY.

Plain Python integers, written from the pages:
  - flat buffer + N-way shards ("thirds" for 3 GPUs): rkmt.cn/news/44736 "Deepspeed
    ZeRO-1" (each GPU is responsible for one third of the gradients/optimizer state);
  - buckets that become ready from the back of the model forward: rkmt.cn/news/44736
    "DDP" (gradients grouped, the first computed group syncs first) and
    "Deepspeed ZeRO-1/-2" (gradients computed back to front), en.pswp.cn/web/84187
    "DDP" (buckets hold several parameters and are reduced bucket by bucket);
  - memory per rank: rkmt.cn/news/44736 "Deepspeed ZeRO" (fp16 params 2B + fp16 grads
    2B + optimizer 12B = 4B first moment + 4B second moment + 4B fp32 params) and which
    of the three each ZeRO stage shards (same page; wangyh.co PaperReading:DeepSpeed
    section 1.5 table);
  - communication per rank: rkmt.cn/news/44736 "DDP" (N-1 rounds of psi/N per phase),
    "Deepspeed ZeRO-1/-2" (same as DDP) and "Deepspeed ZeRO-3" (3 psi in/out per GPU,
    1.5x DDP, "总结").

Readings where the pages are silent: shard S = roundup(ceil(psi/N), A) with zero tail
padding [psi, P); buckets are fixed-size element ranges cut from the tail of the
padded flat buffer (bucket 0 = the last B elements), ignoring tensor boundaries; a
bucket's ring chunk k is its intersection with shard k (a "segment").
"""
from dataclasses import dataclass


def ceil_div(a, b):
    return -(-a // b)


def roundup(a, b):
    return ceil_div(a, b) * b


@dataclass
class OracleLayout:
    psi: int
    n_ranks: int
    shard: int                 # S
    padded: int                # P = N * S
    tensor_off: list           # flat offset of each tensor (concatenated in list order)
    buckets: list              # [(lo, hi)] in bucket order (bucket 0 = tail of the buffer)
    segments: list             # [(bucket, shard, lo, hi)] bucket order, then shard order
    units: list                # [(lo, hi)] stage-3 gather units, ascending, covering [0, P)


def make_layout(tensors, n_ranks, bucket_elems, pad_align=128, units=()):
    if n_ranks < 1 or pad_align < 1 or any(t < 0 for t in tensors):
        raise ValueError("invalid layout description")
    off, acc = [], 0
    for t in tensors:
        off.append(acc)
        acc += t
    psi = acc
    S = roundup(ceil_div(psi, n_ranks), pad_align) if psi > 0 else 0
    P = n_ranks * S

    buckets = []
    if P > 0:
        if bucket_elems <= 0:
            buckets.append((0, P))
        else:
            hi = P
            while hi > 0:
                lo = max(0, hi - bucket_elems)
                buckets.append((lo, hi))
                hi = lo

    segments = []
    for b, (lo, hi) in enumerate(buckets):
        for k in range(n_ranks):
            a, z = max(lo, k * S), min(hi, (k + 1) * S)
            if z > a:
                segments.append((b, k, a, z))

    if P == 0:
        unit_ranges = []
    elif not units:
        unit_ranges = [(0, P)]
    else:
        if units[0] != 0 or any(b <= a for a, b in zip(units, units[1:])) or units[-1] >= len(tensors):
            raise ValueError("gather units must start at tensor 0 and increase")
        starts = [off[u] for u in units]
        ends = starts[1:] + [P]
        unit_ranges = list(zip(starts, ends))
    return OracleLayout(psi, n_ranks, S, P, off, buckets, segments, unit_ranges)


@dataclass
class OracleCounters:
    mem_p16: int      # modelled bytes per rank: fp16 parameters
    mem_g16: int      #                          fp16 gradients
    mem_os: int       #                          fp32 master + first + second moment
    sent_elems: int   # elements each rank sends per step (scatter-reduce + gathers)
    recv_elems: int

    @property
    def mem_total(self):
        return self.mem_p16 + self.mem_g16 + self.mem_os


def counters(lay, stage):
    """Per-rank modelled memory and communication of one training step."""
    psi, S, N = lay.psi, lay.shard, lay.n_ranks
    if stage == 0:        # DDP: everything replicated
        p16, g16, os_ = 2 * psi, 2 * psi, 12 * psi
    elif stage == 1:      # optimizer state sharded
        p16, g16, os_ = 2 * psi, 2 * psi, 12 * S
    elif stage == 2:      # + gradients sharded (each bucket freed after its reduce)
        p16, g16, os_ = 2 * psi, 2 * S, 12 * S
    elif stage == 3:      # + parameters sharded
        p16, g16, os_ = 2 * S, 2 * S, 12 * S
    else:
        raise ValueError("stage must be 0..3")
    # one ring phase moves (N-1) chunks of S per rank; DDP and ZeRO-1/2 have two
    # phases (scatter-reduce + all-gather), ZeRO-3 adds the backward-pass gather.
    phases = 3 if stage == 3 else 2
    comm = phases * (N - 1) * S
    return OracleCounters(p16, g16, os_, comm, comm)
