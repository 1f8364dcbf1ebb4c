"""One buffer per rank, one shard at a time, and the multi-process step over CUDA IPC.

- zero_step_ranks on separately allocated per-rank gradient buffers, and zero_step_shard
  run for every shard with shard-local optimizer state, equal the oracle;
- zero_copy_shard copies exactly the shard's range of the stepped parameters, which
  equals the oracle's;
- zero_gather_unit_ranks, reading each rank's own shard buffer as the CUDA step wrote
  it, gives the oracle's gathered layer (vector and element paths, units across shard
  edges, 16 ranks);
- two or three processes sharing this GPU, each holding one rank's gradients and one
  shard's state, run the multi-GPU step (CUDA IPC mappings of buffers and phase events,
  host barriers over gloo; no kernel waits on another process) and end bit-identical to
  the oracle; for ZeRO-3 each keeps only its parameter shard and gathers every layer
  from all owners.
"""
import datetime
import os
import socket
import sys

import numpy as np
import pytest
import torch.multiprocessing as mp

import oracle
import seeded_inputs as si
from seeded_inputs.workloads import Workload, reduced_workloads
import zero_sharded_optimizer_ring_b200 as zs
import support as S

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _hp(wl, t):
    return zs.AdamW(wl.lr, wl.beta1, wl.beta2, wl.eps, wl.weight_decay, wl.loss_scale, t)


def _np(t):
    a = t.cpu().numpy()
    return a.view(np.uint16) if a.dtype == np.int16 else a


def _layout(wl, wire=False):
    return zs.Layout(list(wl.tensors), wl.n_ranks, wl.stage, wl.bucket_elems, wl.pad_align, list(wl.units),
                     wire_fp16=wire).to_device()


def _oracle_ref(wl, steps, wire=False):
    olay = S.oracle_layout(wl)
    g, master, m, v = S.host_inputs(wl, olay.padded)
    return oracle.run_steps(olay, wl.stage, g, master, m, v, S.hyper(wl), steps, wire16=wire)


@pytest.mark.parametrize("key", ["flat1p3b_n4_zero1", "gpt2_small_n8_zero2", "ragged2000_n16_zero2",
                                 "llama3b_n8_zero3"])
@pytest.mark.parametrize("wire", [False, True])
def test_step_ranks_and_step_shard_match_oracle(key, wire):
    wl = reduced_workloads()[key]
    steps = 2
    ref = _oracle_ref(wl, steps, wire)
    lay = _layout(wl, wire)
    P, S_, N = lay.padded, lay.shard, wl.n_ranks
    g, master, m, v = S.device_inputs(wl, P)
    ranks = [g[r].clone() for r in range(N)]                       # separate allocations
    a = dict(master=master.clone(), m=m.clone(), v=v.clone(), p16s=torch.zeros(P, dtype=torch.int16, device="cuda"),
             p16f=torch.zeros(P, dtype=torch.int16, device="cuda"))
    shards = [[x[k * S_:(k + 1) * S_].clone() for x in (master, m, v)] for k in range(N)]
    p16_sh = torch.zeros(P, dtype=torch.int16, device="cuda")
    p16_k = [torch.zeros(S_, dtype=torch.int16, device="cuda") for _ in range(N)]
    for t in range(1, steps + 1):
        zs.step_ranks(lay, ranks, a["master"], a["m"], a["v"], a["p16s"], a["p16f"], _hp(wl, t))
        for k in range(N):
            out = p16_k[k] if wl.stage == 3 else p16_sh
            zs.step_shard(lay, k, ranks, *shards[k], out, _hp(wl, t))
    torch.cuda.synchronize()
    for name, want in (("master", ref.master), ("m", ref.m), ("v", ref.v)):
        S.assert_bits_equal(_np(a[name]), want, name)
        whole = torch.cat([shards[k][("master", "m", "v").index(name)] for k in range(N)])
        S.assert_bits_equal(_np(whole), want, name + " by shard")
    S.assert_bits_equal(_np(a["p16f"]), ref.p16_full, "p16_full")
    if wl.stage == 3:
        S.assert_bits_equal(_np(a["p16s"]), ref.p16_shard, "p16_shard")
        S.assert_bits_equal(_np(torch.cat(p16_k)), ref.p16_shard, "p16 by shard")
    else:
        S.assert_bits_equal(_np(p16_sh), ref.p16_full, "p16 by shard")


def _stepped(wl, steps=2):
    """The CUDA step's fp16 output (stage 3: the shard buffer; else the full buffer) after
    `steps` steps, and the oracle's result on the same inputs."""
    ref = _oracle_ref(wl, steps)
    lay = _layout(wl)
    P = lay.padded
    g, master, m, v = S.device_inputs(wl, P)
    p16s = torch.zeros(P, dtype=torch.int16, device="cuda")
    p16f = torch.zeros(P, dtype=torch.int16, device="cuda")
    for t in range(1, steps + 1):
        zs.step(lay, g, master, m, v, p16s, p16f, _hp(wl, t))
    torch.cuda.synchronize()
    return lay, (p16s if wl.stage == 3 else p16f), ref


def test_copy_shard_copies_exactly_the_shard():
    wl = reduced_workloads()["flat1p3b_n4_zero1"]
    lay, src, ref = _stepped(wl)
    for k in range(lay.n_ranks):
        dst = torch.zeros_like(src)
        zs.copy_shard(lay, k, src, dst)
        torch.cuda.synchronize()
        lo, hi = k * lay.shard, (k + 1) * lay.shard
        got = _np(dst)
        S.assert_bits_equal(got[lo:hi], ref.p16_full[lo:hi], f"shard {k}")
        assert not got[:lo].any() and not got[hi:].any(), f"shard {k}: written outside its range"


@pytest.mark.parametrize("tensors,N,A,units", [
    ((13, 4099, 8190, 5), 3, 1, (0, 1, 3)),            # S not a multiple of 8: element path
    ((13, 4099, 8190, 5), 3, 8, (0, 1, 3)),            # unit starts not 8-aligned: element path
    ((4096, 8192, 40_960, 8), 4, 8, (0, 1, 2, 3)),     # vector path, units across shard edges
    ((1000,) * 16, 16, 8, tuple(range(16))),
])
@pytest.mark.parametrize("gather_ctas", [0, 1, 3])
def test_gather_unit_ranks_matches_oracle(tensors, N, A, units, gather_ctas):
    """gather_ctas 0: a grid of short blocks; k > 0: k persistent CTAs (grid stride)."""
    wl = Workload(name="gather_ranks", description="stage-3 gather from per-rank shards", tensors=tuple(tensors),
                  units=tuple(units), n_ranks=N, stage=3, bucket_elems=0, steps=2, loss_scale=1024.0, pad_align=A)
    lay, whole, ref = _stepped(wl)
    lay.set_gather_ctas(gather_ctas)
    S_ = lay.shard
    shards = [whole[k * S_:(k + 1) * S_].clone() for k in range(N)]          # one allocation per rank
    _, _, _, u = lay.tables()
    for j, (lo, hi) in enumerate(u):
        got = torch.full((int(hi - lo) + 16,), -1, dtype=torch.int16, device="cuda")
        zs.gather_unit_ranks(lay, j, shards, got)
        torch.cuda.synchronize()
        g = _np(got)
        S.assert_bits_equal(g[:hi - lo], ref.p16_full[lo:hi], f"unit {j}")
        assert (g[hi - lo:] == 0xFFFF).all(), f"unit {j}: write past the unit"


def test_gather_unit_ranks_rejects_bad_arguments():
    lay = zs.Layout([1000] * 65, 65, 3, 0, 8, list(range(65))).to_device()
    shards = [torch.zeros(lay.shard, dtype=torch.int16, device="cuda") for _ in range(65)]
    dst = torch.zeros(1000, dtype=torch.int16, device="cuda")
    for call in (lambda: zs.gather_unit_ranks(lay, 0, shards, dst),          # N > 64
                 lambda: zs.gather_unit_ranks(lay, 65, shards, dst)):         # no such unit
        with pytest.raises(zs.ZeroError) as e:
            call()
        assert e.value.status == 1
    lay4 = zs.Layout([1000] * 4, 4, 3, 0, 8, list(range(4))).to_device()
    s4 = [torch.zeros(lay4.shard + 8, dtype=torch.int16, device="cuda") for _ in range(4)]
    with pytest.raises(zs.ZeroError) as e:
        zs.gather_unit_ranks(lay4, 0, [s4[0][1:]] + s4[1:], dst)              # misaligned shard
    assert e.value.status == 2


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _ipc_worker(rank, world, port, wl, steps, out):
    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import seeded_inputs as si
    import zero_sharded_optimizer_ring_b200 as zs
    from zero_sharded_optimizer_ring_b200.multigpu import RankStep
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=120))
    torch.cuda.set_device(0)
    lay = zs.Layout(list(wl.tensors), world, wl.stage, wl.bucket_elems, wl.pad_align, list(wl.units)).to_device()
    P, S_ = lay.padded, lay.shard
    g_all = si.fill_grads(world, P, wl.psi, wl.seed, wl.grad_sigma, wl.loss_scale)
    master = si.fill_f32(P, wl.psi, wl.seed, si.STREAM_MASTER, wl.master_sigma)
    m = si.fill_f32(P, wl.psi, wl.seed, si.STREAM_M, wl.m_sigma)
    v = si.fill_f32(P, wl.psi, wl.seed, si.STREAM_V, wl.v_sigma, True)
    g = torch.from_numpy(g_all[rank].view(np.int16).copy()).cuda()
    sl = slice(rank * S_, (rank + 1) * S_)
    mk, m1, v1 = (torch.from_numpy(x[sl].copy()).cuda() for x in (master, m, v))
    p16 = torch.zeros(S_ if wl.stage == 3 else P, dtype=torch.int16, device="cuda")   # ZeRO-3: own shard
    torch.cuda.synchronize()
    rs = RankStep(lay, rank, world, g, mk, m1, v1, p16)
    for t in range(1, steps + 1):
        rs.step(zs.AdamW(wl.lr, wl.beta1, wl.beta2, wl.eps, wl.weight_decay, wl.loss_scale, t))
    full = p16
    if wl.stage == 3:                   # every layer from its owners, as a forward pass would
        _, _, _, units = lay.tables()
        full = torch.cat([torch.zeros(int(hi - lo), dtype=torch.int16, device="cuda") for lo, hi in units])
        for j, (lo, hi) in enumerate(units):
            buf = torch.zeros(int(hi - lo), dtype=torch.int16, device="cuda")
            rs.gather_unit(j, buf)
            full[int(lo):int(hi)] = buf
        torch.cuda.synchronize()
        # the same layers through the prefetching schedule over the owners' shards, with its
        # gather width tuned per kind of pass (four forward and four backward passes: an
        # untimed one, one per candidate width, then the chosen width)
        seen = torch.zeros_like(full)
        width = int(max(hi - lo for lo, hi in units))
        pf = rs.prefetch([torch.zeros(width, dtype=torch.int16, device="cuda") for _ in range(2)],
                         torch.cuda.Stream(), torch.cuda.Stream(), candidates=(1, 4), trials=1)

        def layer(unit, buf):
            lo, hi = int(units[unit][0]), int(units[unit][1])
            seen[lo:hi].copy_(buf[:hi - lo])

        for _ in range(4):
            seen.zero_()
            torch.cuda.synchronize()               # the layers write `seen` on the compute stream
            pf.forward(layer)
            pf.backward(layer)
            torch.cuda.synchronize()
            assert torch.equal(seen, full), "prefetched layers differ from the gathered ones"
        assert all(w.chosen is not None for w in pf.widths.values())
    rs.close()
    out.put((rank, mk.cpu().numpy(), m1.cpu().numpy(), v1.cpu().numpy(), full.cpu().numpy().view(np.uint16)))
    dist.destroy_process_group()


@pytest.mark.parametrize("stage,world", [(1, 2), (2, 2), (3, 2), (1, 3), (3, 3)])
def test_process_per_rank_step_over_ipc_matches_oracle(stage, world):
    """One process per rank, all on this GPU: each holds one rank's gradients and one
    shard's state, maps the others' buffers and phase events over CUDA IPC, and steps
    through the fenced phases (no kernel waits on another process).  Every process ends
    with the oracle's shard state and fp16 parameters."""
    wl = Workload(name="ipc", description="ipc", tensors=(100_003, 77_777, 122_227), units=(0, 1, 2),
                  n_ranks=world, stage=stage, bucket_elems=50_001, steps=3, loss_scale=1024.0, m_sigma=1e-4,
                  v_sigma=1e-6, pad_align=8)
    olay = S.oracle_layout(wl)
    g, master, m, v = S.host_inputs(wl, olay.padded)
    ref = oracle.run_steps(olay, stage, g, master, m, v, S.hyper(wl), wl.steps)
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_ipc_worker, args=(r, world, port, wl, wl.steps, q)) for r in range(world)]
    for p in procs:
        p.start()
    try:
        res = sorted([q.get(timeout=300) for _ in range(world)], key=lambda x: x[0])
    finally:
        for p in procs:
            p.join(60)
            if p.exitcode is None:
                p.kill()
    assert all(p.exitcode == 0 for p in procs)
    S_ = olay.shard
    for rank, mk, m1, v1, p16 in res:
        sl = slice(rank * S_, (rank + 1) * S_)
        S.assert_bits_equal(mk, ref.master[sl], f"master shard {rank}")
        S.assert_bits_equal(m1, ref.m[sl], f"m shard {rank}")
        S.assert_bits_equal(v1, ref.v[sl], f"v shard {rank}")
        S.assert_bits_equal(p16, ref.p16_full, f"p16 on rank {rank}")


def _ipc_dyn_worker(rank, world, port, wl, steps, start, out):
    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import seeded_inputs as si
    import zero_sharded_optimizer_ring_b200 as zs
    from zero_sharded_optimizer_ring_b200.multigpu import RankStep
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=120))
    torch.cuda.set_device(0)
    lay = zs.Layout(list(wl.tensors), world, wl.stage, wl.bucket_elems, wl.pad_align, list(wl.units)).to_device()
    P, S_ = lay.padded, lay.shard
    master = si.fill_f32(P, wl.psi, wl.seed, si.STREAM_MASTER, wl.master_sigma)
    m = si.fill_f32(P, wl.psi, wl.seed, si.STREAM_M, wl.m_sigma)
    v = si.fill_f32(P, wl.psi, wl.seed, si.STREAM_V, wl.v_sigma, True)
    sl = slice(rank * S_, (rank + 1) * S_)
    state = [torch.from_numpy(x[sl].copy()).cuda() for x in (master, m, v)]
    spare = [torch.full((S_,), float("nan"), device="cuda") for _ in range(3)]
    n16 = S_ if wl.stage == 3 else P
    p16 = torch.zeros(n16, dtype=torch.int16, device="cuda")
    p16b = torch.zeros(n16, dtype=torch.int16, device="cuda")
    g = torch.zeros(P, dtype=torch.int16, device="cuda")
    nf = torch.zeros(lay.n_buckets, dtype=torch.int32, device="cuda")
    torch.cuda.synchronize()
    rs = RankStep(lay, rank, world, g, *state, p16, spare=(*spare, p16b))
    sc = zs.LossScaler(start, window=3)
    trace = []
    hp = zs.AdamW(wl.lr, wl.beta1, wl.beta2, wl.eps, wl.weight_decay, 1.0, 1)
    for i in range(steps):
        used = sc.scale
        g_all = si.fill_grads(world, P, wl.psi, wl.seed + i, wl.grad_sigma, used)
        g.copy_(torch.from_numpy(g_all[rank].view(np.int16).copy()).cuda())
        torch.cuda.synchronize()
        applied = rs.step_dynamic(hp, sc, nf)
        trace.append((used, not applied, sc.step if applied else 0))
    full = rs.p16
    if wl.stage == 3:
        _, _, _, units = lay.tables()
        full = torch.zeros(P, dtype=torch.int16, device="cuda")
        for j, (lo, hi) in enumerate(units):
            buf = torch.zeros(int(hi - lo), dtype=torch.int16, device="cuda")
            rs.gather_unit(j, buf)
            full[int(lo):int(hi)] = buf
    torch.cuda.synchronize()
    out.put((rank, trace, (sc.scale, sc.clean_steps, sc.step, sc.skipped), [x.cpu().numpy() for x in rs.state],
             full.cpu().numpy().view(np.uint16)))
    rs.close()
    dist.destroy_process_group()


@pytest.mark.parametrize("stage", [1, 2, 3])
def test_two_process_dynamic_commit_matches_oracle(stage):
    """Dynamic loss scaling with one process per rank: both processes take the oracle's
    skip / apply sequence (one shard's overflow skips the step on both) and end with the
    oracle's scaler, state shards and fp16 parameters."""
    wl = Workload(name="ipcdyn", description="ipc dynamic", tensors=(100_003, 77_777, 122_227), units=(0, 1, 2),
                  n_ranks=2, stage=stage, bucket_elems=50_001, steps=8, loss_scale=1.0, m_sigma=1e-4,
                  v_sigma=1e-6, pad_align=8)
    olay = S.oracle_layout(wl)
    P, psi = olay.padded, wl.psi
    _, master, m, v = S.host_inputs(wl, P)
    start = 2.0 ** 24

    def grads_at(scale, i):
        return si.fill_grads(2, P, psi, wl.seed + i, wl.grad_sigma, scale)

    osc = oracle.LossScaler(start, window=3)
    ref, trace = oracle.run_steps_dynamic(olay, stage, grads_at, master, m, v, S.hyper(wl), wl.steps, osc)
    assert any(o for _, o, _ in trace) and not all(o for _, o, _ in trace)
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_ipc_dyn_worker, args=(r, 2, port, wl, wl.steps, start, q)) for r in range(2)]
    for p in procs:
        p.start()
    try:
        res = sorted([q.get(timeout=300) for _ in range(2)], key=lambda x: x[0])
    finally:
        for p in procs:
            p.join(60)
            if p.exitcode is None:
                p.kill()
    assert all(p.exitcode == 0 for p in procs)
    S_ = olay.shard
    for rank, got_trace, scaler, (mk, m1, v1), p16 in res:
        assert got_trace == trace
        assert scaler == (osc.scale, osc.clean_steps, osc.step, osc.skipped)
        sl = slice(rank * S_, (rank + 1) * S_)
        S.assert_bits_equal(mk, ref.master[sl], f"master shard {rank}")
        S.assert_bits_equal(m1, ref.m[sl], f"m shard {rank}")
        S.assert_bits_equal(v1, ref.v[sl], f"v shard {rank}")
        S.assert_bits_equal(p16, ref.p16_full, f"p16 on rank {rank}")
