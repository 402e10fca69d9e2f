"""The ring driver's host logic on CPU: shard cutting, the per-rank schedule,
and the K/V exchange over gloo (world sizes 2 and 3), with the oracle's fp64
partial attention and merge standing in for the GPU steps.  The result of
every rank must equal the oracle's whole-sequence forward on its rows."""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
from oracle import ring as orng
from oracle.backward import token_mask
from block_sparse_attention_rope_b200 import ring

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

GEOM = dict(T=5, H=8, W=40, n_cond=2, local=1, stride=2)   # Cb 10, Nb 15


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _work():
    rp, _ = oracle.block_csr(GEOM["T"], GEOM["H"], GEOM["W"], 64, GEOM["local"],
                             GEOM["stride"], GEOM["n_cond"])
    return np.diff(rp)


def _inputs():
    N = GEOM["T"] * GEOM["H"] * GEOM["W"]
    rng = np.random.default_rng(11)
    return [rng.standard_normal((1, N, 2, 64)) for _ in range(3)]


def _schedule(shards, rank):
    Nc, Nn, Cb, Nb = oracle.segment_sizes(GEOM["T"], GEOM["H"], GEOM["W"], GEOM["n_cond"])
    N = Nc + Nn
    toks = orng.shard_tokens(shards, GEOM["T"], GEOM["H"], GEOM["W"], GEOM["n_cond"])

    def active(r, src):
        (qa, qb), (ka, kb) = toks[r], toks[src]
        return token_mask(N, Nc, 64, GEOM["local"], GEOM["stride"], rows=np.arange(qa, qb),
                          cols=np.arange(ka, kb)).any()
    return ring.RingSchedule(shards, Nc, Cb, N, rank, active)


def _oracle_steps(sched):
    geo = {k: GEOM[k] for k in ("T", "H", "W", "n_cond", "local", "stride")}

    def partial(src, q, k, v, slot):
        return orng.partial_attention(q.numpy(), k.numpy(), v.numpy(),
                                      q_tokens=sched.tokens[sched.rank],
                                      k_tokens=sched.tokens[src], **geo)

    def combine(parts):
        o, l = parts[0]
        for po, pl in parts[1:]:
            o, l = orng.lse_merge(o, l, po, pl)
        return torch.from_numpy(o), torch.from_numpy(l)
    return partial, combine


def _worker(rank, world, port, shards, qout):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        q, k, v = (torch.from_numpy(a) for a in _inputs())
        sched = _schedule(shards, rank)
        a, b = sched.tokens[rank]
        partial, combine = _oracle_steps(sched)
        o, l = ring.ring_forward(sched, q[:, a:b].contiguous(), k[:, a:b].contiguous(),
                                 v[:, a:b].contiguous(), partial, combine)
        qout.put((rank, a, b, o.numpy(), l.numpy(), sched.computes))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_ring_over_gloo_matches_whole_sequence(world):
    shards = ring.balanced_shards(_work(), 10, world)
    ctx = mp.get_context("spawn")
    qout = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, shards, qout))
             for r in range(world)]
    for p in procs:
        p.start()
    res = sorted((qout.get(timeout=300) for _ in range(world)), key=lambda r: r[0])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    q, k, v = _inputs()
    ref_o, ref_l = oracle.forward(q, k, v, **GEOM)
    assert res[0][1] == 0 and res[-1][2] == q.shape[1]
    for rank, a, b, o, l, computes in res:
        assert np.abs(o - ref_o[:, a:b]).max() <= 1e-12 * np.abs(ref_o).max()
        assert np.abs(l - ref_l[:, :, a:b]).max() <= 1e-12 * np.abs(ref_l).max()
        assert computes[0]  # a rank always attends its own shard


def test_balanced_shards_cut_on_group_edges():
    work = _work()
    Cb = 10
    edges = set(ring.group_edges(Cb, len(work) - Cb))
    assert sorted(edges) == [0, 4, 8, 10, 14, 18, 22, 25]
    for world in range(1, len(edges)):
        sh = ring.balanced_shards(work, Cb, world)
        assert sh[0][0] == 0 and sh[-1][1] == len(work)
        assert all(a < b and a in edges and b in edges for a, b in sh)
        assert all(sh[i][1] == sh[i + 1][0] for i in range(world - 1))
    with pytest.raises(ValueError):
        ring.balanced_shards(work, Cb, len(edges))
    # balance: the I2V 480p pattern over 8 ranks is within one group's work of even
    rp, _ = oracle.block_csr(24, 30, 52, 64, 2, 4, 1)
    w = np.diff(rp)
    sh = ring.balanced_shards(w, 25, 8)
    per = [int(w[a:b].sum()) for a, b in sh]
    assert max(per) - min(per) <= 2 * 4 * int(w.max())


def test_schedule_sources_and_skips():
    shards = [(0, 4), (4, 10), (10, 18), (18, 25)]
    s0 = _schedule(shards, 0)
    assert s0.sources == [0, 3, 2, 1]
    # rank 0 holds condition blocks only: noisy-only key shards are skipped
    assert s0.computes == [True, False, False, True]
    s2 = _schedule(shards, 2)
    assert s2.sources == [2, 1, 0, 3] and all(s2.computes)
    assert s0.tokens[1] == (256, 640) and s0.tokens[2] == (640, 1152)


def _worker_subgroup(rank, world, port, shards, qout):
    """Ranks 0 and 2 of three form the ring (a process subgroup); rank 1 only
    takes part in creating the group."""
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        group = dist.new_group([0, 2])
        if rank == 1:
            qout.put(None)
            return
        grank = dist.get_rank(group)
        q, k, v = (torch.from_numpy(a) for a in _inputs())
        sched = _schedule(shards, grank)
        a, b = sched.tokens[grank]
        partial, combine = _oracle_steps(sched)
        o, l = ring.ring_forward(sched, q[:, a:b].contiguous(), k[:, a:b].contiguous(),
                                 v[:, a:b].contiguous(), partial, combine, group=group)
        qout.put((grank, a, b, o.numpy(), l.numpy()))
    finally:
        dist.destroy_process_group()


def test_ring_over_a_process_subgroup():
    shards = ring.balanced_shards(_work(), 10, 2)
    ctx = mp.get_context("spawn")
    qout = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker_subgroup, args=(r, 3, port, shards, qout))
             for r in range(3)]
    for p in procs:
        p.start()
    res = [qout.get(timeout=300) for _ in range(3)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    res = sorted((r for r in res if r is not None), key=lambda r: r[0])
    assert len(res) == 2
    q, k, v = _inputs()
    ref_o, ref_l = oracle.forward(q, k, v, **GEOM)
    for grank, a, b, o, l in res:
        assert np.abs(o - ref_o[:, a:b]).max() <= 1e-12 * np.abs(ref_o).max()
        assert np.abs(l - ref_l[:, :, a:b]).max() <= 1e-12 * np.abs(ref_l).max()


def test_planned_shards_model():
    """The shard planner: a valid layout on group edges whose modeled slowest
    rank is no worse than the even-work layout's; the model sees the wave
    step when a shard's items per step pass a multiple of the SM count."""
    rp, ci = oracle.block_csr(24, 30, 52, 64, 2, 4, 1)     # I2V 480p: Cb 25, Nb 561
    edges = set(ring.group_edges(25, 561))
    even = ring.balanced_shards(ring.block_work(np.diff(rp), 25), 25, 8)
    planned = ring.planned_shards(rp, ci, 25, 8, heads=32)
    assert planned[0][0] == 0 and planned[-1][1] == 586
    assert all(a < b and a in edges and b in edges for a, b in planned)
    assert all(planned[i][1] == planned[i + 1][0] for i in range(7))
    t_even = ring.modeled_rank_cycles(even, rp, ci, 25, 32)
    t_plan = ring.modeled_rank_cycles(planned, rp, ci, 25, 32)
    assert max(t_plan) <= max(t_even)
    # 18 noisy groups x 32 heads = 576 items fill 148 SMs in 4 waves, 19 need 5
    lay18 = [(0, 25), (25, 97), (97, 586)]
    lay19 = [(0, 25), (25, 101), (101, 586)]
    t18 = ring.modeled_rank_cycles(lay18, rp, ci, 25, 32)[1]
    t19 = ring.modeled_rank_cycles(lay19, rp, ci, 25, 32)[1]
    assert t19 > t18 * 1.1


def test_shard_layouts_on_random_geometries():
    """Seeded random geometries and rank counts: the even-work and the planned
    layouts both cover the blocks with contiguous ranges on group edges, and
    the planned one is never worse under the model."""
    rng = np.random.default_rng(7)
    for _ in range(12):
        T = int(rng.integers(2, 6))
        H, W = int(rng.integers(4, 12)), int(rng.integers(16, 48))
        n_cond = int(rng.integers(0, T - 1))
        local, stride = int(rng.integers(0, 3)), int(rng.integers(0, 6))
        Nc, Nn, Cb, Nb = oracle.segment_sizes(T, H, W, n_cond)
        rp, ci = oracle.block_csr(T, H, W, 64, local, stride, n_cond)
        edges = ring.group_edges(Cb, Nb)
        for world in (1, 2, 3):
            if len(edges) - 1 < world:
                continue
            even = ring.balanced_shards(ring.block_work(np.diff(rp), Cb), Cb, world)
            plan = ring.planned_shards(rp, ci, Cb, world, heads=4, n_sm=8)
            for sh in (even, plan):
                assert sh[0][0] == 0 and sh[-1][1] == Cb + Nb and len(sh) == world
                assert all(a < b and a in edges and b in edges for a, b in sh)
                assert all(sh[i][1] == sh[i + 1][0] for i in range(world - 1))
            te = ring.modeled_rank_cycles(even, rp, ci, Cb, 4, n_sm=8)
            tp = ring.modeled_rank_cycles(plan, rp, ci, Cb, 4, n_sm=8)
            assert max(tp) <= max(te) + 1e-6
