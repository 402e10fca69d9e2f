"""The benchmark's multi-rank logic on CPU with gloo (world size 2): the
step time is the max over ranks, every rank draws a different batch element,
and only rank 0 prints a line for the reference arm.  No GPU needed."""
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import bench
    from block_sparse_attention_rope_b200 import synthetic
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w_, r_, l_ = bench.dist_env()
        got = bench.max_over_ranks(1.5 + rank, dist, device="cpu")
        w = synthetic.get("tiny_f32")
        x = synthetic.make_inputs(w, seed_offset=bench.rank_seed_offset(rank))
        q.put((rank, w_, r_, l_, got, float(x["q"].sum())))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_per_rank_inputs_with_gloo():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [r[1:4] for r in res] == [(2, 0, 0), (2, 1, 1)]
    assert all(r[4] == 2.5 for r in res)            # max over ranks of 1.5 + rank
    assert res[0][5] != res[1][5]                    # different batch element per rank


def test_reference_arm_prints_only_on_rank_zero():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "1", "--warmup", "0"], env=env, capture_output=True,
                       text=True, timeout=300)
    assert r.returncode == 0 and r.stdout.strip() == ""


def test_max_over_ranks_without_group_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.25, None) == 3.25
