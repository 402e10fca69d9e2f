"""Ring context parallelism for block-sparse 3D-RoPE attention.

myzaker / QbitAI "美团视频生成模型来了！一出手就是开源 SOTA", section
"背后技术原理": the high-resolution pass pairs block-sparse attention with
context-parallel ring block-sparse attention.  Here: the sequence's blocks are
cut into contiguous shards, one per rank (query bounds on 4-block group
edges, balanced by the plan's per-block work); a rank keeps its query shard,
and at step s holds the K/V shard of rank (r - s) mod world, which it passes
on to rank r + 1 while it computes (NCCL send/recv over NVLink, one
batched group per step, on the communicator's own stream so the transfer
overlaps the attention).  Each step's partial result (lc_bsa_forward_shard)
is folded into the rank's running result by log-sum-exp (lc_bsa_lse_merge);
a step whose K/V shard holds no block the rank's queries attend is skipped
(its K/V still travels on).

The schedule and the exchange are plain host logic; the compute steps are
passed in, so the same ring runs on the GPU library (``gpu_steps``) or, in
tests, on anything with the same shape contract.
"""
from __future__ import annotations

from typing import Callable, List, Optional, Sequence, Tuple

import torch


def group_edges(Cb: int, Nb: int) -> List[int]:
    """Block indices where a shard of query blocks may start or end: the
    4-block group boundaries of the condition and noisy segments."""
    nq = Cb + Nb
    e = set(range(0, Cb, 4)) | {Cb} | set(range(Cb, nq, 4)) | {nq}
    return sorted(e)


def balanced_shards(work: Sequence[int], Cb: int, world: int) -> List[Tuple[int, int]]:
    """Cut blocks 0..len(work) into `world` contiguous ranges at group edges,
    each as close as possible to an equal share of the total work (work[r]:
    key blocks query block r attends).  Raises if there are fewer edges than
    ranks."""
    nq = len(work)
    edges = group_edges(Cb, nq - Cb)
    if len(edges) - 1 < world:
        raise ValueError("%d query groups cannot be split over %d ranks" % (len(edges) - 1, world))
    pre = [0]
    for w in work:
        pre.append(pre[-1] + int(w))
    total = pre[-1]
    cuts = [0]
    for i in range(1, world):
        target = total * i / world
        lo = edges.index(cuts[-1]) + 1
        hi = len(edges) - 1 - (world - i)  # leave one edge per remaining rank
        best = min(range(lo, hi + 1), key=lambda j: abs(pre[edges[j]] - target))
        cuts.append(edges[best])
    cuts.append(nq)
    return [(cuts[i], cuts[i + 1]) for i in range(world)]


def block_token(r: int, Nc: int, Cb: int, N: int, block: int = 64) -> int:
    """First token of block r in the whole sequence (r == block count: N)."""
    return min(block * r if r < Cb else Nc + block * (r - Cb), N)


class RingSchedule:
    """One rank's view of the ring: the shards' token ranges, which shard it
    holds at each step, and which steps compute."""

    def __init__(self, shards: Sequence[Tuple[int, int]], Nc: int, Cb: int, N: int, rank: int,
                 active: Callable[[int, int], bool], block: int = 64):
        self.shards = list(shards)
        self.world = len(self.shards)
        self.rank = rank
        self.tokens = [(block_token(a, Nc, Cb, N, block), block_token(b, Nc, Cb, N, block))
                       for a, b in self.shards]
        self.sources = [(rank - s) % self.world for s in range(self.world)]
        self.computes = [bool(active(rank, src)) for src in self.sources]
        if not any(self.computes):
            raise ValueError("rank %d attends no key shard" % rank)
        self.last = max(s for s, c in enumerate(self.computes) if c)

    def n_tokens(self, shard: int) -> int:
        a, b = self.tokens[shard]
        return b - a


def _exchange(send: Sequence[torch.Tensor], recv: Sequence[torch.Tensor], dst: int, src: int,
              group) -> list:
    import torch.distributed as dist
    ops = [dist.P2POp(dist.isend, t, dst, group) for t in send]
    ops += [dist.P2POp(dist.irecv, t, src, group) for t in recv]
    return dist.batch_isend_irecv(ops)


def ring_forward(sched: RingSchedule, q: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
                 partial: Callable, merge: Callable, group=None, fetch: Optional[Callable] = None):
    """Run the ring for one rank.

    q, k, v: this rank's shard [B, n_rank, heads, hd].
    partial(src, q, k_src, v_src) -> (o, lse): attention over shard src's keys.
    merge(acc, part, first, last) -> acc: fold a part in; the value returned
      after the last computing step is the result.
    fetch(src) -> (k_src, v_src): instead of the NCCL exchange, take shard src
      directly (one process standing in for every rank).
    """
    world, rank = sched.world, sched.rank
    cur_k, cur_v = k, v
    acc = None
    first = True
    for s in range(world):
        src = sched.sources[s]
        reqs = []
        nxt_k = nxt_v = None
        if s + 1 < world:
            if fetch is not None:
                nxt_k, nxt_v = fetch(sched.sources[s + 1])
            else:
                n = sched.n_tokens(sched.sources[s + 1])
                shape = (k.shape[0], n) + tuple(k.shape[2:])
                nxt_k = torch.empty(shape, dtype=k.dtype, device=k.device)
                nxt_v = torch.empty(shape, dtype=v.dtype, device=v.device)
                reqs = _exchange((cur_k, cur_v), (nxt_k, nxt_v), (rank + 1) % world,
                                 (rank - 1) % world, group)
        if sched.computes[s]:
            part = partial(src, q, cur_k, cur_v)
            acc = merge(acc, part, first, s == sched.last)
            first = False
        for r in reqs:
            r.wait()
        cur_k, cur_v = nxt_k, nxt_v
    return acc


def gpu_steps(api, T: int, H: int, W: int, *, local: int, stride: int, n_cond: int,
              shards: Sequence[Tuple[int, int]], rank: int, rope, softmax_scale: float = 0.0,
              q_norm=None, k_norm=None, norm_eps: float = 1e-6):
    """Shard plans of one rank (one per K/V shard it attends) and the partial
    / merge steps on the GPU library.  Returns (schedule, partial, merge)."""
    full = api.Plan(T, H, W, local=local, stride=stride, n_cond=n_cond)
    inf = full.info()
    Cb, N, Nc = inf.num_cond_blocks, full.n_tokens, full.n_cond_tokens
    plans = {}
    for src in range(len(shards)):
        p = api.Plan(T, H, W, local=local, stride=stride, n_cond=n_cond, q_blocks=shards[rank],
                     k_blocks=shards[src])
        if p.info().nnz > 0:
            plans[src] = p
    sched = RingSchedule(shards, Nc, Cb, N, rank, lambda r, src: src in plans)
    kw = dict(softmax_scale=softmax_scale, q_norm=q_norm, k_norm=k_norm, norm_eps=norm_eps)

    def partial(src, q, k_src, v_src):
        return api.forward_shard(q, k_src, v_src, plans[src], rope, **kw)

    def merge(acc, part, first, last):
        o_p, l_p = part
        if first and last:
            return o_p, l_p
        if first:
            o_acc = torch.empty(o_p.shape, dtype=torch.float32, device=o_p.device)
            l_acc = torch.empty_like(l_p)
            api.lse_merge(o_acc, l_acc, o_p, l_p, init=True)
            return o_acc, l_acc
        o_acc, l_acc = acc
        if last:
            out = torch.empty_like(o_p)
            api.lse_merge(o_acc, l_acc, o_p, l_p, out=out)
            return out, l_acc
        api.lse_merge(o_acc, l_acc, o_p, l_p)
        return o_acc, l_acc

    sched.plans = plans
    return sched, partial, merge
