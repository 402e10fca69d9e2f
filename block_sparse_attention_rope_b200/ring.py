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
is kept, and after the last step the rank's partial results are combined by
log-sum-exp in one pass (lc_bsa_lse_merge_parts); a step whose K/V shard
holds no block the rank's queries attend is skipped (its K/V still travels
on).

The schedule and the exchange are plain host logic; the compute steps are
passed in, so the same ring runs on the GPU library (``GpuRingRank``) or, in
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
    """Send to ring neighbour `dst`, receive from `src` (ranks within `group`,
    None = the default group), as one batched group of point-to-point ops."""
    import torch.distributed as dist
    if group is not None:
        dst, src = dist.get_global_rank(group, dst), dist.get_global_rank(group, src)
    ops = [dist.P2POp(dist.isend, t, dst, group) for t in send]
    ops += [dist.P2POp(dist.irecv, t, src, group) for t in recv]
    return dist.batch_isend_irecv(ops)


def ring_forward(sched: RingSchedule, q: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
                 partial: Callable, combine: Callable, group=None,
                 fetch: Optional[Callable] = None):
    """Run the ring for one rank.

    q, k, v: this rank's shard [B, n_rank, heads, hd].
    partial(src, q, k_src, v_src, slot): the attention over shard src's keys
      (slot counts the computing steps from 0); its results are collected.
    combine(results): the rank's result from the collected partial results.
    fetch(src) -> (k_src, v_src): instead of the NCCL exchange, take shard src
      directly (one process standing in for every rank).
    """
    world, rank = sched.world, sched.rank
    cur_k, cur_v = k, v
    parts = []
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
            parts.append(partial(src, q, cur_k, cur_v, len(parts)))
        for r in reqs:
            r.wait()
        cur_k, cur_v = nxt_k, nxt_v
    return combine(parts)


class GpuRingRank:
    """One rank of the ring on the GPU library: its shard plans (one per K/V
    shard its queries attend), the buffers of its partial results, and the
    steps.  The rank rotates its own q and k once (lc_rope3d_apply_ex, with
    the RMSNorm if given); the rotated K shard is what travels, so no step
    rotates again.  Partial results stay in one buffer until the last step
    and are combined in one pass (lc_bsa_lse_merge_parts)."""

    def __init__(self, api, T: int, H: int, W: int, *, local: int, stride: int, n_cond: int,
                 shards: Sequence[Tuple[int, int]], rank: int, rope, batch: int, heads: int,
                 dtype=torch.bfloat16, device="cuda", softmax_scale: float = 0.0,
                 q_norm=None, k_norm=None, norm_eps: float = 1e-6):
        self.api, self.rope = api, rope
        self.q_norm, self.k_norm, self.norm_eps = q_norm, k_norm, norm_eps
        self.softmax_scale = softmax_scale
        full = api.Plan(T, H, W, local=local, stride=stride, n_cond=n_cond)
        Cb, N, Nc = full.info().num_cond_blocks, full.n_tokens, full.n_cond_tokens
        self.plans = {}
        for src in range(len(shards)):
            p = api.Plan(T, H, W, local=local, stride=stride, n_cond=n_cond,
                         q_blocks=shards[rank], k_blocks=shards[src])
            if p.info().nnz > 0:
                self.plans[src] = p
        self.sched = RingSchedule(shards, Nc, Cb, N, rank, lambda r, src: src in self.plans)
        nq = self.sched.n_tokens(rank)
        n_parts = sum(self.sched.computes)
        self.parts = torch.empty(n_parts, batch, nq, heads, 64, dtype=dtype, device=device)
        self.lses = torch.empty(n_parts, batch, heads, nq, dtype=torch.float32, device=device)

    def rotate(self, x: torch.Tensor, shard: int, norm) -> torch.Tensor:
        """R(norm(x)) of shard `shard`'s tokens at their sequence positions."""
        return self.rope.apply(x, tok_offset=self.sched.tokens[shard][0], norm=norm,
                               norm_eps=self.norm_eps)

    def partial(self, src, q_rot, k_rot, v, slot):
        self.api.forward_shard(q_rot, k_rot, v, self.plans[src], self.rope, out=self.parts[slot],
                               lse=self.lses[slot], softmax_scale=self.softmax_scale,
                               q_rotated=True, k_rotated=True)
        return slot

    def combine(self, slots):
        n = len(slots)
        if n == 1:
            return self.parts[0], self.lses[0]
        return self.api.lse_merge_parts(self.parts[:n], self.lses[:n])

    def forward(self, q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, group=None,
                fetch: Optional[Callable] = None):
        """This rank's attention output and lse over the whole sequence.  q, k,
        v: the rank's own shard, pre-RoPE.  With `fetch(src) -> (R(norm(k_src)),
        v_src)` the K/V shards are taken from it instead of the ring exchange."""
        r = self.sched.rank
        q_rot = self.rotate(q, r, self.q_norm)
        k_rot = self.rotate(k, r, self.k_norm)
        return ring_forward(self.sched, q_rot, k_rot, v, self.partial, self.combine, group, fetch)
