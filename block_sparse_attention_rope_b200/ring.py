"""Ring context parallelism for block-sparse 3D-RoPE attention.

myzaker / QbitAI "美团视频生成模型来了！一出手就是开源 SOTA", section
"背后技术原理": the high-resolution pass pairs block-sparse attention with
context-parallel ring block-sparse attention.  Here: the sequence's blocks are
cut into contiguous shards, one per rank (query bounds on 4-block group
edges; `planned_shards` picks the cuts with a model of the kernel's work
items, which fill the SMs in whole waves); a rank keeps its query shard,
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
    pre = [0.0]
    for w in work:
        pre.append(pre[-1] + float(w))
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


# Cost of a query block in the tensor-core kernel, in units of its CSR
# entries: a work item (4 query blocks) costs about 8,500 cycles beyond its
# key tiles (3,070 cycles per 2-block tile for both query tiles), i.e. about
# 5.5 entries per block (least-squares fit over the sparsity sweep on B200).
ITEM_OVERHEAD_ENTRIES = 5.5


def block_work(row_counts: Sequence[int], num_cond_blocks: int = 0) -> List[float]:
    """Per query block: its CSR entries plus its share of the per-item cost,
    the work measure `balanced_shards` splits evenly."""
    return [float(c) + ITEM_OVERHEAD_ENTRIES for c in row_counts]


def block_token(r: int, Nc: int, Cb: int, N: int, block: int = 64) -> int:
    """First token of block r in the whole sequence (r == block count: N)."""
    return min(block * r if r < Cb else Nc + block * (r - Cb), N)


# Cycles of one work item of the tensor-core kernel beyond its key tiles, and
# of one 2-block key tile (both query tiles), from a least-squares fit over
# the sparsity sweep on B200; used only to compare shard layouts.
ITEM_CYCLES = 8500.0
TILE_CYCLES = 3070.0
STEP_CYCLES = 30000.0  # per computing step: launch and kernel ramp (ring measurements)


def _group_unions(row_ptr: Sequence[int], col_idx: Sequence[int], Cb: int):
    """Per work item group (4 query blocks of one segment): first block and
    the sorted union of its members' key blocks."""
    nq = len(row_ptr) - 1
    out = []
    for seg_lo, seg_hi in ((0, Cb), (Cb, nq)):
        for g0 in range(seg_lo, seg_hi, 4):
            u = set()
            for r in range(g0, min(g0 + 4, seg_hi)):
                u.update(int(c) for c in col_idx[row_ptr[r]:row_ptr[r + 1]])
            out.append((g0, sorted(u)))
    return out


def _makespan(costs: List[float], n_sm: int) -> float:
    """Finish time of items taken in order by n_sm persistent CTAs, each CTA
    taking the next item as soon as it is free (the kernel's atomic queue)."""
    import heapq
    if not costs:
        return 0.0
    free = [0.0] * min(n_sm, len(costs))
    heapq.heapify(free)
    end = 0.0
    for c in costs:
        t = heapq.heappop(free) + c
        end = max(end, t)
        heapq.heappush(free, t)
    return end


def modeled_rank_cycles(shards: Sequence[Tuple[int, int]], row_ptr: Sequence[int],
                        col_idx: Sequence[int], Cb: int, heads: int, batch: int = 1,
                        n_sm: int = 148, unions=None, cache=None) -> List[float]:
    """Modeled device cycles of each rank's ring: per step, the makespan of
    the step's work items (one per batch entry, head and active group; cost =
    ITEM_CYCLES + TILE_CYCLES x key tiles in the source shard, longest first,
    head-major, as the kernel orders them) on n_sm CTAs."""
    import bisect
    import math
    unions = unions if unions is not None else _group_unions(row_ptr, col_idx, Cb)
    out = []
    cache = {} if cache is None else cache
    for r, (qa, qb) in enumerate(shards):
        groups = None
        total = 0.0
        for ka, kb in shards:
            key = (qa, qb, ka, kb)
            if key not in cache:
                if groups is None:
                    groups = [u for g0, u in unions if qa <= g0 < qb]
                tiles = [math.ceil((bisect.bisect_left(u, kb) - bisect.bisect_left(u, ka)) / 2)
                         for u in groups]
                lens = sorted((t for t in tiles if t > 0), reverse=True)
                costs = [ITEM_CYCLES + TILE_CYCLES * t for t in lens] * (heads * batch)
                cache[key] = _makespan(costs, n_sm) + STEP_CYCLES if lens else 0.0
            total += cache[key]
        out.append(total)
    return out


def planned_shards(row_ptr: Sequence[int], col_idx: Sequence[int], Cb: int, world: int,
                   heads: int, batch: int = 1, n_sm: int = 148,
                   max_rounds: int = 8) -> List[Tuple[int, int]]:
    """Shard layout for the ring that minimises the slowest rank's modeled
    time (modeled_rank_cycles): start from the layout even in work, then take
    the best move of a run of consecutive cuts by one or two group edges,
    while the slowest rank (then the total) improves.  The model captures what an even
    split of work misses: each step's items fill the SMs in whole waves."""
    nq = len(row_ptr) - 1
    counts = [row_ptr[r + 1] - row_ptr[r] for r in range(nq)]
    shards = balanced_shards(block_work(counts, Cb), Cb, world)
    if world == 1:
        return shards
    unions = _group_unions(row_ptr, col_idx, Cb)
    edges = group_edges(Cb, nq - Cb)
    pos = {e: k for k, e in enumerate(edges)}
    cuts = [pos[a] for a, _ in shards[1:]]  # as edge indices

    def layout(c):
        b = [0] + [edges[k] for k in c] + [nq]
        return [(b[i], b[i + 1]) for i in range(len(b) - 1)]

    cache = {}

    def cost(c):
        t = modeled_rank_cycles(layout(c), row_ptr, col_idx, Cb, heads, batch, n_sm, unions,
                                cache)
        return max(t), sum(t)

    best = cost(cuts)
    for _ in range(max_rounds):
        cand_best, cand = best, None
        for i in range(len(cuts)):
            for j in range(i, len(cuts)):
                for d in (-2, -1, 1, 2):
                    c = cuts[:i] + [k + d for k in cuts[i:j + 1]] + cuts[j + 1:]
                    if c[0] < 1 or c[-1] > len(edges) - 2 or any(
                            c[m] >= c[m + 1] for m in range(len(c) - 1)):
                        continue
                    cc = cost(c)
                    if cc < cand_best:
                        cand_best, cand = cc, c
        if cand is None:
            break
        best, cuts = cand_best, cand
    return layout(cuts)


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
        # Rows that a step's shard gives no key stay (0, -inf) from here on:
        # each slot always holds the same step, so the launches skip them.
        self.parts = torch.zeros(n_parts, batch, nq, heads, 64, dtype=dtype, device=device)
        self.lses = torch.full((n_parts, batch, heads, nq), -float("inf"), dtype=torch.float32,
                               device=device)

    def rotate(self, x: torch.Tensor, shard: int, norm) -> torch.Tensor:
        """R(norm(x)) of shard `shard`'s tokens at their sequence positions."""
        return self.rope.apply(x, tok_offset=self.sched.tokens[shard][0], norm=norm,
                               norm_eps=self.norm_eps)

    def partial(self, src, q_rot, k_rot, v, slot):
        # Steps after the rank's first write their own slot and read inputs
        # that were complete before the first step: each may start on the SMs
        # the previous step's kernel frees while its last items finish.
        self.api.forward_shard(q_rot, k_rot, v, self.plans[src], self.rope, out=self.parts[slot],
                               lse=self.lses[slot], softmax_scale=self.softmax_scale,
                               q_rotated=True, k_rotated=True, keep_empty_rows=True,
                               overlap_previous=slot > 0)
        return slot

    def combine(self, slots):
        """The rank's result, always in fresh tensors (the partial buffers are
        reused by the next forward, so a one-step result is copied out)."""
        n = len(slots)
        if n == 1:
            return self.parts[0].clone(), self.lses[0].clone()
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
