"""fp64 oracle of ring context parallelism: partial attention over one key
shard, the log-sum-exp merge, and the ring as a whole.

TEST INFRASTRUCTURE ONLY (see the package docstring): the library never
imports it.

Source: myzaker / QbitAI "美团视频生成模型来了！一出手就是开源 SOTA",
section "背后技术原理": the high-resolution pass combines block-sparse
attention with context-parallel ring block-sparse attention.  The pages say
no more.  Readings (the plainest ones the rest supports):
  - the sequence's blocks (condition blocks, then noisy blocks, 64 tokens
    each) are cut into contiguous shards, one per rank; a rank keeps its query
    shard and the K/V shards pass around the ring, so at step s rank r holds
    the K/V shard of rank (r - s) mod world;
  - each step computes the masked attention of the rank's queries over the
    keys it holds, as a normalised output o and its log-sum-exp lse (0 and
    -inf for a row with no attended key there), and folds it into the running
    result by log-sum-exp;
  - a step whose K/V shard holds no key block the rank's query blocks attend
    computes nothing ("block-sparse" ring).
The merge of results over a partition of the keys is exactly the attention
over all of them: with l = log sum_k e^{s_k} over each part,
    o = sum_parts e^{l_part - L} o_part,   L = log sum_parts e^{l_part}.
"""
from __future__ import annotations

from typing import List, Optional, Sequence, Tuple

import numpy as np

from . import _f64, rms_norm, rope3d_apply, segment_sizes
from .backward import token_mask


def block_token(r: int, Nc: int, Cb: int, N: int, block: int = 64) -> int:
    """First token of block r (condition blocks, then noisy ones); r == Cb + Nb: N."""
    t = block * r if r < Cb else Nc + block * (r - Cb)
    return min(t, N)


def partial_attention(q, k, v, *, T: int, H: int, W: int, n_cond: int, block: int = 64,
                      local: int, stride: int, q_tokens: Tuple[int, int],
                      k_tokens: Tuple[int, int], scale: Optional[float] = None,
                      q_norm=None, k_norm=None, norm_eps: float = 1e-6):
    """Attention of the queries q (tokens q_tokens of the sequence) over the
    keys k, v (tokens k_tokens) only, under the block pattern.  q: [B, nq,
    heads, hd], k / v: [B, nk, heads, hd], pre-RoPE.  Returns o [B, nq, heads,
    hd] and lse [B, heads, nq] (natural log); rows with no attended key: o = 0,
    lse = -inf."""
    qf, kf, vf = _f64(q), _f64(k), _f64(v)
    B, nq, heads, hd = qf.shape
    N = T * H * W
    Nc = n_cond * H * W
    assert nq == q_tokens[1] - q_tokens[0] and kf.shape[1] == k_tokens[1] - k_tokens[0]
    if q_norm is not None:
        qf = rms_norm(qf, q_norm, norm_eps)
    if k_norm is not None:
        kf = rms_norm(kf, k_norm, norm_eps)
    qr = rope3d_apply(qf, H, W, q_tokens[0])
    kr = rope3d_apply(kf, H, W, k_tokens[0])
    if scale is None:
        scale = 1.0 / np.sqrt(hd)
    mask = token_mask(N, Nc, block, local, stride, rows=np.arange(*q_tokens),
                      cols=np.arange(*k_tokens))
    o = np.zeros((B, nq, heads, hd))
    lse = np.full((B, heads, nq), -np.inf)
    for b in range(B):
        for h in range(heads):
            s = scale * (qr[b, :, h] @ kr[b, :, h].T)
            s = np.where(mask, s, -np.inf)
            m = s.max(axis=1, initial=-np.inf)
            has = np.isfinite(m)
            p = np.zeros_like(s)
            p[has] = np.exp(s[has] - m[has, None])
            l = p.sum(axis=1)
            o[b, has, h] = (p[has] @ vf[b, :, h]) / l[has, None]
            lse[b, h, has] = m[has] + np.log(l[has])
    return o, lse


def lse_merge(o_a, l_a, o_b, l_b):
    """Combine two results over disjoint key sets: o [B, n, heads, hd],
    l [B, heads, n].  A row with both lse -inf stays (0, -inf)."""
    o_a, o_b = np.asarray(o_a, np.float64), np.asarray(o_b, np.float64)
    l_a, l_b = np.asarray(l_a, np.float64), np.asarray(l_b, np.float64)
    m = np.maximum(l_a, l_b)
    fin = np.isfinite(m)
    ms = np.where(fin, m, 0.0)
    w_a = np.where(fin, np.exp(l_a - ms), 0.0)
    w_b = np.where(fin, np.exp(l_b - ms), 0.0)
    tot = w_a + w_b
    l = np.where(fin, ms + np.log(np.where(fin, tot, 1.0)), -np.inf)
    # weights [B, heads, n] -> [B, n, heads, 1]
    c_a = np.where(fin, w_a / np.where(fin, tot, 1.0), 0.0).transpose(0, 2, 1)[..., None]
    c_b = np.where(fin, w_b / np.where(fin, tot, 1.0), 0.0).transpose(0, 2, 1)[..., None]
    o = c_a * o_a + c_b * o_b
    return o, l


def shard_tokens(shards: Sequence[Tuple[int, int]], T: int, H: int, W: int, n_cond: int,
                 block: int = 64) -> List[Tuple[int, int]]:
    """Token range of each block range."""
    Nc, Nn, Cb, Nb = segment_sizes(T, H, W, n_cond, block)
    N = Nc + Nn
    return [(block_token(lo, Nc, Cb, N, block), block_token(hi, Nc, Cb, N, block))
            for lo, hi in shards]


def ring_forward(q, k, v, shards: Sequence[Tuple[int, int]], *, T: int, H: int, W: int,
                 n_cond: int, block: int = 64, local: int, stride: int,
                 scale: Optional[float] = None, q_norm=None, k_norm=None,
                 norm_eps: float = 1e-6):
    """The whole ring, rank by rank and step by step in ring order, on the
    full tensors q, k, v [B, N, heads, hd].  Returns (out, lse) over the whole
    sequence and the list of (rank, step, source shard, attended pairs)."""
    toks = shard_tokens(shards, T, H, W, n_cond, block)
    G = len(shards)
    qf = _f64(q)
    B, N, heads, hd = qf.shape
    Nc = n_cond * H * W
    out = np.zeros((B, N, heads, hd))
    lse = np.zeros((B, heads, N))
    steps = []
    for r in range(G):
        qa, qb = toks[r]
        o_acc = np.zeros((B, qb - qa, heads, hd))
        l_acc = np.full((B, heads, qb - qa), -np.inf)
        for s in range(G):
            src = (r - s) % G
            ka, kb = toks[src]
            pairs = int(token_mask(N, Nc, block, local, stride, rows=np.arange(qa, qb),
                                   cols=np.arange(ka, kb)).sum())
            steps.append((r, s, src, pairs))
            if pairs == 0:
                continue
            o_p, l_p = partial_attention(q[:, qa:qb], k[:, ka:kb], v[:, ka:kb], T=T, H=H, W=W,
                                         n_cond=n_cond, block=block, local=local, stride=stride,
                                         q_tokens=(qa, qb), k_tokens=(ka, kb), scale=scale,
                                         q_norm=q_norm, k_norm=k_norm, norm_eps=norm_eps)
            o_acc, l_acc = lse_merge(o_acc, l_acc, o_p, l_p)
        out[:, qa:qb] = o_acc
        lse[:, :, qa:qb] = l_acc
    return out, lse, steps
