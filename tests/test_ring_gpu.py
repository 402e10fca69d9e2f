"""Ring context parallelism on the GPU: shard plans, the shard forward
(lc_bsa_forward_shard), the log-sum-exp merge (lc_bsa_lse_merge) and the
whole ring, one process standing in for every rank (each rank's K/V shard is
taken from the full tensors instead of arriving over NCCL; the exchange itself
is covered on CPU with gloo), against the fp64 oracle.

Tolerances: bf16 as the forward's (|out - ref| <= 1.5e-2, mean <= 1e-3; lse
<= 5e-2), plus at most one more bf16 rounding of the merged output; the merge
kernel alone works in fp32 on exact inputs: 1e-6 relative.
"""
import numpy as np
import pytest
import torch

import oracle
from oracle import ring as orng
from block_sparse_attention_rope_b200 import ring, synthetic
from block_sparse_attention_rope_b200.synthetic import Workload

pytestmark = pytest.mark.gpu

SMALL = Workload("ring_small", T=5, H=8, W=40, n_cond=2, heads=2, local=1, stride=2,
                 dtype="bf16")                       # Cb 10, Nb 15: 25 blocks, ragged tails
RAGGED = Workload("ring_ragged", T=6, H=13, W=21, n_cond=1, heads=2, local=2, stride=3,
                  dtype="bf16", batch=2)


@pytest.fixture(scope="module")
def api():
    from block_sparse_attention_rope_b200 import build
    build.build()
    from block_sparse_attention_rope_b200 import api as a
    return a


def geo(w):
    return dict(T=w.T, H=w.H, W=w.W, n_cond=w.n_cond, local=w.local, stride=w.stride)


def blocks(w):
    Nc, Nn, Cb, Nb = oracle.segment_sizes(w.T, w.H, w.W, w.n_cond)
    return Cb, Nb


def test_shard_plans_partition_the_full_plan(api):
    w = SMALL
    Cb, Nb = blocks(w)
    full = api.Plan(w.T, w.H, w.W, local=w.local, stride=w.stride, n_cond=w.n_cond)
    rp, ci = (x.numpy() for x in full.csr())
    fi = full.info()
    shards = [(0, 4), (4, 10), (10, 18), (18, 25)]
    nnz = pairs = 0
    for qs in shards:
        for ks in shards:
            p = api.Plan(w.T, w.H, w.W, local=w.local, stride=w.stride, n_cond=w.n_cond,
                         q_blocks=qs, k_blocks=ks)
            inf = p.info()
            srp, sci = (x.numpy() for x in p.csr())
            # the shard's CSR is the full CSR with rows and columns restricted (bit-exact)
            for r in range(Cb + Nb):
                row = ci[rp[r]:rp[r + 1]]
                want = row[(row >= ks[0]) & (row < ks[1])] if qs[0] <= r < qs[1] else row[:0]
                assert np.array_equal(sci[srp[r]:srp[r + 1]], want)
            nnz += inf.nnz
            pairs += inf.attended_token_pairs
    assert nnz == fi.nnz and pairs == fi.attended_token_pairs


def test_shard_plan_argument_errors(api):
    w = SMALL
    with pytest.raises(api.LcError):   # query bound inside a group
        api.Plan(w.T, w.H, w.W, local=1, stride=2, n_cond=2, q_blocks=(0, 6), k_blocks=(0, 25))
    with pytest.raises(api.LcError):   # past the last block
        api.Plan(w.T, w.H, w.W, local=1, stride=2, n_cond=2, q_blocks=(0, 4), k_blocks=(0, 26))
    p = api.Plan(w.T, w.H, w.W, local=1, stride=2, n_cond=2, q_blocks=(4, 10), k_blocks=(3, 7))
    assert p.q_tokens == (256, 640) and p.k_tokens == (192, 448)
    rope = api.Rope3D(w.T, w.H, w.W)
    x = synthetic.make_inputs(w)
    q = x["q"].cuda()
    # a shard plan is refused by the whole-sequence entry points
    with pytest.raises(api.LcError):
        api.forward(q, x["k"].cuda(), x["v"].cuda(), p, rope)
    with pytest.raises(api.LcError):   # fp32 shards are not supported
        qf = torch.zeros(1, 384, 2, 64, device="cuda")
        kf = torch.zeros(1, 256, 2, 64, device="cuda")
        api.forward_shard(qf, kf, kf, p, rope)


def _shard_case(api, w, x, rope, qs, ks):
    p = api.Plan(w.T, w.H, w.W, local=w.local, stride=w.stride, n_cond=w.n_cond,
                 q_blocks=qs, k_blocks=ks)
    (qa, qb), (ka, kb) = p.q_tokens, p.k_tokens
    d = {n: x[n].cuda() for n in ("q", "k", "v")}
    out = torch.full((w.batch, qb - qa, w.heads, 64), float("nan"), dtype=torch.bfloat16,
                     device="cuda")
    lse = torch.full((w.batch, w.heads, qb - qa), float("nan"), device="cuda")
    api.forward_shard(d["q"][:, qa:qb].contiguous(), d["k"][:, ka:kb].contiguous(),
                      d["v"][:, ka:kb].contiguous(), p, rope, out=out, lse=lse)
    torch.cuda.synchronize()
    assert api.last_device_status() == 0
    ref_o, ref_l = orng.partial_attention(x["q"][:, qa:qb], x["k"][:, ka:kb], x["v"][:, ka:kb],
                                          q_tokens=(qa, qb), k_tokens=(ka, kb), **geo(w))
    return out.double().cpu().numpy(), lse.double().cpu().numpy(), ref_o, ref_l


@pytest.mark.parametrize("qs,ks", [((4, 10), (0, 25)), ((10, 18), (10, 18)), ((0, 4), (10, 25)),
                                   ((18, 25), (3, 11)), ((10, 14), (20, 25)), ((0, 10), (0, 3))])
def test_forward_shard_matches_oracle(api, qs, ks):
    w = SMALL
    x = synthetic.make_inputs(w)
    rope = api.Rope3D(w.T, w.H, w.W)
    o, l, ref_o, ref_l = _shard_case(api, w, x, rope, qs, ks)
    empty = ref_l == -np.inf
    # rows that attend no key of the shard: exactly (0, -inf); every other row is written
    assert np.array_equal(l == -np.inf, empty)
    assert np.all(o.transpose(0, 2, 1, 3)[empty] == 0)
    assert not np.isnan(o).any() and not np.isnan(l).any()
    err = np.abs(o - ref_o)
    assert err.max() <= 1.5e-2 and err.mean() <= 1e-3, (err.max(), err.mean())
    fin = ~empty
    if fin.any():
        assert np.abs(l[fin] - ref_l[fin]).max() <= 5e-2


def test_lse_merge_kernel(api):
    g = torch.Generator().manual_seed(5)
    B, n, heads = 2, 300, 3
    o_a = torch.randn(B, n, heads, 64, generator=g)
    l_a = 3 * torch.randn(B, heads, n, generator=g)
    o_b = torch.randn(B, n, heads, 64, generator=g).bfloat16()
    l_b = 3 * torch.randn(B, heads, n, generator=g)
    l_a[0, 0, :7] = -float("inf")          # empty running rows
    o_a[0, :7, 0] = 0
    l_b[1, 2, 10:20] = -float("inf")       # empty part rows (their o is 0)
    o_b[1, 10:20, 2] = 0
    l_a[1, 1, 30:33] = l_b[1, 1, 30:33] = -float("inf")
    o_a[1, 30:33, 1] = 0
    o_b[1, 30:33, 1] = 0
    ref_o, ref_l = orng.lse_merge(o_a.double().numpy(), l_a.double().numpy(),
                                  o_b.double().numpy(), l_b.double().numpy())
    acc_o, acc_l = o_a.cuda(), l_a.cuda()
    api.lse_merge(acc_o, acc_l, o_b.cuda(), l_b.cuda())
    torch.cuda.synchronize()
    assert np.abs(acc_o.double().cpu().numpy() - ref_o).max() <= 1e-6 * np.abs(ref_o).max()
    gl = acc_l.double().cpu().numpy()
    assert np.array_equal(gl == -np.inf, ref_l == -np.inf)
    fin = np.isfinite(ref_l)
    assert np.abs(gl[fin] - ref_l[fin]).max() <= 1e-6 * np.abs(ref_l[fin]).max()
    # init: the part is copied (empty rows -> 0); out: the merged o in the part's dtype
    acc_o2, acc_l2 = torch.full_like(acc_o, float("nan")), torch.full_like(acc_l, float("nan"))
    api.lse_merge(acc_o2, acc_l2, o_b.cuda(), l_b.cuda(), init=True)
    torch.cuda.synchronize()
    assert torch.equal(acc_o2.cpu(), o_b.float()) and torch.equal(acc_l2.cpu(), l_b)
    out = torch.empty_like(o_b).cuda()
    acc_o3, acc_l3 = o_a.cuda(), l_a.cuda()
    api.lse_merge(acc_o3, acc_l3, o_b.cuda(), l_b.cuda(), out=out)
    torch.cuda.synchronize()
    assert torch.equal(acc_o3.cpu(), o_a)  # not written when out is given
    assert torch.equal(out.cpu(), torch.from_numpy(ref_o).float().bfloat16()) or \
        np.abs(out.double().cpu().numpy() - ref_o).max() <= 2 ** -8 * np.abs(ref_o).max()


def run_ring(api, w, x, shards, rope, dev, q_norm=None, k_norm=None):
    """Every rank of the ring in this process; returns out [B, N, heads, 64], lse."""
    d = {n: x[n].to(dev) for n in ("q", "k", "v")}
    out = torch.empty_like(d["q"])
    lse = torch.empty(w.batch, w.heads, w.n_tokens, device=dev)
    ranks = [ring.GpuRingRank(api, w.T, w.H, w.W, local=w.local, stride=w.stride,
                              n_cond=w.n_cond, shards=shards, rank=r, rope=rope, batch=w.batch,
                              heads=w.heads, device=dev, q_norm=q_norm, k_norm=k_norm)
             for r in range(len(shards))]
    toks = ranks[0].sched.tokens
    # what each rank sends around the ring: its K shard normalised and rotated once
    k_rot = {s: ranks[s].rotate(d["k"][:, a:b].contiguous(), s, k_norm)
             for s, (a, b) in enumerate(toks)}
    v_sh = {s: d["v"][:, a:b].contiguous() for s, (a, b) in enumerate(toks)}
    for rank, rr in enumerate(ranks):
        a, b = toks[rank]
        o, l = rr.forward(d["q"][:, a:b].contiguous(), d["k"][:, a:b].contiguous(), v_sh[rank],
                          fetch=lambda src: (k_rot[src], v_sh[src]))
        out[:, a:b] = o
        lse[:, :, a:b] = l
    torch.cuda.synchronize()
    assert api.last_device_status() == 0
    return out, lse


def test_prerotated_shards_are_bit_exact(api):
    """q / k rotated (and normalised) once by lc_rope3d_apply_ex and flagged
    give the same bits as the shard kernel's own rotations."""
    w = SMALL
    x = synthetic.make_inputs(w, device="cuda")
    rope = api.Rope3D(w.T, w.H, w.W)
    g = torch.Generator().manual_seed(4)
    for norm in (False, True):
        qn = (1 + 0.3 * torch.randn(64, generator=g)).cuda() if norm else None
        kn = (1 + 0.3 * torch.randn(64, generator=g)).cuda() if norm else None
        for qs, ks in (((4, 10), (0, 25)), ((10, 18), (3, 11))):
            p = api.Plan(w.T, w.H, w.W, local=w.local, stride=w.stride, n_cond=w.n_cond,
                         q_blocks=qs, k_blocks=ks)
            (qa, qb), (ka, kb) = p.q_tokens, p.k_tokens
            q, k, v = (x[n][:, a:b].contiguous() for n, a, b in
                       (("q", qa, qb), ("k", ka, kb), ("v", ka, kb)))
            o1, l1 = api.forward_shard(q, k, v, p, rope, q_norm=qn, k_norm=kn)
            qr = rope.apply(q, tok_offset=qa, norm=qn)
            kr = rope.apply(k, tok_offset=ka, norm=kn)
            o2, l2 = api.forward_shard(qr, kr, v, p, rope, q_rotated=True, k_rotated=True)
            o3, l3 = api.forward_shard(q, kr, v, p, rope, q_norm=qn, k_rotated=True)
            torch.cuda.synchronize()
            assert torch.equal(o1, o2) and torch.equal(l1, l2)
            assert torch.equal(o1, o3) and torch.equal(l1, l3)


def test_keep_empty_rows_leaves_groups_without_keys(api):
    """With LC_FLAG_KEEP_EMPTY_ROWS the rows of work groups that have no key in
    the shard are not written; every other row is the same as without it."""
    w = SMALL
    x = synthetic.make_inputs(w, device="cuda")
    rope = api.Rope3D(w.T, w.H, w.W)
    p = api.Plan(w.T, w.H, w.W, local=w.local, stride=w.stride, n_cond=w.n_cond,
                 q_blocks=(0, 18), k_blocks=(18, 25))   # condition groups see no key here
    (qa, qb), (ka, kb) = p.q_tokens, p.k_tokens
    q, k, v = (x[n][:, a:b].contiguous() for n, a, b in
               (("q", qa, qb), ("k", ka, kb), ("v", ka, kb)))
    o1, l1 = api.forward_shard(q, k, v, p, rope)
    o2 = torch.full_like(o1, float("nan"))
    l2 = torch.full_like(l1, float("nan"))
    api.forward_shard(q, k, v, p, rope, out=o2, lse=l2, keep_empty_rows=True)
    torch.cuda.synchronize()
    Nc = w.n_cond_tokens                                  # 640: the condition rows
    assert torch.isnan(o2[:, :Nc]).all() and torch.isnan(l2[:, :, :Nc]).all()
    assert torch.equal(o2[:, Nc:], o1[:, Nc:]) and torch.equal(l2[:, :, Nc:], l1[:, :, Nc:])
    assert (o1[:, :Nc] == 0).all() and (l1[:, :, :Nc] == -float("inf")).all()


def test_overlapping_shard_launches_are_bit_exact(api):
    """LC_FLAG_OVERLAP_PREVIOUS (programmatic dependent launch, the plan's
    self-resetting scheduler): a rank's steps launched back to back, each
    overlapping the previous one, give the same bits as separate launches;
    launching the same plans again (their schedulers reset by the previous
    launch's last CTA) gives them once more.  The flag needs keep_empty_rows."""
    w = RAGGED
    x = synthetic.make_inputs(w, device="cuda")
    rope = api.Rope3D(w.T, w.H, w.W)
    Cb, Nb = blocks(w)
    qs = (4, 13)                     # group edges: condition block 4, noisy 5 + 8
    steps = [(0, 6), (6, 14), (14, Cb + Nb), (3, 9)]
    plans = [api.Plan(w.T, w.H, w.W, local=w.local, stride=w.stride, n_cond=w.n_cond,
                      q_blocks=qs, k_blocks=ks) for ks in steps]
    (qa, qb) = plans[0].q_tokens
    q = rope.apply(x["q"][:, qa:qb].contiguous(), tok_offset=qa)
    kv = []
    for p in plans:
        ka, kb = p.k_tokens
        kv.append((rope.apply(x["k"][:, ka:kb].contiguous(), tok_offset=ka),
                   x["v"][:, ka:kb].contiguous()))

    def run(overlap):
        outs = [torch.zeros(w.batch, qb - qa, w.heads, 64, dtype=torch.bfloat16, device="cuda")
                for _ in plans]
        lses = [torch.full((w.batch, w.heads, qb - qa), -float("inf"), device="cuda")
                for _ in plans]
        for i, (p, (k, v)) in enumerate(zip(plans, kv)):
            api.forward_shard(q, k, v, p, rope, out=outs[i], lse=lses[i], q_rotated=True,
                              k_rotated=True, keep_empty_rows=True,
                              overlap_previous=overlap and i > 0)
        torch.cuda.synchronize()
        assert api.last_device_status() == 0
        return outs, lses

    ref = run(False)
    for _ in range(2):
        got = run(True)
        for a, b in zip(ref[0] + ref[1], got[0] + got[1]):
            assert torch.equal(a, b)
    with pytest.raises(api.LcError) as e:
        api.forward_shard(q, kv[0][0], kv[0][1], plans[0], rope, q_rotated=True,
                          k_rotated=True, overlap_previous=True)
    assert e.value.status == api.LC_ERR_INVALID_ARGUMENT


@pytest.mark.parametrize("n_parts", [1, 3, 8])
def test_lse_merge_parts_kernel(api, n_parts):
    g = torch.Generator().manual_seed(n_parts)
    B, n, heads = 2, 257, 3
    parts = torch.randn(n_parts, B, n, heads, 64, generator=g).bfloat16()
    lses = 4 * torch.randn(n_parts, B, heads, n, generator=g)
    lses[:, 0, 1, :5] = -float("inf")          # rows empty in every part
    parts[:, 0, :5, 1] = 0
    lses[0, 1, 2, 7:40] = -float("inf")        # rows empty in one part
    parts[0, 1, 7:40, 2] = 0
    ref_o, ref_l = parts[0].double().numpy(), lses[0].double().numpy()
    for i in range(1, n_parts):
        ref_o, ref_l = orng.lse_merge(ref_o, ref_l, parts[i].double().numpy(),
                                      lses[i].double().numpy())
    out, lse = api.lse_merge_parts(parts.cuda(), lses.cuda())
    torch.cuda.synchronize()
    o = out.double().cpu().numpy()
    # one rounding to bf16 of an fp32 combination
    assert np.all(np.abs(o - ref_o) <= 2 ** -8 * np.abs(ref_o) + 1e-6 * np.abs(ref_o).max())
    gl = lse.double().cpu().numpy()
    assert np.array_equal(gl == -np.inf, ref_l == -np.inf)
    fin = np.isfinite(ref_l)
    assert np.abs(gl[fin] - ref_l[fin]).max() <= 1e-6 * np.abs(ref_l[fin]).max()
    assert np.all(o.transpose(0, 2, 1, 3)[~fin] == 0)


@pytest.mark.parametrize("w,world", [(SMALL, 1), (SMALL, 2), (SMALL, 4), (RAGGED, 3), (RAGGED, 5)])
def test_ring_matches_oracle_and_full_forward(api, w, world):
    x = synthetic.make_inputs(w)
    Cb, Nb = blocks(w)
    rp, _ = oracle.block_csr(w.T, w.H, w.W, 64, w.local, w.stride, w.n_cond)
    shards = ring.balanced_shards(np.diff(rp), Cb, world)
    rope = api.Rope3D(w.T, w.H, w.W)
    out, lse = run_ring(api, w, x, shards, rope, "cuda")
    ref_o, ref_l = oracle.forward(x["q"], x["k"], x["v"], **geo(w))
    o = out.double().cpu().numpy()
    err = np.abs(o - ref_o)
    assert err.max() <= 1.5e-2 and err.mean() <= 1e-3, (err.max(), err.mean())
    assert np.abs(lse.double().cpu().numpy() - ref_l).max() <= 5e-2
    # and next to the single-launch forward: the same up to one more rounding
    plan = api.Plan(w.T, w.H, w.W, local=w.local, stride=w.stride, n_cond=w.n_cond)
    full_o, full_l = api.forward(x["q"].cuda(), x["k"].cuda(), x["v"].cuda(), plan, rope,
                                 return_lse=True)
    assert (out.float() - full_o.float()).abs().max().item() <= 1.6e-2
    assert (lse - full_l).abs().max().item() <= 1e-2


def test_ring_with_rms_norm(api):
    w = SMALL
    x = synthetic.make_inputs(w)
    g = torch.Generator().manual_seed(8)
    qn, kn = 1 + 0.3 * torch.randn(64, generator=g), 1 + 0.3 * torch.randn(64, generator=g)
    shards = [(0, 4), (4, 10), (10, 18), (18, 25)]
    rope = api.Rope3D(w.T, w.H, w.W)
    out, lse = run_ring(api, w, x, shards, rope, "cuda", qn.cuda(), kn.cuda())
    ref_o, ref_l, _ = orng.ring_forward(x["q"], x["k"], x["v"], shards, q_norm=qn.double().numpy(),
                                        k_norm=kn.double().numpy(), norm_eps=1e-6, **geo(w))
    err = np.abs(out.double().cpu().numpy() - ref_o)
    assert err.max() <= 1.5e-2 and err.mean() <= 1e-3, (err.max(), err.mean())
    assert np.abs(lse.double().cpu().numpy() - ref_l).max() <= 5e-2


def test_ring_full_size_sampled(api):
    """I2V 480p (37,440 tokens, 32 heads) over 8 ring ranks in one process:
    sampled rows against the oracle, every row against the single launch."""
    from parity import compare, oracle_rows, sample_rows
    w = synthetic.get("i2v_480p")
    x = synthetic.make_inputs(w)
    rp, _ = oracle.block_csr(w.T, w.H, w.W, 64, w.local, w.stride, w.n_cond)
    Cb, Nb = blocks(w)
    shards = ring.balanced_shards(np.diff(rp), Cb, 8)
    rope = api.Rope3D(w.T, w.H, w.W)
    out, lse = run_ring(api, w, x, shards, rope, "cuda")
    rows = sample_rows(w, n_random_blocks=16)
    # rows on both sides of every shard boundary
    toks = orng.shard_tokens(shards, w.T, w.H, w.W, w.n_cond)
    edge = np.array([t for a, _ in toks[1:] for t in (a - 1, a)], dtype=np.int64)
    rows = np.unique(np.concatenate([rows, edge]))
    heads = [0, 31]
    ref_o, ref_l = oracle_rows(w, x, rows, heads)
    compare(w, out.cpu(), lse.cpu(), ref_o, ref_l, rows, heads)
    plan = api.Plan(w.T, w.H, w.W, local=w.local, stride=w.stride, n_cond=w.n_cond)
    full_o, full_l = api.forward(x["q"].cuda(), x["k"].cuda(), x["v"].cuda(), plan, rope,
                                 return_lse=True)
    assert (out.float() - full_o.float()).abs().max().item() <= 1.6e-2
    assert (lse - full_l).abs().max().item() <= 1e-2


def test_ring_720p_equals_single_launch():
    """720p refine (86,400 tokens, 1,350 blocks, no condition frames) over 8
    ranks with the planned cuts: the same as the whole-sequence launch up to
    one more bf16 rounding of the output, every element."""
    from block_sparse_attention_rope_b200 import api as a
    w = synthetic.get("refine_720p")
    x = synthetic.make_inputs(w)
    plan = a.Plan(w.T, w.H, w.W, local=w.local, stride=w.stride, n_cond=w.n_cond)
    rp, ci = plan.csr()
    shards = ring.planned_shards(rp.tolist(), ci.tolist(), 0, 8, heads=w.heads)
    rope = a.Rope3D(w.T, w.H, w.W)
    out, lse = run_ring(a, w, x, shards, rope, "cuda")
    full_o, full_l = a.forward(x["q"].cuda(), x["k"].cuda(), x["v"].cuda(), plan, rope,
                               return_lse=True)
    torch.cuda.synchronize()
    assert (out.float() - full_o.float()).abs().max().item() <= 1.6e-2
    assert (lse - full_l).abs().max().item() <= 1e-2


def test_forward_shard_custom_scale(api):
    w = SMALL
    x = synthetic.make_inputs(w)
    rope = api.Rope3D(w.T, w.H, w.W)
    p = api.Plan(w.T, w.H, w.W, local=w.local, stride=w.stride, n_cond=w.n_cond,
                 q_blocks=(10, 18), k_blocks=(5, 20))
    (qa, qb), (ka, kb) = p.q_tokens, p.k_tokens
    o, l = api.forward_shard(x["q"][:, qa:qb].contiguous().cuda(),
                             x["k"][:, ka:kb].contiguous().cuda(),
                             x["v"][:, ka:kb].contiguous().cuda(), p, rope, softmax_scale=0.3)
    torch.cuda.synchronize()
    ref_o, ref_l = orng.partial_attention(x["q"][:, qa:qb], x["k"][:, ka:kb], x["v"][:, ka:kb],
                                          q_tokens=(qa, qb), k_tokens=(ka, kb), scale=0.3,
                                          **geo(w))
    # logits 2.4x those of the default scale, so 2.4x the bf16 bounds (as in
    # the forward's large-logit test)
    k = 0.3 / 0.125
    err = np.abs(o.double().cpu().numpy() - ref_o)
    assert err.max() <= 1.5e-2 * k and err.mean() <= 1e-3 * k
    fin = np.isfinite(ref_l)
    assert np.abs(l.double().cpu().numpy()[fin] - ref_l[fin]).max() <= 5e-2 * k


def test_merges_with_fp32_parts(api):
    """lc_bsa_lse_merge and lc_bsa_lse_merge_parts on fp32 partial outputs."""
    g = torch.Generator().manual_seed(21)
    P, B, n, heads = 3, 1, 130, 2
    parts = torch.randn(P, B, n, heads, 64, generator=g)
    lses = 2 * torch.randn(P, B, heads, n, generator=g)
    lses[1, 0, 0, :9] = -float("inf")
    parts[1, 0, :9, 0] = 0
    ref_o, ref_l = parts[0].double().numpy(), lses[0].double().numpy()
    for i in range(1, P):
        ref_o, ref_l = orng.lse_merge(ref_o, ref_l, parts[i].double().numpy(),
                                      lses[i].double().numpy())
    out, lse = api.lse_merge_parts(parts.cuda(), lses.cuda())
    acc_o, acc_l = parts[0].cuda().clone(), lses[0].cuda().clone()
    for i in range(1, P):
        api.lse_merge(acc_o, acc_l, parts[i].cuda(), lses[i].cuda())
    torch.cuda.synchronize()
    for o, l in ((out, lse), (acc_o, acc_l)):
        assert np.abs(o.double().cpu().numpy() - ref_o).max() <= 1e-5 * np.abs(ref_o).max()
        assert np.abs(l.double().cpu().numpy() - ref_l).max() <= 1e-5 * np.abs(ref_l).max()
