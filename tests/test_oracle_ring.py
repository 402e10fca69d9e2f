"""Pins of the ring context-parallelism oracle (no GPU).

The ring (partial attention per K/V shard, merged by log-sum-exp in ring
order) is checked against the whole-sequence forward of the pinned C oracle,
an independent implementation; the merge against a two-key closed form and
its identities; the per-step attended pairs against the C brute-force count.
"""
import numpy as np
import pytest

import oracle
from oracle import ring as orng

CASES = [
    # (geometry, shards as block ranges; query bounds on 4-block group edges)
    (dict(T=5, H=8, W=40, n_cond=2, local=1, stride=2), [(0, 4), (4, 10), (10, 18), (18, 25)]),
    (dict(T=6, H=5, W=13, n_cond=0, local=0, stride=3), [(0, 4), (4, 7)]),
    (dict(T=8, H=3, W=22, n_cond=2, local=2, stride=0), [(0, 3), (3, 7), (7, 10)]),
    (dict(T=7, H=8, W=16, n_cond=1, local=1, stride=4), [(0, 2), (2, 6), (6, 10), (10, 14)]),
]


def _inputs(c, heads=2, B=1, seed=0):
    N = c["T"] * c["H"] * c["W"]
    rng = np.random.default_rng(seed)
    return [rng.standard_normal((B, N, heads, 64)) for _ in range(3)]


@pytest.mark.parametrize("case", range(len(CASES)))
def test_ring_equals_whole_sequence_forward(case):
    c, shards = CASES[case]
    Nc, Nn, Cb, Nb = oracle.segment_sizes(c["T"], c["H"], c["W"], c["n_cond"])
    assert shards[0][0] == 0 and shards[-1][1] == Cb + Nb
    q, k, v = _inputs(c, B=2 if case == 1 else 1, seed=case)
    out, lse, steps = orng.ring_forward(q, k, v, shards, **c)
    ref_o, ref_l = oracle.forward(q, k, v, **c)
    assert np.abs(out - ref_o).max() <= 1e-12 * max(1.0, np.abs(ref_o).max())
    assert np.abs(lse - ref_l).max() <= 1e-12 * max(1.0, np.abs(ref_l).max())
    # every attended pair is computed by exactly one (rank, step)
    N = c["T"] * c["H"] * c["W"]
    assert sum(p for *_, p in steps) == oracle.count_token_pairs(N, Nc, 64, c["local"],
                                                                  c["stride"])


def test_ring_with_rms_norm():
    c, shards = CASES[0]
    q, k, v = _inputs(c, seed=5)
    g = np.random.default_rng(6)
    qn, kn = 1 + 0.3 * g.standard_normal(64), 1 + 0.3 * g.standard_normal(64)
    out, lse, _ = orng.ring_forward(q, k, v, shards, q_norm=qn, k_norm=kn, norm_eps=1e-6, **c)
    ref_o, ref_l = oracle.forward(q, k, v, q_norm=qn, k_norm=kn, norm_eps=1e-6, **c)
    assert np.abs(out - ref_o).max() <= 1e-12 * max(1.0, np.abs(ref_o).max())
    assert np.abs(lse - ref_l).max() <= 1e-12 * max(1.0, np.abs(ref_l).max())


def test_partial_over_all_keys_is_the_forward():
    c, _ = CASES[3]
    q, k, v = _inputs(c, seed=9)
    N = q.shape[1]
    o, l = orng.partial_attention(q, k, v, q_tokens=(0, N), k_tokens=(0, N), **c)
    ref_o, ref_l = oracle.forward(q, k, v, **c)
    assert np.abs(o - ref_o).max() <= 1e-12 * np.abs(ref_o).max()
    assert np.abs(l - ref_l).max() <= 1e-12 * np.abs(ref_l).max()


def test_condition_rows_see_no_noisy_keys():
    """Condition queries against a noisy-only key shard: out 0, lse -inf; the
    step has no attended pair, so the ring skips it."""
    c, shards = CASES[0]
    q, k, v = _inputs(c, seed=2)
    toks = orng.shard_tokens(shards, c["T"], c["H"], c["W"], c["n_cond"])
    (qa, qb), (ka, kb) = toks[0], toks[2]
    o, l = orng.partial_attention(q[:, qa:qb], k[:, ka:kb], v[:, ka:kb], q_tokens=(qa, qb),
                                  k_tokens=(ka, kb), **c)
    assert np.all(o == 0) and np.all(l == -np.inf)
    _, _, steps = orng.ring_forward(q, k, v, shards, **c)
    assert any(r == 0 and src == 2 and p == 0 for r, _, src, p in steps)


def test_merge_two_keys_closed_form():
    """Logits 0 and log 3 over values e0 and e1: weights 1/4 and 3/4, lse log 4."""
    e0 = np.zeros((1, 1, 1, 64)); e0[..., 0] = 1.0
    e1 = np.zeros((1, 1, 1, 64)); e1[..., 1] = 1.0
    o, l = orng.lse_merge(e0, np.zeros((1, 1, 1)), e1, np.full((1, 1, 1), np.log(3.0)))
    assert abs(o[0, 0, 0, 0] - 0.25) < 1e-15 and abs(o[0, 0, 0, 1] - 0.75) < 1e-15
    assert abs(l[0, 0, 0] - np.log(4.0)) < 1e-15
    assert np.all(o[0, 0, 0, 2:] == 0)


def test_merge_identities():
    rng = np.random.default_rng(3)
    o = rng.standard_normal((2, 5, 3, 64))
    l = rng.standard_normal((2, 3, 5))
    empty_o, empty_l = np.zeros_like(o), np.full_like(l, -np.inf)
    # an empty part changes nothing, on either side
    for a, b in (((o, l), (empty_o, empty_l)), ((empty_o, empty_l), (o, l))):
        mo, ml = orng.lse_merge(*a, *b)
        assert np.array_equal(mo, o) and np.array_equal(ml, l)
    # two empty parts stay empty
    mo, ml = orng.lse_merge(empty_o, empty_l, empty_o, empty_l)
    assert np.all(mo == 0) and np.all(ml == -np.inf)
    # order does not matter (up to rounding)
    o2, l2 = rng.standard_normal(o.shape), rng.standard_normal(l.shape) + 2.0
    a_o, a_l = orng.lse_merge(o, l, o2, l2)
    b_o, b_l = orng.lse_merge(o2, l2, o, l)
    assert np.abs(a_o - b_o).max() < 1e-14 and np.abs(a_l - b_l).max() < 1e-14
    # equal lse: the plain mean, lse + log 2
    m_o, m_l = orng.lse_merge(o, l, o2, l)
    assert np.abs(m_o - 0.5 * (o + o2)).max() < 1e-14
    assert np.abs(m_l - (l + np.log(2.0))).max() < 1e-14
