"""GPU planner and RoPE kernels against the oracle (bit-exact CSR, RoPE)."""
import json
import os

import numpy as np
import pytest
import torch

import oracle
from block_sparse_attention_rope_b200 import synthetic

pytestmark = pytest.mark.gpu
GOLDEN = os.path.join(os.path.dirname(__file__), "golden")

EDGE_PLANS = [  # (T, H, W, local, stride, n_cond)
    (4, 8, 16, 2, 4, 0), (6, 13, 21, 1, 3, 1), (5, 5, 13, 0, 0, 2), (3, 4, 11, 2, 1, 1),
    (1, 1, 1, 0, 0, 0), (2, 1, 65, 3, 5, 1), (9, 7, 9, 40, 2, 3), (24, 30, 52, 2, 4, 1),
    (32, 30, 52, 2, 4, 8), (24, 45, 80, 1, 16, 0), (24, 30, 52, 0, 1, 0), (24, 30, 52, 1, 32, 0),
]


@pytest.fixture(scope="module")
def api():
    from block_sparse_attention_rope_b200 import build
    build.build()
    from block_sparse_attention_rope_b200 import api as a
    return a


@pytest.mark.parametrize("T,H,W,local,stride,n_cond", EDGE_PLANS)
def test_plan_csr_bit_exact(api, T, H, W, local, stride, n_cond):
    plan = api.Plan(T, H, W, local=local, stride=stride, n_cond=n_cond)
    rp, ci = plan.csr()
    ref_rp, ref_ci = oracle.block_csr(T, H, W, 64, local, stride, n_cond)
    np.testing.assert_array_equal(rp.numpy(), ref_rp)
    np.testing.assert_array_equal(ci.numpy(), ref_ci)
    inf = plan.info()
    Nc, Nn, Cb, Nb = oracle.segment_sizes(T, H, W, n_cond)
    assert (inf.num_q_blocks, inf.num_cond_blocks, inf.num_noisy_blocks) == (Cb + Nb, Cb, Nb)
    assert (inf.n_cond_tokens, inf.n_noisy_tokens, inf.nnz) == (Nc, Nn, len(ref_ci))
    if T * H * W <= 6000:
        pairs = oracle.count_token_pairs(T * H * W, Nc, 64, local, stride)
        assert inf.attended_token_pairs == pairs
        assert inf.attended_token_pairs_noisy == pairs - Nc * Nc
    plan.close()


def test_plan_counts_of_named_workloads(api):
    counts = json.load(open(os.path.join(GOLDEN, "plan_counts.json")))
    for name, w in synthetic.WORKLOADS.items():
        plan = api.Plan(w.T, w.H, w.W, local=w.local, stride=w.stride, n_cond=w.n_cond)
        inf = plan.info()
        c = counts[name]
        assert inf.nnz == c["nnz"] and inf.num_q_blocks == c["q_blocks"]
        got = inf.attended_token_pairs_noisy if w.cached else inf.attended_token_pairs
        assert got == c["attended_token_pairs_per_head"], name


@pytest.mark.parametrize("T,H,W", [(4, 8, 16), (24, 45, 80), (32, 30, 52)])
def test_rope_tables(api, T, H, W):
    rope = api.Rope3D(T, H, W)
    tab = rope.tables().numpy().astype(np.float64)
    off = 0
    for npos, d in [(T, 16), (H, 24), (W, 24)]:
        k = np.arange(d // 2)
        ang = np.arange(npos)[:, None] * 10000.0 ** (-2.0 * k[None, :] / d)
        n = npos * d // 2
        np.testing.assert_allclose(tab[off:off + n], np.cos(ang).ravel(), rtol=0, atol=1.2e-7)
        np.testing.assert_allclose(tab[off + n:off + 2 * n], np.sin(ang).ravel(), rtol=0, atol=1.2e-7)
        off += 2 * n


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_rope_apply_matches_oracle(api, dtype):
    T, H, W = 5, 6, 7
    rope = api.Rope3D(T, H, W)
    g = torch.Generator().manual_seed(3)
    x = torch.randn(2, T * H * W - 30, 3, 64, generator=g).to(dtype)
    y = rope.apply(x.cuda(), tok_offset=30).cpu()
    ref = oracle.rope3d_apply(x.float().numpy(), H, W, tok_offset=30)
    err = np.abs(y.float().numpy() - ref).max()
    assert err <= (2e-6 if dtype == torch.float32 else 3e-2), err
    if dtype == torch.bfloat16:  # one bf16 rounding of the fp32 rotation
        rel = np.abs(y.float().numpy() - ref) / np.maximum(np.abs(ref), 1e-3)
        assert np.median(rel) < 4e-3
