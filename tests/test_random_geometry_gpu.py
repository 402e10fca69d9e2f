"""Seeded random geometries through the GPU kernels, every row against the
fp64 oracle: latent grids with ragged segment tails, 0..T-1 condition
frames, local windows 0..3, strides (none, dense, strided, past the end),
1..3 batch entries and 1..5 heads, in bf16 (tensor cores) and fp32 (SIMT);
the cached form on the same shapes; the backward on a subset.  Also one
full-size workload with two batch entries (the benchmark's launch), sampled
rows of every head of both entries.  Bounds are the parity bounds of the
dtype (tests/parity.py) and of the backward tests."""
import numpy as np
import pytest
import torch

import oracle
import parity
from oracle import backward as ob
from block_sparse_attention_rope_b200 import synthetic
from block_sparse_attention_rope_b200.synthetic import Workload

pytestmark = pytest.mark.gpu


def geometries(n, seed):
    rng = np.random.default_rng(seed)
    out = []
    while len(out) < n:
        T = int(rng.integers(1, 7))
        H = int(rng.integers(1, 14))
        W = int(rng.integers(1, 40))
        if T * H * W < 16 or T * H * W > 3000:
            continue
        n_cond = int(rng.integers(0, T))
        local = int(rng.integers(0, 4))
        stride = int(rng.choice([0, 1, 2, 3, 5, 1000]))
        heads = int(rng.integers(1, 6))
        batch = int(rng.integers(1, 4))
        out.append(dict(T=T, H=H, W=W, n_cond=n_cond, local=local, stride=stride, heads=heads,
                        batch=batch))
    return out


GEOS = geometries(24, seed=2026)


@pytest.fixture(scope="module")
def api():
    from block_sparse_attention_rope_b200 import build
    build.build()
    from block_sparse_attention_rope_b200 import api as a
    return a


def _run(api, w, x):
    d = {k: v.cuda() for k, v in x.items()}
    plan = api.Plan(w.T, w.H, w.W, local=w.local, stride=w.stride, n_cond=w.n_cond)
    rope = api.Rope3D(w.T, w.H, w.W)
    if w.cached:
        out, lse = api.forward_cached(d["q"], d["k"], d["v"], d.get("cond_k"), d.get("cond_v"),
                                      plan, rope, return_lse=True)
    else:
        out, lse = api.forward(d["q"], d["k"], d["v"], plan, rope, return_lse=True)
    torch.cuda.synchronize()
    assert api.last_device_status() == 0
    return out.cpu(), lse.cpu()


def _check(w, out, lse, ref_out, ref_lse):
    err = np.abs(out.float().numpy().astype(np.float64) - ref_out)
    lerr = np.abs(lse.numpy().astype(np.float64) - ref_lse)
    fin = np.isfinite(ref_lse)
    assert np.array_equal(np.isfinite(lse.numpy()), fin)  # rows without keys: none here
    if w.dtype == "f32":
        assert err.max() <= parity.F32_MAX_ABS, err.max()
        assert lerr[fin].max() <= parity.F32_LSE_ABS
    else:
        assert err.max() <= parity.BF16_MAX_ABS and err.mean() <= parity.BF16_MEAN_ABS, \
            (err.max(), err.mean())
        assert lerr[fin].max() <= parity.BF16_LSE_ABS


@pytest.mark.parametrize("i", range(len(GEOS)))
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_random_geometry_forward(api, i, dtype):
    g = GEOS[i]
    w = Workload("rand%d" % i, dtype=dtype, **g)
    x = synthetic.make_inputs(w, seed_offset=i)
    out, lse = _run(api, w, x)
    ref_out, ref_lse = oracle.forward(x["q"], x["k"], x["v"], T=w.T, H=w.H, W=w.W,
                                      n_cond=w.n_cond, local=w.local, stride=w.stride)
    _check(w, out, lse, ref_out, ref_lse)


@pytest.mark.parametrize("i", range(0, len(GEOS), 2))
def test_random_geometry_cached(api, i):
    g = GEOS[i]
    w = Workload("randc%d" % i, dtype="bf16", cached=True, **g)
    x = synthetic.make_inputs(w, seed_offset=i)
    out, lse = _run(api, w, x)
    ref_out, ref_lse = oracle.forward_cached(x["q"], x["k"], x["v"], x.get("cond_k"),
                                             x.get("cond_v"), T=w.T, H=w.H, W=w.W,
                                             n_cond=w.n_cond, local=w.local, stride=w.stride)
    _check(w, out, lse, ref_out, ref_lse)


@pytest.mark.parametrize("i", range(1, len(GEOS), 3))
def test_random_geometry_backward(api, i):
    g = GEOS[i]
    w = Workload("randb%d" % i, dtype="bf16", **g)
    x = synthetic.make_inputs(w, seed_offset=i)
    dout = synthetic.make_dout(w, seed_offset=i)
    d = {k: v.cuda() for k, v in x.items()}
    plan = api.Plan(w.T, w.H, w.W, local=w.local, stride=w.stride, n_cond=w.n_cond)
    rope = api.Rope3D(w.T, w.H, w.W)
    out, lse = api.forward(d["q"], d["k"], d["v"], plan, rope, return_lse=True)
    grads = api.backward(d["q"], d["k"], d["v"], out, lse, dout.cuda(), plan, rope)
    torch.cuda.synchronize()
    assert api.last_device_status() == 0
    ref = ob.backward(x["q"], x["k"], x["v"], dout, T=w.T, H=w.H, W=w.W, n_cond=w.n_cond,
                      local=w.local, stride=w.stride)
    for got, r, what in zip(grads, ref, ("dq", "dk", "dv")):
        gg = got.cpu().double().numpy()
        err = np.abs(gg - r)
        scale = max(np.abs(r).max(), 1e-30)
        assert np.all(err <= 2.0 ** -8 * np.abs(r) + 1.5e-2 * scale), (what, err.max(), scale)
        rel = np.sqrt((err ** 2).sum() / max((r ** 2).sum(), 1e-300))
        assert rel <= 6e-3, (what, rel)


def test_full_size_two_batch_entries_sampled(api):
    """I2V 480p with two batch entries in one launch (each its own seeded
    q, k, v): sampled rows of every head of both entries against the oracle."""
    w = synthetic.get("i2v_480p", batch=2)
    x = synthetic.make_inputs(w)
    out, lse = _run(api, w, x)
    rows = parity.sample_rows(w, n_random_blocks=16)
    for b in range(2):
        xb = {k: v[b:b + 1] for k, v in x.items()}
        ref_out, ref_lse = parity.oracle_rows(w, xb, rows)
        parity.compare(w, out[b:b + 1], lse[b:b + 1], ref_out, ref_lse, rows)
