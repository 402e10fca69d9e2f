"""GPU backward pass (lc_bsa_backward) against the fp64 oracle's gradients.

Tolerances: fp32 path |g - ref| <= 1e-4 * max|ref| + 1e-5 (fp32 accumulation
on exact inputs, the forward's lse good to ~1e-6).  bf16 path
|g - ref| <= 2^-8 |ref| + 1.5e-2 * max|ref|: the first term is the final
rounding of the gradient to bf16; the second covers the forward's bf16 lse
(rounded q', k' and P: errors up to ~2e-3, which scale every p of a row) and
its bf16 output O inside D = rowsum(dO * O).
"""
import numpy as np
import pytest
import torch

import oracle
from oracle import backward as ob
from block_sparse_attention_rope_b200 import synthetic
from block_sparse_attention_rope_b200.synthetic import Workload

pytestmark = pytest.mark.gpu

CASES = {
    "small_i2v": Workload("small_i2v", T=4, H=16, W=40, n_cond=1, heads=2, local=2, stride=4,
                          dtype="bf16"),
    "ragged": Workload("ragged", T=6, H=13, W=21, n_cond=1, heads=2, local=1, stride=3,
                       dtype="bf16", batch=2),
    "dense": Workload("dense", T=3, H=8, W=24, n_cond=0, heads=2, local=0, stride=1,
                      dtype="bf16"),
    "ragged_f32": Workload("ragged_f32", T=6, H=13, W=21, n_cond=1, heads=2, local=1, stride=3,
                           dtype="f32"),
    "local_f32": Workload("local_f32", T=2, H=10, W=30, n_cond=0, heads=3, local=0, stride=0,
                          dtype="f32"),
    "short_noisy": Workload("short_noisy", T=4, H=6, W=10, n_cond=3, heads=2, local=1, stride=2,
                            dtype="bf16"),
    "tiny_tokens": Workload("tiny_tokens", T=5, H=1, W=7, n_cond=2, heads=2, local=0, stride=3,
                            dtype="bf16"),
    # a grid whose RoPE table (16 T + 24 H + 24 W floats) does not fit in the
    # tensor-core kernel's shared memory beside its tiles: read from global memory
    "wide_grid": Workload("wide_grid", T=2, H=1, W=330, n_cond=0, heads=2, local=1, stride=2,
                          dtype="bf16"),
}


@pytest.fixture(scope="module")
def api():
    from block_sparse_attention_rope_b200 import build
    build.build()
    from block_sparse_attention_rope_b200 import api as a
    return a


# Relative RMS error bound ||g - ref|| / ||ref|| of the bf16 path.  Three
# bf16 roundings of about the same size add up: the rotated q', k' (logits,
# hence every p), the P^T and dS^T operands of the gradient products, and
# the gradient's own rounding (each ~2^-8 / sqrt(12)... 2^-9 relative RMS).
# Measured 2.7e-3 .. 4.4e-3 at the default softmax scale; 6e-3 holds that,
# and an error that is systematic rather than rounding (a gradient off by
# 1 % everywhere, a dropped term) exceeds it.  A larger softmax scale grows
# the logit term in proportion (rms_scale).  fp32 path: measured ~1e-6.
BF16_REL_RMS = 6e-3
F32_REL_RMS = 1e-5


def assert_close(w, got, ref, what, rms_scale=1.0):
    g = got.cpu().double().numpy()
    err = np.abs(g - ref)
    scale = max(np.abs(ref).max(), 1e-30)
    if w.dtype == "f32":
        bound = 1e-4 * scale + 1e-5
        rms_bound = F32_REL_RMS
    else:
        bound = 2.0 ** -8 * np.abs(ref) + 1.5e-2 * scale
        rms_bound = BF16_REL_RMS * rms_scale
    assert np.all(err <= bound), (what, err.max(), scale)
    rel = float(np.sqrt((err ** 2).sum() / max((np.asarray(ref) ** 2).sum(), 1e-300)))
    print("%s %s: max %.3g (of max|ref| %.3g), rel rms %.3g" % (w.name, what, err.max(), scale,
                                                                 rel))
    assert rel <= rms_bound, (what, rel)


def run(api, w, x, dout, qn=None, kn=None, eps=1e-6):
    d = {k: v.cuda() for k, v in x.items()}
    plan = api.Plan(w.T, w.H, w.W, local=w.local, stride=w.stride, n_cond=w.n_cond)
    rope = api.Rope3D(w.T, w.H, w.W)
    kw = dict(q_norm=qn, k_norm=kn, norm_eps=eps) if qn is not None or kn is not None else {}
    out, lse = api.forward(d["q"], d["k"], d["v"], plan, rope, return_lse=True, **kw)
    grads = api.backward(d["q"], d["k"], d["v"], out, lse, dout.cuda(), plan, rope, **kw)
    torch.cuda.synchronize()
    assert api.last_device_status() == 0
    return grads


@pytest.mark.parametrize("name", list(CASES))
def test_backward_matches_oracle(api, name):
    w = CASES[name]
    x = synthetic.make_inputs(w)
    dout = synthetic.make_dout(w)
    dq, dk, dv = run(api, w, x, dout)
    ref = ob.backward(x["q"], x["k"], x["v"], dout, T=w.T, H=w.H, W=w.W, n_cond=w.n_cond,
                      local=w.local, stride=w.stride)
    for got, r, what in zip((dq, dk, dv), ref, ("dq", "dk", "dv")):
        assert_close(w, got, r, what)
    # Every query's probabilities sum to one, so sum_m dv_m = sum_n dO_n per
    # head and channel.  The backward recomputes each row's p from the same
    # rounded q', k' the forward used and the forward's lse, so a row's p
    # still sum to one up to their rounding in the dV product (bf16 P: at
    # most 2^-9 relative each, of random sign, so the row's sum is off by
    # ~2^-9 |p_n| <= 2^-9); the dv_m are then rounded once more.  Bound: 6
    # standard deviations of those two sums of random-sign terms.
    do = dout.double().numpy()                            # [B, N, heads, 64]
    dvn = dv.double().cpu().numpy()
    s_dv, s_do = dvn.sum(axis=1), do.sum(axis=1)          # [B, heads, 64]
    rnd = 1e-6 if w.dtype == "f32" else 2.0 ** -9
    sd = rnd * (np.sqrt((do ** 2).sum(axis=1)) + np.sqrt((dvn ** 2).sum(axis=1)))
    gap = np.abs(s_dv - s_do)
    print("%s sum(dv) - sum(dO): max %.3g, bound min %.3g" % (name, gap.max(), (6 * sd).min()))
    assert np.all(gap <= 6 * sd), (gap.max(), (6 * sd).min())


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_backward_with_rms_norm(api, dtype):
    w = Workload("n", T=3, H=8, W=20, n_cond=1, heads=2, local=1, stride=2, dtype=dtype)
    x = synthetic.make_inputs(w)
    dout = synthetic.make_dout(w)
    g = torch.Generator().manual_seed(77)
    qn = 1.0 + 0.3 * torch.randn(64, generator=g)
    kn = 1.0 + 0.3 * torch.randn(64, generator=g)
    dq, dk, dv = run(api, w, x, dout, qn.cuda(), kn.cuda())
    ref = ob.backward(x["q"], x["k"], x["v"], dout, T=w.T, H=w.H, W=w.W, n_cond=w.n_cond,
                      local=w.local, stride=w.stride, q_norm=qn.double().numpy(),
                      k_norm=kn.double().numpy(), norm_eps=1e-6)
    for got, r, what in zip((dq, dk, dv), ref, ("dq", "dk", "dv")):
        assert_close(w, got, r, what)


@pytest.mark.parametrize("name", ["i2v_480p", "refine_720p", "continuation_cached"])
def test_plan_csc_bit_exact(api, name):
    w = synthetic.get(name)
    plan = api.Plan(w.T, w.H, w.W, local=w.local, stride=w.stride, n_cond=w.n_cond)
    cp, ri = plan.csc()
    rp, ci = oracle.block_csr(w.T, w.H, w.W, 64, w.local, w.stride, w.n_cond)
    nq = len(rp) - 1
    rows = np.repeat(np.arange(nq), np.diff(rp))
    order = np.lexsort((rows, ci))  # by column, then row
    ref_ri = rows[order].astype(np.int32)
    ref_cp = np.concatenate([[0], np.cumsum(np.bincount(ci, minlength=nq))]).astype(np.int32)
    assert np.array_equal(cp.numpy(), ref_cp)
    assert np.array_equal(ri.numpy(), ref_ri)


def test_backward_full_size_sampled(api):
    """I2V 480p (37,440 tokens, 32 heads, bf16): dq on sampled rows and dk / dv
    on a local-only noisy key block, a global column block and the last
    (partial) block, of two heads, against the oracle."""
    w = synthetic.get("i2v_480p")
    x = synthetic.make_inputs(w)
    dout = synthetic.make_dout(w)
    dq, dk, dv = run(api, w, x, dout)
    Nc, N = w.n_cond_tokens, w.n_tokens
    kw = dict(H=w.H, W=w.W, Nc=Nc, block=64, local=w.local, stride=w.stride)
    rng = np.random.default_rng(9)
    rows_n = np.unique(np.concatenate([[0, Nc - 1, Nc, N - 1], rng.integers(0, N, 40)]))
    for h in (0, 31):
        # one head at a time (the oracle upcasts whole tensors to fp64)
        xh = {k: x[k][:, :, h:h + 1].contiguous() for k in ("q", "k", "v")}
        gh = dout[:, :, h:h + 1].contiguous()
        trip = np.stack([np.zeros_like(rows_n), np.zeros_like(rows_n), rows_n], axis=1)
        ref = ob.backward_dq_rows(xh["q"], xh["k"], xh["v"], gh, rows=trip, **kw)
        assert_close(w, dq[0, torch.as_tensor(rows_n), h], ref, "dq rows")
        # noisy block 9 (9 % 4 != 0: local only), block 8 (global column), last block
        for j in (9, 8, (N - Nc - 1) // 64):
            keys = np.arange(Nc + 64 * j, min(N, Nc + 64 * j + 64))
            rk, rv = ob.backward_dkdv_keys(xh["q"], xh["k"], xh["v"], gh, b=0, h=0, keys=keys,
                                           **kw)
            kt = torch.as_tensor(keys)
            assert_close(w, dk[0, kt, h], rk, "dk block %d" % j)
            assert_close(w, dv[0, kt, h], rv, "dv block %d" % j)


def test_backward_argument_errors(api):
    w = CASES["small_i2v"]
    plan = api.Plan(w.T, w.H, w.W, local=w.local, stride=w.stride, n_cond=w.n_cond)
    rope = api.Rope3D(w.T, w.H, w.W)
    t = torch.zeros(1, w.n_tokens, w.heads, 64, dtype=torch.bfloat16, device="cuda")
    lse = torch.zeros(1, w.heads, w.n_tokens, device="cuda")
    o = [torch.empty_like(t) for _ in range(3)]
    lib, INV = api.lib, 1
    args = [t.data_ptr()] * 4 + [lse.data_ptr(), t.data_ptr()] + [x.data_ptr() for x in o]
    tail = [1, w.heads, 64, 0, 0.0, None, plan.handle, rope.handle, None]
    assert lib.lc_bsa_backward(*args, *tail) == 0
    bad = list(args)
    bad[6] = None                       # dq missing
    assert lib.lc_bsa_backward(*bad, *tail) == INV
    bad = list(args)
    bad[2] = t.data_ptr() + 2           # misaligned v
    assert lib.lc_bsa_backward(*bad, *tail) == INV
    assert lib.lc_bsa_backward(*args, 1, w.heads, 32, 0, 0.0, None, plan.handle, rope.handle,
                               None) == 2  # head_dim 32 unsupported
    torch.cuda.synchronize()


def test_backward_full_size_with_rms_norm_sampled(api):
    """I2V 480p backward with RMSNorm weights (dq and dk through the norm
    transpose, the finalize pass): dq on sampled rows and dk / dv on two key
    blocks of head 0, against the oracle."""
    w = synthetic.get("i2v_480p")
    x = synthetic.make_inputs(w)
    dout = synthetic.make_dout(w)
    g = torch.Generator().manual_seed(78)
    qn = 1.0 + 0.3 * torch.randn(64, generator=g)
    kn = 1.0 + 0.3 * torch.randn(64, generator=g)
    dq, dk, dv = run(api, w, x, dout, qn.cuda(), kn.cuda())
    Nc, N = w.n_cond_tokens, w.n_tokens
    kw = dict(H=w.H, W=w.W, Nc=Nc, block=64, local=w.local, stride=w.stride,
              q_norm=qn.double().numpy(), k_norm=kn.double().numpy(), norm_eps=1e-6)
    xh = {k: x[k][:, :, 0:1].contiguous() for k in ("q", "k", "v")}
    gh = dout[:, :, 0:1].contiguous()
    rng = np.random.default_rng(10)
    rows_n = np.unique(np.concatenate([[0, Nc - 1, Nc, N - 1], rng.integers(0, N, 24)]))
    trip = np.stack([np.zeros_like(rows_n), np.zeros_like(rows_n), rows_n], axis=1)
    ref = ob.backward_dq_rows(xh["q"], xh["k"], xh["v"], gh, rows=trip, **kw)
    assert_close(w, dq[0, torch.as_tensor(rows_n), 0], ref, "dq rows")
    for j in (9, 8):
        keys = np.arange(Nc + 64 * j, Nc + 64 * j + 64)
        rk, rv = ob.backward_dkdv_keys(xh["q"], xh["k"], xh["v"], gh, b=0, h=0, keys=keys, **kw)
        kt = torch.as_tensor(keys)
        assert_close(w, dk[0, kt, 0], rk, "dk block %d" % j)
        assert_close(w, dv[0, kt, 0], rv, "dv block %d" % j)


def test_backward_reproducibility():
    """dk and dv are bit-for-bit reproducible (one CTA owns each key group and
    adds its steps in a fixed order); dq is summed by reduce-adds from many
    CTAs in whatever order they land, so two runs agree only to rounding."""
    from block_sparse_attention_rope_b200 import api as a
    w = CASES["small_i2v"]
    x = synthetic.make_inputs(w)
    dout = synthetic.make_dout(w)
    g1 = run(a, w, x, dout)
    g2 = run(a, w, x, dout)
    assert torch.equal(g1[1], g2[1]) and torch.equal(g1[2], g2[2])
    d = (g1[0].float() - g2[0].float()).abs().max().item()
    assert d <= 2 ** -7 * g1[0].float().abs().max().item()


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_backward_custom_softmax_scale(dtype):
    from block_sparse_attention_rope_b200 import api as a
    w = Workload("sc", T=3, H=8, W=20, n_cond=1, heads=2, local=1, stride=2, dtype=dtype)
    x = synthetic.make_inputs(w)
    dout = synthetic.make_dout(w)
    d = {k: v.cuda() for k, v in x.items()}
    plan = a.Plan(w.T, w.H, w.W, local=w.local, stride=w.stride, n_cond=w.n_cond)
    rope = a.Rope3D(w.T, w.H, w.W)
    out, lse = a.forward(d["q"], d["k"], d["v"], plan, rope, return_lse=True, softmax_scale=0.3)
    grads = a.backward(d["q"], d["k"], d["v"], out, lse, dout.cuda(), plan, rope,
                       softmax_scale=0.3)
    torch.cuda.synchronize()
    assert a.last_device_status() == 0
    ref = ob.backward(x["q"], x["k"], x["v"], dout, T=w.T, H=w.H, W=w.W, n_cond=w.n_cond,
                      local=w.local, stride=w.stride, scale=0.3)
    for got, r, what in zip(grads, ref, ("dq", "dk", "dv")):
        assert_close(w, got, r, what, rms_scale=0.3 / 0.125)
