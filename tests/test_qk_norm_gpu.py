"""RMSNorm of q and k fused ahead of the 3D-RoPE (lc_bsa_forward_ex,
lc_bsa_forward_cached_ex, lc_bsa_cond_cache with lc_bsa_opts) against the fp64
oracle, plus the bit-for-bit agreements between the cached and uncached forms
(myzaker / QbitAI, "背后技术原理": RMSNorm in the attention modules; KV cache
of the condition tokens)."""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import parity
from block_sparse_attention_rope_b200 import synthetic
from block_sparse_attention_rope_b200.synthetic import Workload

pytestmark = pytest.mark.gpu

CASES = {
    "i2v_like": Workload("i2v_like", T=4, H=16, W=40, n_cond=1, heads=4, local=2, stride=4,
                         dtype="bf16"),
    "ragged": Workload("ragged", T=6, H=13, W=21, n_cond=1, heads=3, local=1, stride=3,
                       dtype="bf16"),
    "ragged_f32": Workload("ragged_f32", T=6, H=13, W=21, n_cond=1, heads=3, local=1, stride=3,
                           dtype="f32"),
    "cached": Workload("cached", T=5, H=8, W=20, n_cond=2, heads=2, local=1, stride=3,
                       dtype="bf16", cached=True),
    "cached_f32": Workload("cached_f32", T=5, H=8, W=20, n_cond=2, heads=2, local=1, stride=3,
                           dtype="f32", cached=True),
}
EPS = 1e-6


@pytest.fixture(scope="module")
def api():
    from block_sparse_attention_rope_b200 import build
    build.build()
    from block_sparse_attention_rope_b200 import api as a
    return a


def weights(seed):
    g = torch.Generator().manual_seed(seed)
    return 1.0 + 0.3 * torch.randn(64, generator=g, dtype=torch.float32)


def check(w, out, lse, ref_out, ref_lse):
    err = np.abs(out.cpu().double().numpy() - ref_out)
    lerr = np.abs(lse.cpu().double().numpy() - ref_lse).max()
    if w.dtype == "f32":
        assert err.max() <= parity.F32_MAX_ABS, err.max()
        assert lerr <= parity.F32_LSE_ABS, lerr
    else:
        assert err.max() <= parity.BF16_MAX_ABS, (err.max(), err.mean())
        assert err.mean() <= parity.BF16_MEAN_ABS, (err.max(), err.mean())
        assert lerr <= parity.BF16_LSE_ABS, lerr


@pytest.mark.parametrize("name", list(CASES))
def test_norm_matches_oracle(api, name):
    w = CASES[name]
    x = synthetic.make_inputs(w)
    d = {k: v.cuda() for k, v in x.items()}
    qn, kn = weights(7), weights(8)
    plan = api.Plan(w.T, w.H, w.W, local=w.local, stride=w.stride, n_cond=w.n_cond)
    rope = api.Rope3D(w.T, w.H, w.W)
    kw = dict(T=w.T, H=w.H, W=w.W, n_cond=w.n_cond, local=w.local, stride=w.stride,
              q_norm=qn.double().numpy(), k_norm=kn.double().numpy(), norm_eps=EPS)
    if w.cached:
        out, lse = api.forward_cached(d["q"], d["k"], d["v"], d["cond_k"], d["cond_v"], plan,
                                      rope, return_lse=True, q_norm=qn.cuda(), k_norm=kn.cuda(),
                                      norm_eps=EPS)
        ref = oracle.forward_cached(x["q"], x["k"], x["v"], x["cond_k"], x["cond_v"], **kw)
    else:
        out, lse = api.forward(d["q"], d["k"], d["v"], plan, rope, return_lse=True,
                               q_norm=qn.cuda(), k_norm=kn.cuda(), norm_eps=EPS)
        ref = oracle.forward(x["q"], x["k"], x["v"], **kw)
    torch.cuda.synchronize()
    assert api.last_device_status() == 0
    check(w, out, lse, *ref)
    # the norm changes the result (it is not silently skipped)
    plain = (api.forward_cached(d["q"], d["k"], d["v"], d["cond_k"], d["cond_v"], plan, rope)
             if w.cached else api.forward(d["q"], d["k"], d["v"], plan, rope))
    assert (plain.float() - out.float()).abs().max().item() > 1e-2


def test_norm_q_only_and_k_only(api):
    w = CASES["i2v_like"]
    x = synthetic.make_inputs(w)
    d = {k: v.cuda() for k, v in x.items()}
    plan = api.Plan(w.T, w.H, w.W, local=w.local, stride=w.stride, n_cond=w.n_cond)
    rope = api.Rope3D(w.T, w.H, w.W)
    base = dict(T=w.T, H=w.H, W=w.W, n_cond=w.n_cond, local=w.local, stride=w.stride,
                norm_eps=EPS)
    for side in ("q", "k"):
        wt = weights(11)
        gkw = {side + "_norm": wt.cuda()}
        okw = {side + "_norm": wt.double().numpy()}
        out, lse = api.forward(d["q"], d["k"], d["v"], plan, rope, return_lse=True,
                               norm_eps=EPS, **gkw)
        ref = oracle.forward(x["q"], x["k"], x["v"], **base, **okw)
        torch.cuda.synchronize()
        check(w, out, lse, *ref)


def test_norm_removes_input_scale(api):
    """With eps 0, scaling q and k by 64 (exact in bf16) leaves the output as is."""
    w = CASES["ragged"]
    d = synthetic.make_inputs(w, device="cuda")
    plan = api.Plan(w.T, w.H, w.W, local=w.local, stride=w.stride, n_cond=w.n_cond)
    rope = api.Rope3D(w.T, w.H, w.W)
    qn, kn = weights(3).cuda(), weights(4).cuda()
    o1 = api.forward(d["q"], d["k"], d["v"], plan, rope, q_norm=qn, k_norm=kn, norm_eps=0.0)
    o2 = api.forward(d["q"] * 64, d["k"] * 64, d["v"], plan, rope, q_norm=qn, k_norm=kn,
                     norm_eps=0.0)
    torch.cuda.synchronize()
    assert (o1.float() - o2.float()).abs().max().item() <= 1e-6


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_norm_with_condition_cache_bitwise(api, dtype):
    """cond_cache with the norm weights gives the condition rows of the normed
    whole-sequence forward, and the noisy step on its K equals the one on the
    raw condition K, bit for bit."""
    w = Workload("c", T=5, H=8, W=20, n_cond=2, heads=2, local=1, stride=3, dtype=dtype)
    x = synthetic.make_inputs(w)
    d = {k: v.cuda() for k, v in x.items()}
    plan = api.Plan(w.T, w.H, w.W, local=w.local, stride=w.stride, n_cond=w.n_cond)
    rope = api.Rope3D(w.T, w.H, w.W)
    qn, kn = weights(21).cuda(), weights(22).cuda()
    Nc = w.n_cond_tokens
    cq, ck, cv = (d[k][:, :Nc].contiguous() for k in ("q", "k", "v"))
    nq, nk, nv = (d[k][:, Nc:].contiguous() for k in ("q", "k", "v"))
    k_rot, c_out, c_lse = api.cond_cache(ck, plan, rope, cond_q=cq, cond_v=cv, return_lse=True,
                                         q_norm=qn, k_norm=kn, norm_eps=EPS)
    full_out, full_lse = api.forward(d["q"], d["k"], d["v"], plan, rope, return_lse=True,
                                     q_norm=qn, k_norm=kn, norm_eps=EPS)
    o_raw = api.forward_cached(nq, nk, nv, ck, cv, plan, rope, q_norm=qn, k_norm=kn,
                               norm_eps=EPS)
    o_cache = api.forward_cached(nq, nk, nv, k_rot, cv, plan, rope, cond_k_rotated=True,
                                 q_norm=qn, k_norm=kn, norm_eps=EPS)
    torch.cuda.synchronize()
    assert api.last_device_status() == 0
    assert torch.equal(c_out, full_out[:, :Nc]) and torch.equal(c_lse, full_lse[:, :, :Nc])
    assert torch.equal(o_cache, o_raw)
    assert torch.equal(o_raw, full_out[:, Nc:])
    # the cached K is R(norm(k)) of the oracle within rounding
    ref = oracle.rope3d_apply(oracle.rms_norm(x["k"][:, :Nc], kn.cpu().double().numpy(), EPS),
                              w.H, w.W)
    tol = (2.0 ** -8 if dtype == "bf16" else 1e-5) * np.abs(ref) + 1e-5
    assert np.all(np.abs(k_rot.cpu().double().numpy() - ref) <= tol)


def test_norm_option_errors(api):
    w = CASES["i2v_like"]
    plan = api.Plan(w.T, w.H, w.W, local=w.local, stride=w.stride, n_cond=w.n_cond)
    rope = api.Rope3D(w.T, w.H, w.W)
    t = torch.zeros(1, w.n_tokens, w.heads, 64, dtype=torch.bfloat16, device="cuda")
    o = torch.empty_like(t)
    wt = torch.ones(65, device="cuda")
    lib, INV = api.lib, 1

    def call(opts):
        return lib.lc_bsa_forward_ex(t.data_ptr(), t.data_ptr(), t.data_ptr(), o.data_ptr(),
                                     None, 1, w.heads, 64, 0, 0.0, ctypes.byref(opts),
                                     plan.handle, rope.handle, None)
    assert call(api.Opts(1, wt.data_ptr(), None, 1e-6)) == INV        # flags not allowed
    assert call(api.Opts(0, wt.data_ptr(), None, float("nan"))) == INV  # eps NaN
    assert call(api.Opts(0, None, wt.data_ptr(), -1.0)) == INV         # eps < 0
    assert call(api.Opts(0, wt.data_ptr() + 2, None, 1e-6)) == INV     # misaligned weight
    assert call(api.Opts(0, None, None, 0.0)) == 0                     # empty options
    torch.cuda.synchronize()
    with pytest.raises(ValueError):
        api.forward(t, t, t, plan, rope, q_norm=torch.ones(64))  # host tensor


def test_norm_full_size_sampled(api):
    """I2V 480p with RMSNorm weights (the <true> instantiation of the kernel at
    full size): every row of the sample of parity.sample_rows, heads 0 and 31."""
    w = synthetic.get("i2v_480p")
    x = synthetic.make_inputs(w)
    qn, kn = weights(31), weights(32)
    plan = api.Plan(w.T, w.H, w.W, local=w.local, stride=w.stride, n_cond=w.n_cond)
    rope = api.Rope3D(w.T, w.H, w.W)
    d = {k: v.cuda() for k, v in x.items()}
    out, lse = api.forward(d["q"], d["k"], d["v"], plan, rope, return_lse=True,
                           q_norm=qn.cuda(), k_norm=kn.cuda(), norm_eps=EPS)
    torch.cuda.synchronize()
    assert api.last_device_status() == 0
    rows = parity.sample_rows(w, n_random_blocks=16)
    heads = [0, w.heads - 1]
    sub = {k: v[:, :, heads].contiguous() for k, v in x.items()}
    trip = np.array([(0, h, r) for h in range(2) for r in rows], dtype=np.int64)
    ref_o, ref_l = oracle.attention_rows(
        sub["q"], sub["k"], sub["v"], H=w.H, W=w.W, Nc=w.n_cond_tokens, block=w.block,
        local=w.local, stride=w.stride, rows=trip, q_norm=qn.double().numpy(),
        k_norm=kn.double().numpy(), norm_eps=EPS)
    g = out[0][:, heads].float().cpu().numpy().astype(np.float64)   # [N, 2, 64]
    g = np.transpose(g[rows], (1, 0, 2)).reshape(-1, 64)
    err = np.abs(g - ref_o)
    assert err.max() <= parity.BF16_MAX_ABS and err.mean() <= parity.BF16_MEAN_ABS, \
        (err.max(), err.mean())
    gl = lse[0][heads][:, rows].cpu().numpy().astype(np.float64).reshape(-1)
    assert np.abs(gl - ref_l).max() <= parity.BF16_LSE_ABS
