"""The condition-token KV cache (lc_bsa_cond_cache, lc_bsa_forward_cached_ex).

Condition tokens never attend noise tokens (myzaker / QbitAI "背后技术原理",
block attention with a KV cache), so their rotated K and their own attention
outputs can be produced once and reused.  Checked here:
  - cond_k_rot is the RoPE of cond_k: bit for bit the library's public
    rotation, and within bf16 rounding of the fp64 oracle's rotation;
  - cond_out / cond_lse are the condition rows of lc_bsa_forward on the whole
    sequence, bit for bit, and match the oracle within the parity tolerances;
  - lc_bsa_forward_cached_ex on the cached cond_k_rot gives the bits of
    lc_bsa_forward_cached on the pre-RoPE cond_k;
  - argument errors.
"""
import numpy as np
import pytest
import torch

import oracle
import parity
from block_sparse_attention_rope_b200 import synthetic
from block_sparse_attention_rope_b200.synthetic import Workload

pytestmark = pytest.mark.gpu

CASES = {
    "one_cond_frame": Workload("one_cond_frame", T=4, H=16, W=40, n_cond=1, heads=4, local=2,
                               stride=4, dtype="bf16"),
    # 273 tokens per frame: the condition segment ends in a partial block
    "ragged": Workload("ragged", T=6, H=13, W=21, n_cond=1, heads=3, local=1, stride=3,
                       dtype="bf16"),
    # five condition blocks: two query groups in the condition segment
    "two_cond_frames": Workload("two_cond_frames", T=5, H=8, W=20, n_cond=2, heads=2, local=1,
                                stride=3, dtype="bf16", batch=2),
    "ragged_f32": Workload("ragged_f32", T=6, H=13, W=21, n_cond=1, heads=3, local=1, stride=3,
                           dtype="f32"),
}


@pytest.fixture(scope="module")
def api():
    from block_sparse_attention_rope_b200 import build
    build.build()
    from block_sparse_attention_rope_b200 import api as a
    return a


def split(w, d):
    Nc = w.n_cond_tokens
    return ({k: d[k][:, :Nc].contiguous() for k in ("q", "k", "v")},
            {k: d[k][:, Nc:].contiguous() for k in ("q", "k", "v")})


@pytest.mark.parametrize("name", list(CASES))
def test_cond_cache_matches_forward_and_oracle(api, name):
    w = CASES[name]
    x = synthetic.make_inputs(w)
    d = {k: v.cuda() for k, v in x.items()}
    plan = api.Plan(w.T, w.H, w.W, local=w.local, stride=w.stride, n_cond=w.n_cond)
    rope = api.Rope3D(w.T, w.H, w.W)
    cond, noisy = split(w, d)
    k_rot, c_out, c_lse = api.cond_cache(cond["k"], plan, rope, cond_q=cond["q"],
                                         cond_v=cond["v"], return_lse=True)
    full_out, full_lse = api.forward(d["q"], d["k"], d["v"], plan, rope, return_lse=True)
    torch.cuda.synchronize()
    assert api.last_device_status() == 0
    Nc = w.n_cond_tokens
    # rotation: the public entry point's bits, and the oracle within rounding
    assert torch.equal(k_rot, rope.apply(cond["k"]))
    ref_rot = oracle.rope3d_apply(x["k"][:, :Nc], w.H, w.W)
    g = k_rot.cpu().double().numpy()
    tol = (2.0 ** -8 if w.dtype == "bf16" else 1e-6) * np.abs(ref_rot) + 1e-6
    assert np.all(np.abs(g - ref_rot) <= tol)
    # condition rows of the whole-sequence forward, bit for bit
    assert torch.equal(c_out, full_out[:, :Nc])
    assert torch.equal(c_lse, full_lse[:, :, :Nc])
    # and the oracle on every condition row of every head
    ref = oracle.forward(x["q"], x["k"], x["v"], T=w.T, H=w.H, W=w.W, n_cond=w.n_cond,
                         local=w.local, stride=w.stride)
    err = np.abs(c_out.cpu().double().numpy() - ref[0][:, :Nc])
    lerr = np.abs(c_lse.cpu().double().numpy() - ref[1][:, :, :Nc]).max()
    if w.dtype == "f32":
        assert err.max() <= parity.F32_MAX_ABS and lerr <= parity.F32_LSE_ABS
    else:
        assert err.max() <= parity.BF16_MAX_ABS and err.mean() <= parity.BF16_MEAN_ABS
        assert lerr <= parity.BF16_LSE_ABS
    # the noisy step on the cached, already rotated K
    o_ref, l_ref = api.forward_cached(noisy["q"], noisy["k"], noisy["v"], cond["k"], cond["v"],
                                      plan, rope, return_lse=True)
    o_ex, l_ex = api.forward_cached(noisy["q"], noisy["k"], noisy["v"], k_rot, cond["v"], plan,
                                    rope, return_lse=True, cond_k_rotated=True)
    torch.cuda.synchronize()
    assert api.last_device_status() == 0
    assert torch.equal(o_ex, o_ref) and torch.equal(l_ex, l_ref)


def test_cond_cache_rotation_only(api):
    w = CASES["two_cond_frames"]
    x = synthetic.make_inputs(w, device="cuda")
    plan = api.Plan(w.T, w.H, w.W, local=w.local, stride=w.stride, n_cond=w.n_cond)
    rope = api.Rope3D(w.T, w.H, w.W)
    ck = x["k"][:, :w.n_cond_tokens].contiguous()
    k_rot = api.cond_cache(ck, plan, rope)
    assert torch.equal(k_rot, rope.apply(ck))


def test_cond_cache_no_condition_frames(api):
    w = Workload("t2v", T=3, H=8, W=16, n_cond=0, heads=2, local=1, stride=2, dtype="bf16")
    plan = api.Plan(w.T, w.H, w.W, local=w.local, stride=w.stride, n_cond=0)
    rope = api.Rope3D(w.T, w.H, w.W)
    empty = torch.empty(1, 0, 2, 64, dtype=torch.bfloat16, device="cuda")
    assert api.cond_cache(empty, plan, rope).shape == (1, 0, 2, 64)


def test_cond_cache_errors(api):
    import ctypes
    w = CASES["one_cond_frame"]
    plan = api.Plan(w.T, w.H, w.W, local=w.local, stride=w.stride, n_cond=w.n_cond)
    rope = api.Rope3D(w.T, w.H, w.W)
    Nc = w.n_cond_tokens
    t = torch.zeros(1, Nc, w.heads, 64, dtype=torch.bfloat16, device="cuda")
    big = torch.zeros(1, 2 * Nc, w.heads, 64, dtype=torch.bfloat16, device="cuda")
    lib, INV = api.lib, 1
    # cond_k_rot overlapping cond_k
    assert lib.lc_bsa_cond_cache(None, big.data_ptr(), None, big[:, 1:].data_ptr(), None, None,
                                 1, w.heads, 64, 0, 0.0, None, plan.handle, rope.handle,
                                 None) == INV
    # lse without an output, output without q/v
    lse = torch.zeros(1, w.heads, Nc, device="cuda")
    k_rot = torch.empty_like(t)
    assert lib.lc_bsa_cond_cache(None, t.data_ptr(), None, k_rot.data_ptr(), None,
                                 lse.data_ptr(), 1, w.heads, 64, 0, 0.0, None, plan.handle,
                                 rope.handle, None) == INV
    assert lib.lc_bsa_cond_cache(None, t.data_ptr(), t.data_ptr(), k_rot.data_ptr(),
                                 torch.empty_like(t).data_ptr(), None, 1, w.heads, 64, 0, 0.0,
                                 None, plan.handle, rope.handle, None) == INV
    # unknown flag bits
    n = torch.zeros(1, w.n_noisy_tokens, w.heads, 64, dtype=torch.bfloat16, device="cuda")
    assert lib.lc_bsa_forward_cached_ex(n.data_ptr(), n.data_ptr(), n.data_ptr(), t.data_ptr(),
                                        t.data_ptr(), torch.empty_like(n).data_ptr(), None, 1,
                                        w.heads, 64, 0, 0.0, ctypes.byref(api.Opts(6)),
                                        plan.handle, rope.handle, None) == INV
    # cond_cache takes no flags
    assert lib.lc_bsa_cond_cache(None, t.data_ptr(), None, k_rot.data_ptr(), None, None, 1,
                                 w.heads, 64, 0, 0.0, ctypes.byref(api.Opts(1)), plan.handle,
                                 rope.handle, None) == INV
    with pytest.raises(ValueError):
        api.cond_cache(t, plan, rope, cond_q=t)  # cond_v missing


def test_cond_cache_continuation_full_size(api):
    """The continuation workload (8 condition frames, 12,480 condition tokens,
    32 heads): the cache's condition rows equal the whole-sequence forward's
    bit for bit, sampled rows match the oracle, and the noisy step on the
    cached K equals the uncached one."""
    c = synthetic.get("continuation_cached")
    w = Workload("continuation_full", T=c.T, H=c.H, W=c.W, n_cond=c.n_cond, heads=c.heads,
                 local=c.local, stride=c.stride, dtype="bf16")
    x = synthetic.make_inputs(w)
    d = {k: v.cuda() for k, v in x.items()}
    plan = api.Plan(w.T, w.H, w.W, local=w.local, stride=w.stride, n_cond=w.n_cond)
    rope = api.Rope3D(w.T, w.H, w.W)
    cond, noisy = split(w, d)
    k_rot, c_out, c_lse = api.cond_cache(cond["k"], plan, rope, cond_q=cond["q"],
                                         cond_v=cond["v"], return_lse=True)
    full_out, full_lse = api.forward(d["q"], d["k"], d["v"], plan, rope, return_lse=True)
    torch.cuda.synchronize()
    assert api.last_device_status() == 0
    Nc = w.n_cond_tokens
    assert torch.equal(c_out, full_out[:, :Nc]) and torch.equal(c_lse, full_lse[:, :, :Nc])
    del full_out, full_lse
    o_ref = api.forward_cached(noisy["q"], noisy["k"], noisy["v"], cond["k"], cond["v"], plan,
                               rope)
    o_ex = api.forward_cached(noisy["q"], noisy["k"], noisy["v"], k_rot, cond["v"], plan, rope,
                              cond_k_rotated=True)
    torch.cuda.synchronize()
    assert torch.equal(o_ex, o_ref)
    # sampled condition rows against the oracle (two heads)
    rows = np.unique(np.concatenate([np.arange(0, 64), np.arange(Nc - 64, Nc),
                                     np.random.default_rng(3).integers(0, Nc, 64)]))
    ref_o, ref_l = parity.oracle_rows(w, x, rows, heads=[0, 31])
    g = c_out[0, rows][:, [0, 31]].cpu().double().numpy().transpose(1, 0, 2)
    err = np.abs(g - ref_o)
    assert err.max() <= parity.BF16_MAX_ABS and err.mean() <= parity.BF16_MEAN_ABS
    gl = c_lse[0][[0, 31]][:, rows].cpu().double().numpy()
    assert np.abs(gl - ref_l).max() <= parity.BF16_LSE_ABS
