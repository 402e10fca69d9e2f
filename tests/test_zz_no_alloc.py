"""lc_bsa_forward_noalloc: the attention entry point for callers that cannot
allocate device memory during the call (an allocator that owns the whole GPU,
a serving loop that forbids allocations after warm-up).  Its scheduler
counter and status word live in a fixed device array inside the library, so
this checks that two calls in a row, on different inputs, each give what the
allocating entry point lc_bsa_forward gives.

Kept in a file that pytest collects last, so that a run stopping at the first
failure has already run every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

import parity
from block_sparse_attention_rope_b200 import synthetic
from block_sparse_attention_rope_b200.synthetic import Workload

pytestmark = pytest.mark.gpu

W = Workload("noalloc", T=6, H=13, W=21, n_cond=1, heads=3, local=1, stride=3, dtype="bf16")


@pytest.fixture(scope="module")
def api():
    from block_sparse_attention_rope_b200 import build
    build.build()
    from block_sparse_attention_rope_b200 import api as a
    return a


def _call_noalloc_c_abi(api, q, k, v, out, lse, plan, rope):
    """Straight through the C ABI (ctypes), no Python-side help."""
    B, N, heads, hd = q.shape
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return api.lib.lc_bsa_forward_noalloc(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                                          lse.data_ptr(), B, heads, hd, api.LC_DTYPE_BF16,
                                          ctypes.c_float(0.0), plan.handle, rope.handle, stream)


def test_noalloc_matches_forward_on_two_calls_in_a_row(api):
    plan = api.Plan(W.T, W.H, W.W, local=W.local, stride=W.stride, n_cond=W.n_cond)
    rope = api.Rope3D(W.T, W.H, W.W)
    for call, seed in enumerate((0, 17)):
        x = {k: v.cuda() for k, v in synthetic.make_inputs(W, seed_offset=seed).items()}
        ref_out, ref_lse = api.forward(x["q"], x["k"], x["v"], plan, rope, return_lse=True)
        out = torch.zeros_like(x["q"])
        lse = torch.zeros(1, W.heads, W.n_tokens, dtype=torch.float32, device="cuda")
        st = _call_noalloc_c_abi(api, x["q"], x["k"], x["v"], out, lse, plan, rope)
        assert st == api.LC_OK, api.status_string(st)
        torch.cuda.synchronize()
        assert api.last_device_status() == api.LC_OK
        err = (out.float() - ref_out.float()).abs()
        assert err.max().item() <= parity.BF16_MAX_ABS, (call, err.max().item())
        assert err.mean().item() <= parity.BF16_MEAN_ABS, (call, err.mean().item())
        lerr = (lse - ref_lse).abs().max().item()
        assert lerr <= parity.BF16_LSE_ABS, (call, lerr)
        assert np.isfinite(out.float().cpu().numpy()).all()


def test_noalloc_draws_no_scratch_from_the_library_pool(api):
    """The allocating entry point draws its per-call scratch (rotated K, the
    scheduler counter) from the library's pool; the allocation-free one must
    not touch it.  The pool's high-water mark, reset to what is in use when
    no call is running, stays there across a noalloc call, while one
    lc_bsa_forward call raises it."""
    plan = api.Plan(W.T, W.H, W.W, local=W.local, stride=W.stride, n_cond=W.n_cond)
    rope = api.Rope3D(W.T, W.H, W.W)
    x = {k: v.cuda() for k, v in synthetic.make_inputs(W).items()}
    out = torch.zeros_like(x["q"])
    lse = torch.zeros(1, W.heads, W.n_tokens, dtype=torch.float32, device="cuda")
    api.forward(x["q"], x["k"], x["v"], plan, rope)  # the pool exists and holds nothing now
    torch.cuda.synchronize()
    base = api.scratch_pool_used_high(reset=True)
    assert _call_noalloc_c_abi(api, x["q"], x["k"], x["v"], out, lse, plan, rope) == api.LC_OK
    torch.cuda.synchronize()
    assert api.scratch_pool_used_high() == base
    api.forward(x["q"], x["k"], x["v"], plan, rope)
    torch.cuda.synchronize()
    assert api.scratch_pool_used_high() > base
    assert api.last_device_status() == api.LC_OK
