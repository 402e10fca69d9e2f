"""GPU attention (fp32 SIMT and bf16 tcgen05 kernels) against the fp64 oracle."""
import numpy as np
import pytest
import torch

import oracle
import parity
from block_sparse_attention_rope_b200 import synthetic
from block_sparse_attention_rope_b200.synthetic import Workload

pytestmark = pytest.mark.gpu

SMALL = {
    # several 256-row groups, a condition frame, ragged nothing
    "small_i2v": Workload("small_i2v", T=4, H=16, W=40, n_cond=1, heads=4, local=2, stride=4,
                          dtype="bf16"),
    # partial blocks at the end of both segments (273 tokens per frame)
    "ragged": Workload("ragged", T=6, H=13, W=21, n_cond=1, heads=3, local=1, stride=3,
                       dtype="bf16"),
    "dense_small": Workload("dense_small", T=3, H=16, W=32, n_cond=0, heads=2, local=0, stride=1,
                            dtype="bf16"),
    "local_only": Workload("local_only", T=2, H=10, W=30, n_cond=0, heads=2, local=0, stride=0,
                           dtype="bf16"),
    "batch2": Workload("batch2", T=3, H=8, W=24, n_cond=1, heads=2, local=1, stride=2,
                       dtype="bf16", batch=2),
    "many_heads": Workload("many_heads", T=2, H=8, W=32, n_cond=0, heads=32, local=2, stride=4,
                           dtype="bf16"),
    "one_block": Workload("one_block", T=1, H=5, W=12, n_cond=0, heads=2, local=2, stride=4,
                          dtype="bf16"),
    "cached_small": Workload("cached_small", T=5, H=8, W=20, n_cond=2, heads=2, local=1,
                             stride=3, dtype="bf16", cached=True),
    "cached_ragged": Workload("cached_ragged", T=4, H=7, W=19, n_cond=1, heads=2, local=2,
                              stride=4, dtype="bf16", cached=True),
    "ragged_f32": Workload("ragged_f32", T=6, H=13, W=21, n_cond=1, heads=3, local=1, stride=3,
                           dtype="f32"),
    # degenerate shapes: a noisy segment shorter than one block after three
    # condition frames; one token row per frame (both segments one partial
    # block); a stride past the last block (block 0 is the only global one)
    "short_noisy": Workload("short_noisy", T=4, H=6, W=10, n_cond=3, heads=2, local=1, stride=2,
                            dtype="bf16"),
    "short_noisy_cached": Workload("short_noisy_cached", T=4, H=6, W=10, n_cond=3, heads=2,
                                   local=1, stride=2, dtype="bf16", cached=True),
    "tiny_tokens": Workload("tiny_tokens", T=5, H=1, W=7, n_cond=2, heads=2, local=0, stride=3,
                            dtype="bf16"),
    "tiny_tokens_f32": Workload("tiny_tokens_f32", T=5, H=1, W=7, n_cond=2, heads=2, local=0,
                                stride=3, dtype="f32"),
    "stride_past_end": Workload("stride_past_end", T=3, H=8, W=16, n_cond=0, heads=2, local=0,
                                stride=100, dtype="bf16"),
    "local1": Workload("local1", T=4, H=12, W=32, n_cond=0, heads=2, local=1, stride=0,
                       dtype="bf16"),
    # the cached form with no condition frames (no cond_k / cond_v at all)
    "cached_nocond": Workload("cached_nocond", T=3, H=8, W=24, n_cond=0, heads=2, local=1,
                              stride=2, dtype="bf16", cached=True),
    "cached_nocond_f32": Workload("cached_nocond_f32", T=3, H=8, W=24, n_cond=0, heads=2,
                                  local=1, stride=2, dtype="f32", cached=True),
    "cached_f32": Workload("cached_f32", T=5, H=8, W=20, n_cond=2, heads=2, local=1, stride=3,
                           dtype="f32", cached=True),
}


@pytest.fixture(scope="module")
def api():
    from block_sparse_attention_rope_b200 import build
    build.build()
    from block_sparse_attention_rope_b200 import api as a
    return a


def run_gpu(api, w, inputs):
    plan = api.Plan(w.T, w.H, w.W, local=w.local, stride=w.stride, n_cond=w.n_cond)
    rope = api.Rope3D(w.T, w.H, w.W)
    d = {k: v.cuda() for k, v in inputs.items()}
    if w.cached:
        out, lse = api.forward_cached(d["q"], d["k"], d["v"], d.get("cond_k"), d.get("cond_v"),
                                      plan, rope, return_lse=True)
    else:
        out, lse = api.forward(d["q"], d["k"], d["v"], plan, rope, return_lse=True)
    torch.cuda.synchronize()
    assert api.last_device_status() == 0
    return out.cpu(), lse.cpu()


def full_oracle(w, inputs):
    kw = dict(T=w.T, H=w.H, W=w.W, n_cond=w.n_cond, local=w.local, stride=w.stride)
    if w.cached:
        return oracle.forward_cached(inputs["q"], inputs["k"], inputs["v"], inputs["cond_k"],
                                     inputs["cond_v"], **kw)
    return oracle.forward(inputs["q"], inputs["k"], inputs["v"], **kw)


def check_all_rows(w, out, lse, ref_out, ref_lse):
    g = out.float().numpy().astype(np.float64)
    err = np.abs(g - ref_out)
    lerr = np.abs(lse.numpy().astype(np.float64) - ref_lse).max()
    if w.dtype == "f32":
        assert err.max() <= parity.F32_MAX_ABS, err.max()
        assert lerr <= parity.F32_LSE_ABS, lerr
    else:
        assert err.max() <= parity.BF16_MAX_ABS, (err.max(), err.mean())
        assert err.mean() <= parity.BF16_MEAN_ABS, (err.max(), err.mean())
        assert lerr <= parity.BF16_LSE_ABS, lerr
    return err.max(), err.mean(), lerr


def test_tiny_f32_all_rows(api):
    w = synthetic.get("tiny_f32")
    inputs = synthetic.make_inputs(w)
    out, lse = run_gpu(api, w, inputs)
    ref_out, ref_lse = full_oracle(w, inputs)
    mx, mean, lerr = check_all_rows(w, out, lse, ref_out, ref_lse)
    print("tiny_f32 max %.3g mean %.3g lse %.3g" % (mx, mean, lerr))


@pytest.mark.parametrize("name", sorted(SMALL))
def test_small_all_rows(api, name):
    w = SMALL[name]
    inputs = synthetic.make_inputs(w)
    out, lse = run_gpu(api, w, inputs)
    assert torch.isfinite(out.float()).all()
    ref_out, ref_lse = full_oracle(w, inputs)
    mx, mean, lerr = check_all_rows(w, out, lse, ref_out, ref_lse)
    print("%s max %.3g mean %.3g lse %.3g" % (name, mx, mean, lerr))


@pytest.mark.parametrize("name,qscale", [("small_i2v", 4.0), ("ragged", 8.0), ("dense_small", 6.0),
                                         ("local_only", 6.0), ("local1", 6.0)])
def test_large_logits_exercise_rescaling(api, name, qscale):
    """Scaled queries give logits with a wide range, so the running maximum
    moves often and the kernel's rescaling path (new reference max, O and l
    rescaled, P recomputed) runs on many tiles.  With no condition frame and
    no global blocks (local_only, local1) the first key tile of a 4-block
    group is fully masked for some member rows, which then meet their first
    attended key -- and possibly a rescale -- in a later tile."""
    w = SMALL[name]
    inputs = synthetic.make_inputs(w)
    inputs["q"] = (inputs["q"].float() * qscale).to(inputs["q"].dtype)
    out, lse = run_gpu(api, w, inputs)
    ref_out, ref_lse = full_oracle(w, inputs)
    g = out.float().numpy().astype(np.float64)
    err = np.abs(g - ref_out)
    # outputs are larger and sharper here; bf16 rounding of R(q), R(k) moves
    # logits by up to ~|s| * 2^-8, so the bound against the exact oracle
    # scales with the query scale.
    assert err.max() <= parity.BF16_MAX_ABS * qscale, err.max()
    assert err.mean() <= parity.BF16_MEAN_ABS * qscale, err.mean()
    assert np.abs(lse.numpy() - ref_lse).max() <= parity.BF16_LSE_ABS * qscale
    # Against the oracle on bf16-rounded R(q), R(k) the logit rounding is
    # gone, so bounds that do not grow with the logits apply: a fault in the
    # rescaling (a wrong correction factor, a lost or doubled P) shows here.
    r_out, r_lse = parity.oracle_on_rounded_operands(w, inputs)
    rmx, rmean, rl = parity.assert_rounded_operand_close(g, lse.numpy(), r_out, r_lse,
                                                         inputs["v"])
    print("%s x%g: exact max %.3g mean %.3g | rounded-operand max %.3g mean %.3g lse %.3g" %
          (name, qscale, err.max(), err.mean(), rmx, rmean, rl))


@pytest.mark.parametrize("name", ["small_i2v", "ragged", "many_heads", "batch2"])
def test_in_kernel_k_rotation_path(api, name):
    """The allocation-free entry point rotates each loaded K tile in shared
    memory (no pre-rotated copy of K); check that path against the oracle."""
    w = SMALL[name]
    inputs = synthetic.make_inputs(w)
    plan = api.Plan(w.T, w.H, w.W, local=w.local, stride=w.stride, n_cond=w.n_cond)
    rope = api.Rope3D(w.T, w.H, w.W)
    d = {k: v.cuda() for k, v in inputs.items()}
    out = torch.empty_like(d["q"])
    lse = torch.empty(w.batch, w.heads, w.n_tokens, device="cuda")
    api.forward_noalloc(d["q"], d["k"], d["v"], plan, rope, out=out, lse=lse)
    torch.cuda.synchronize()
    assert api.last_device_status() == 0
    ref_out, ref_lse = full_oracle(w, inputs)
    check_all_rows(w, out.cpu(), lse.cpu(), ref_out, ref_lse)


def test_in_kernel_k_rotation_full_size_sampled(api):
    w = synthetic.get("i2v_480p")
    inputs = synthetic.make_inputs(w)
    plan = api.Plan(w.T, w.H, w.W, local=w.local, stride=w.stride, n_cond=w.n_cond)
    rope = api.Rope3D(w.T, w.H, w.W)
    d = {k: v.cuda() for k, v in inputs.items()}
    out = torch.empty_like(d["q"])
    lse = torch.empty(w.batch, w.heads, w.n_tokens, device="cuda")
    api.forward_noalloc(d["q"], d["k"], d["v"], plan, rope, out=out, lse=lse)
    torch.cuda.synchronize()
    assert api.last_device_status() == 0
    rows = parity.sample_rows(w, n_random_blocks=16)
    ref_out, ref_lse = parity.oracle_rows(w, inputs, rows)
    parity.compare(w, out.cpu(), lse.cpu(), ref_out, ref_lse, rows)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_cached_equals_noisy_rows_of_forward(api, dtype):
    w = Workload("x", T=5, H=8, W=24, n_cond=2, heads=3, local=1, stride=3, dtype=dtype)
    full = synthetic.make_inputs(w)
    out_full, lse_full = run_gpu(api, w, full)
    Nc = w.n_cond_tokens
    cin = {"q": full["q"][:, Nc:].contiguous(), "k": full["k"][:, Nc:].contiguous(),
           "v": full["v"][:, Nc:].contiguous(), "cond_k": full["k"][:, :Nc].contiguous(),
           "cond_v": full["v"][:, :Nc].contiguous()}
    wc = Workload("xc", T=5, H=8, W=24, n_cond=2, heads=3, local=1, stride=3, dtype=dtype,
                  cached=True)
    out_c, lse_c = run_gpu(api, wc, cin)
    assert torch.equal(out_c, out_full[:, Nc:])
    assert torch.equal(lse_c, lse_full[:, :, Nc:])


def test_condition_rows_ignore_noise_tokens(api):
    w = SMALL["small_i2v"]
    inputs = synthetic.make_inputs(w)
    out1, lse1 = run_gpu(api, w, inputs)
    Nc = w.n_cond_tokens
    g = torch.Generator().manual_seed(77)
    pert = {k: v.clone() for k, v in inputs.items()}
    for k in ("q", "k", "v"):
        pert[k][:, Nc:] = torch.randn(pert[k][:, Nc:].shape, generator=g).to(pert[k].dtype)
    out2, lse2 = run_gpu(api, w, pert)
    assert torch.equal(out1[:, :Nc], out2[:, :Nc])
    assert torch.equal(lse1[:, :, :Nc], lse2[:, :, :Nc])
    assert not torch.equal(out1[:, Nc:], out2[:, Nc:])


def test_deterministic(api):
    w = SMALL["ragged"]
    inputs = synthetic.make_inputs(w)
    a, la = run_gpu(api, w, inputs)
    b, lb = run_gpu(api, w, inputs)
    assert torch.equal(a, b) and torch.equal(la, lb)


FULL = ["i2v_480p", "refine_720p", "continuation_cached", "sweep_dense", "sweep_l2s4",
        "sweep_l2s8", "sweep_l1s16", "sweep_l1s32"]


@pytest.mark.parametrize("name", FULL)
def test_full_size_sampled_rows(api, name):
    """Full-size workloads in the benchmark's launch configuration; every head
    on a fixed sample of query rows (see parity.sample_rows)."""
    w = synthetic.get(name)
    inputs = synthetic.make_inputs(w)
    out, lse = run_gpu(api, w, inputs)
    assert torch.isfinite(out.float()).all() and torch.isfinite(lse).all()
    nrand = 8 if name == "sweep_dense" else 64
    rows = parity.sample_rows(w, n_random_blocks=nrand)
    ref_out, ref_lse = parity.oracle_rows(w, inputs, rows)
    mx, mean, lerr = parity.compare(w, out, lse, ref_out, ref_lse, rows)
    print("%s rows=%d x %d heads: max %.3g mean %.3g lse %.3g" % (name, len(rows), w.heads, mx,
                                                                  mean, lerr))


@pytest.mark.parametrize("name", ["i2v_480p", "refine_720p", "continuation_cached"])
def test_full_size_all_rows_of_two_heads(api, name):
    """Every query row of heads 0 and 31 at full size (the benchmark's launch),
    element by element against the oracle; for the cached form the rows are
    the noisy queries over the cached condition keys plus the noisy keys."""
    w = synthetic.get(name)
    inputs = synthetic.make_inputs(w)
    out, lse = run_gpu(api, w, inputs)
    heads = [0, w.heads - 1]
    nq = w.n_noisy_tokens if w.cached else w.n_tokens
    sub = {k: v[:, :, heads].contiguous() for k, v in inputs.items()}
    ref_out, ref_lse = parity.oracle_rows(w, sub, np.arange(nq), heads=[0, 1])
    mx, mean, lerr = parity.compare(w, out, lse, ref_out, ref_lse, np.arange(nq), heads=heads)
    print("%s all rows of heads %s: max %.3g mean %.3g lse %.3g" % (name, heads, mx, mean, lerr))


def test_argument_errors_on_gpu(api):
    w = SMALL["small_i2v"]
    plan = api.Plan(w.T, w.H, w.W, local=w.local, stride=w.stride, n_cond=w.n_cond)
    rope = api.Rope3D(w.T, w.H, w.W)
    other = api.Rope3D(w.T, w.H, w.W + 1)
    q = torch.randn(1, w.n_tokens, w.heads, 64, device="cuda").bfloat16()
    with pytest.raises(api.LcError) as e:
        api.forward(q, q, q, plan, other)
    assert e.value.status == api.LC_ERR_INVALID_ARGUMENT
    # a pointer that is not 16-byte aligned
    buf = torch.empty(w.n_tokens * w.heads * 64 + 8, device="cuda", dtype=torch.bfloat16)
    mis = buf[1:1 + w.n_tokens * w.heads * 64].view(1, w.n_tokens, w.heads, 64)
    with pytest.raises(api.LcError) as e:
        api.forward(mis, q, q, plan, rope)
    assert e.value.status == api.LC_ERR_INVALID_ARGUMENT
    assert api.last_device_status() == 0


def test_watchdog_gives_up_and_context_survives(api):
    """A bounded wait on a barrier that nothing arrives on reports a timeout
    instead of hanging; the context keeps working afterwards."""
    assert api.watchdog_selftest(20000) == api.LC_ERR_TIMEOUT
    assert api.last_device_status() == 0
    w = SMALL["one_block"]
    inputs = synthetic.make_inputs(w)
    out, lse = run_gpu(api, w, inputs)
    ref_out, ref_lse = full_oracle(w, inputs)
    check_all_rows(w, out, lse, ref_out, ref_lse)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_custom_softmax_scale(api, dtype):
    """A softmax scale other than 1/sqrt(64), forward and cached forms."""
    w = Workload("sc", T=4, H=8, W=24, n_cond=1, heads=2, local=1, stride=2, dtype=dtype)
    x = synthetic.make_inputs(w)
    plan = api.Plan(w.T, w.H, w.W, local=w.local, stride=w.stride, n_cond=w.n_cond)
    rope = api.Rope3D(w.T, w.H, w.W)
    d = {k: v.cuda() for k, v in x.items()}
    out, lse = api.forward(d["q"], d["k"], d["v"], plan, rope, return_lse=True,
                           softmax_scale=0.3)
    Nc = w.n_cond_tokens
    oc, lc = api.forward_cached(d["q"][:, Nc:].contiguous(), d["k"][:, Nc:].contiguous(),
                                d["v"][:, Nc:].contiguous(), d["k"][:, :Nc].contiguous(),
                                d["v"][:, :Nc].contiguous(), plan, rope, return_lse=True,
                                softmax_scale=0.3)
    torch.cuda.synchronize()
    assert api.last_device_status() == 0
    ref_o, ref_l = oracle.forward(x["q"], x["k"], x["v"], T=w.T, H=w.H, W=w.W, n_cond=w.n_cond,
                                  local=w.local, stride=w.stride, scale=0.3)
    if dtype == "f32":
        check_all_rows(w, out.cpu(), lse.cpu(), ref_o, ref_l)
    else:
        # logits 2.4x those of the default scale: the bf16 rounding of R(q),
        # R(k) moves them 2.4x as far (as in the large-logit test)
        err = np.abs(out.cpu().float().numpy().astype(np.float64) - ref_o)
        k = 0.3 / 0.125
        assert err.max() <= parity.BF16_MAX_ABS * k and err.mean() <= parity.BF16_MEAN_ABS * k
        assert np.abs(lse.cpu().numpy() - ref_l).max() <= parity.BF16_LSE_ABS * k
        # with the logit rounding modelled, the plain bf16 bounds
        r_o, r_l = parity.oracle_on_rounded_operands(w, x, scale=0.3)
        rmx, rmean, rl = parity.assert_rounded_operand_close(
            out.cpu().float().numpy(), lse.cpu().numpy(), r_o, r_l, x["v"])
        print("scale 0.3: exact max %.3g mean %.3g | rounded-operand max %.3g mean %.3g lse %.3g"
              % (err.max(), err.mean(), rmx, rmean, rl))
    assert torch.equal(oc, out[:, Nc:]) and torch.equal(lc, lse[:, :, Nc:])
