"""Helpers shared by the GPU parity tests: tolerances, row sampling, and the
comparison of GPU outputs with the fp64 oracle."""
import numpy as np
import torch

import oracle

# Tolerances on |gpu - oracle| of the attention output (N(0,1) inputs).
F32_MAX_ABS = 1e-4
BF16_MAX_ABS = 1.5e-2
BF16_MEAN_ABS = 1e-3
# LSE (natural log): fp32 path, and the bf16 path (rounded q/k/P).
F32_LSE_ABS = 1e-4
BF16_LSE_ABS = 5e-2
# The bf16 path against the oracle on bf16-rounded R(q), R(k)
# (oracle_on_rounded_operands), any logit scale.  What is left is (a) P's
# rounding to bf16, at most 2^-8 p_j relative per key, so at most
# 2^-8 max|v| on an output; (b) the output's rounding, at most 2^-8 |o|; and
# (c) the rare R(q) / R(k) element whose fp32 rotation rounds to the other
# bf16 neighbour than the fp64 one (a few per 10^5 elements), which moves its
# logits by one bf16 step: allowed 2e-3 on outputs, 5e-3 on the LSE (whose l
# is summed from unrounded fp32 exp2 values, so (a) and (b) do not reach it).
# Mean: random-sign roundings of (a) and (b), measured 0.7-0.9e-3 at query
# scales 4-8; 1.5e-3 catches a doubling.
BF16_ROUNDED_MEAN_ABS = 1.5e-3
BF16_ROUNDED_LSE_ABS = 5e-3


def assert_rounded_operand_close(gpu_out, gpu_lse, r_out, r_lse, v):
    """Asserts the bounds above; returns (max, mean, lse) errors."""
    err = np.abs(np.asarray(gpu_out, dtype=np.float64) - r_out)
    vmax = float(np.abs(oracle._f64(v)).max())
    bound = 2.0 ** -8 * (vmax + np.abs(r_out)) + 2e-3
    lerr = float(np.abs(np.asarray(gpu_lse, dtype=np.float64) - r_lse).max())
    assert np.all(err <= bound), (err.max(), float((err - bound).max()))
    assert err.mean() <= BF16_ROUNDED_MEAN_ABS, err.mean()
    assert lerr <= BF16_ROUNDED_LSE_ABS, lerr
    return float(err.max()), float(err.mean()), lerr


def sample_rows(w, n_random_blocks=64, rows_per_random_block=4, seed=0):
    """Query rows (indices into the q tensor) for full-size checks: every row
    of the first and last blocks of each segment, of the partial tail blocks,
    of the blocks on both sides of the condition/noise boundary, of one global
    column block and one middle block; plus a few rows of seeded random
    blocks.  Returns a sorted int array."""
    rng = np.random.default_rng(seed)
    Nc, Nn = w.n_cond_tokens, w.n_noisy_tokens
    nq_tokens = Nn if w.cached else Nc + Nn
    base_noisy = 0 if w.cached else Nc
    blocks = set()
    nb = -(-Nn // 64)
    for j in [0, 1, nb // 2, nb - 2, nb - 1, w.stride if w.stride > 1 else 2]:
        if 0 <= j < nb:
            lo = base_noisy + 64 * j
            blocks.update(range(lo, min(base_noisy + Nn, lo + 64)))
    if not w.cached and Nc > 0:
        cb = -(-Nc // 64)
        for j in [0, cb - 1]:
            lo = 64 * j
            blocks.update(range(lo, min(Nc, lo + 64)))
    for j in rng.integers(0, nb, size=n_random_blocks):
        lo = base_noisy + 64 * int(j)
        hi = min(base_noisy + Nn, lo + 64)
        blocks.update(int(x) for x in rng.integers(lo, hi, size=rows_per_random_block))
    rows = np.array(sorted(r for r in blocks if 0 <= r < nq_tokens), dtype=np.int64)
    return rows


def oracle_rows(w, inputs, rows, heads=None):
    """Oracle outputs for the given q-tensor rows of every head in `heads`.
    Returns (out [len(heads), R, 64], lse [len(heads), R])."""
    heads = list(range(w.heads)) if heads is None else list(heads)
    if w.cached:
        k = np.concatenate([oracle._f64(inputs["cond_k"]), oracle._f64(inputs["k"])], axis=1)
        v = np.concatenate([oracle._f64(inputs["cond_v"]), oracle._f64(inputs["v"])], axis=1)
        q_off = w.n_cond_tokens
    else:
        k, v, q_off = inputs["k"], inputs["v"], 0
    trip = np.array([(0, h, r) for h in heads for r in rows], dtype=np.int64)
    o, l = oracle.attention_rows(inputs["q"], k, v, H=w.H, W=w.W, Nc=w.n_cond_tokens,
                                 block=w.block, local=w.local, stride=w.stride, rows=trip,
                                 q_offset=q_off)
    return o.reshape(len(heads), len(rows), -1), l.reshape(len(heads), len(rows))


def compare(w, gpu_out, gpu_lse, ref_out, ref_lse, rows, heads=None):
    """Element-wise comparison; returns (max_abs, mean_abs, max_lse_abs) and
    asserts the tolerances of the workload's dtype."""
    heads = list(range(w.heads)) if heads is None else list(heads)
    g = gpu_out[0][:, heads].float().cpu().numpy()         # [N, H, 64]
    g = np.transpose(g[rows], (1, 0, 2)).astype(np.float64)  # [H, R, 64]
    err = np.abs(g - ref_out)
    max_abs, mean_abs = float(err.max()), float(err.mean())
    lse_err = None
    if gpu_lse is not None:
        gl = gpu_lse[0][heads][:, rows].cpu().numpy().astype(np.float64)
        lse_err = float(np.abs(gl - ref_lse).max())
    if w.dtype == "f32":
        assert max_abs <= F32_MAX_ABS, (max_abs, mean_abs)
        if lse_err is not None:
            assert lse_err <= F32_LSE_ABS, lse_err
    else:
        assert max_abs <= BF16_MAX_ABS, (max_abs, mean_abs)
        assert mean_abs <= BF16_MEAN_ABS, (max_abs, mean_abs)
        if lse_err is not None:
            assert lse_err <= BF16_LSE_ABS, lse_err
    return max_abs, mean_abs, lse_err


def oracle_on_rounded_operands(w, inputs, scale=None):
    """The oracle's attention (all rows, whole sequence) on R(q) and R(k)
    rounded to bf16, the precision in which the bf16 kernels hold the rotated
    operands.  The rotation is the oracle's own fp64 one; only the storage
    rounding is modelled (torch's round-to-nearest-even to bf16).  What is left
    between this and the kernel is P's rounding to bf16, fp32 accumulation and
    the output's rounding, none of which grows with the size of the logits --
    so the plain bf16 bounds hold at any logit scale.  Returns (out [B, N,
    heads, hd], lse [B, heads, N])."""
    Nc = w.n_cond_tokens
    qr = oracle.rope3d_apply(inputs["q"], w.H, w.W)
    kr = oracle.rope3d_apply(inputs["k"], w.H, w.W)
    qr = torch.from_numpy(qr).to(torch.bfloat16).double().numpy()
    kr = torch.from_numpy(kr).to(torch.bfloat16).double().numpy()
    B, N, heads, hd = qr.shape
    rows = oracle.all_rows(B, N, heads)
    o, l = oracle.attention_rows(inputs["q"], inputs["k"], inputs["v"], H=w.H, W=w.W, Nc=Nc,
                                 block=w.block, local=w.local, stride=w.stride, rows=rows,
                                 scale=scale, q_rotated=qr, k_rotated=kr)
    out = np.zeros((B, N, heads, hd))
    lse = np.zeros((B, heads, N))
    out[rows[:, 0], rows[:, 2], rows[:, 1]] = o
    lse[rows[:, 0], rows[:, 1], rows[:, 2]] = l
    return out, lse
