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
