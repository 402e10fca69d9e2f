"""Pins of the oracle's masked softmax attention (no GPU).

Checks against a library routine (torch's scaled_dot_product_attention on CPU
in fp64), special cases with a textbook answer and invariants the pages fix
(condition tokens unaffected by noise tokens: myzaker / QbitAI page,
"背后技术原理"; dense inside blocks: zhichai.net page, "Block Sparse Attention").
"""
import numpy as np
import pytest
import torch

import oracle


def _rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


def _sdpa(q, k, v, mask=None):
    """Library reference: torch SDPA in fp64 on CPU.  q,k,v: [N, hd]."""
    qt, kt, vt = (torch.from_numpy(a)[None, None] for a in (q, k, v))
    m = None if mask is None else torch.from_numpy(mask)[None, None]
    return torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, attn_mask=m)[0, 0].numpy()


@pytest.mark.parametrize("T,H,W", [(2, 4, 16), (3, 5, 7)])
def test_all_blocks_mask_equals_dense_attention(T, H, W):
    N, heads = T * H * W, 2
    q, k, v = _rand((1, N, heads, 64), 1), _rand((1, N, heads, 64), 2), _rand((1, N, heads, 64), 3)
    out, lse = oracle.forward(q, k, v, T=T, H=H, W=W, n_cond=0, local=0, stride=1)
    qr, kr = oracle.rope3d_apply(q, H, W), oracle.rope3d_apply(k, H, W)
    for h in range(heads):
        ref = _sdpa(qr[0, :, h], kr[0, :, h], v[0, :, h])
        np.testing.assert_allclose(out[0, :, h], ref, rtol=0, atol=1e-12)
        s = qr[0, :, h] @ kr[0, :, h].T / 8.0
        ref_lse = np.log(np.exp(s - s.max(1, keepdims=True)).sum(1)) + s.max(1)
        np.testing.assert_allclose(lse[0, h], ref_lse, rtol=0, atol=1e-12)


def test_dense_with_condition_frames_equals_masked_sdpa():
    T, H, W, nc = 3, 4, 8, 1
    N, Nc = T * H * W, nc * H * W
    q, k, v = _rand((1, N, 1, 64), 4), _rand((1, N, 1, 64), 5), _rand((1, N, 1, 64), 6)
    out, _ = oracle.forward(q, k, v, T=T, H=H, W=W, n_cond=nc, local=0, stride=1)
    mask = np.ones((N, N), dtype=bool)
    mask[:Nc, Nc:] = False        # condition queries see condition keys only
    qr, kr = oracle.rope3d_apply(q, H, W), oracle.rope3d_apply(k, H, W)
    ref = _sdpa(qr[0, :, 0], kr[0, :, 0], v[0, :, 0], mask)
    np.testing.assert_allclose(out[0, :, 0], ref, rtol=0, atol=1e-12)


def test_local_zero_is_independent_per_block_attention():
    # 3 frames of 5x13 = 195 tokens -> blocks of 64, 64, 64, 3 (partial tail)
    T, H, W = 3, 5, 13
    N = T * H * W
    q, k, v = _rand((1, N, 2, 64), 7), _rand((1, N, 2, 64), 8), _rand((1, N, 2, 64), 9)
    out, _ = oracle.forward(q, k, v, T=T, H=H, W=W, n_cond=0, local=0, stride=0)
    qr, kr = oracle.rope3d_apply(q, H, W), oracle.rope3d_apply(k, H, W)
    for h in range(2):
        for s in range(0, N, 64):
            e = min(N, s + 64)
            ref = _sdpa(qr[0, s:e, h], kr[0, s:e, h], v[0, s:e, h])
            np.testing.assert_allclose(out[0, s:e, h], ref, rtol=0, atol=1e-12)


def test_rows_sum_to_one_and_vanish_off_mask():
    T, H, W, nc = 4, 4, 16, 1
    N, Nc = T * H * W, nc * H * W
    q, k = _rand((1, N, 1, 64), 10), _rand((1, N, 1, 64), 11)
    for r in [0, 63, 64, 100, 200, 255]:
        p = oracle.row_probs(q, k, H=H, W=W, Nc=Nc, block=64, local=0, stride=2, b=0, head=0, r=r)
        assert abs(p.sum() - 1.0) < 1e-12
        for m in range(N):
            if not oracle.token_allowed(r, m, Nc, 64, 0, 2):
                assert p[m] == 0.0
            else:
                assert p[m] > 0.0


def test_single_key_row_returns_its_value():
    # 1 frame of 5x13 = 65 tokens: block 1 holds the single token 64, which
    # with local=0, stride=0 attends only itself.
    T, H, W = 1, 5, 13
    N = T * H * W
    q, k, v = _rand((1, N, 1, 64), 12), _rand((1, N, 1, 64), 13), _rand((1, N, 1, 64), 14)
    out, lse = oracle.forward(q, k, v, T=T, H=H, W=W, n_cond=0, local=0, stride=0)
    np.testing.assert_allclose(out[0, 64, 0], v[0, 64, 0], rtol=0, atol=1e-15)
    qr, kr = oracle.rope3d_apply(q, H, W), oracle.rope3d_apply(k, H, W)
    assert abs(lse[0, 0, 64] - qr[0, 64, 0] @ kr[0, 64, 0] / 8.0) < 1e-12


def test_constant_values_return_the_constant():
    T, H, W, nc = 4, 8, 16, 1
    N = T * H * W
    q, k = _rand((1, N, 2, 64), 15), _rand((1, N, 2, 64), 16)
    v = np.broadcast_to(_rand((1, 1, 2, 64), 17), (1, N, 2, 64)).copy()
    out, _ = oracle.forward(q, k, v, T=T, H=H, W=W, n_cond=nc, local=1, stride=3)
    np.testing.assert_allclose(out, v, rtol=0, atol=1e-12)


def test_condition_outputs_ignore_noise_tokens():
    T, H, W, nc = 4, 8, 16, 2
    N, Nc = T * H * W, nc * H * W
    q, k, v = _rand((1, N, 2, 64), 18), _rand((1, N, 2, 64), 19), _rand((1, N, 2, 64), 20)
    out, lse = oracle.forward(q, k, v, T=T, H=H, W=W, n_cond=nc, local=2, stride=4)
    q2, k2, v2 = q.copy(), k.copy(), v.copy()
    rng = np.random.default_rng(21)
    for a in (q2, k2, v2):
        a[:, Nc:] += rng.standard_normal(a[:, Nc:].shape)
    out2, lse2 = oracle.forward(q2, k2, v2, T=T, H=H, W=W, n_cond=nc, local=2, stride=4)
    np.testing.assert_array_equal(out2[:, :Nc], out[:, :Nc])
    np.testing.assert_array_equal(lse2[:, :, :Nc], lse[:, :, :Nc])
    assert np.abs(out2[:, Nc:] - out[:, Nc:]).max() > 0.1


def test_cached_form_equals_noisy_rows_of_full_form():
    T, H, W, nc = 5, 4, 16, 2
    N, Nc = T * H * W, nc * H * W
    q, k, v = _rand((1, N, 2, 64), 22), _rand((1, N, 2, 64), 23), _rand((1, N, 2, 64), 24)
    full, full_lse = oracle.forward(q, k, v, T=T, H=H, W=W, n_cond=nc, local=1, stride=2)
    out, lse = oracle.forward_cached(q[:, Nc:], k[:, Nc:], v[:, Nc:], k[:, :Nc], v[:, :Nc],
                                     T=T, H=H, W=W, n_cond=nc, local=1, stride=2)
    np.testing.assert_allclose(out, full[:, Nc:], rtol=0, atol=1e-13)
    np.testing.assert_allclose(lse, full_lse[:, :, Nc:], rtol=0, atol=1e-13)


def test_explicit_small_case_by_hand():
    """Two tokens, one frame: brute force written out with numpy."""
    T, H, W = 1, 1, 2
    q, k, v = _rand((1, 2, 1, 64), 25), _rand((1, 2, 1, 64), 26), _rand((1, 2, 1, 64), 27)
    out, _ = oracle.forward(q, k, v, T=T, H=H, W=W, n_cond=0, local=0, stride=0)
    # token 0 is at (0,0,0): unrotated; token 1 at (0,0,1): only the W slice turns.
    q1 = q[0, 1, 0].copy()
    k1 = k[0, 1, 0].copy()
    for x in (q1, k1):
        z = x[40::2] + 1j * x[41::2]
        z = z * np.exp(1j * 10000.0 ** (-2.0 * np.arange(12) / 24))
        x[40::2], x[41::2] = z.real, z.imag
    qs = [q[0, 0, 0], q1]
    ks = [k[0, 0, 0], k1]
    for r in range(2):
        s = np.array([qs[r] @ ks[m] / 8.0 for m in range(2)])
        p = np.exp(s - s.max())
        p /= p.sum()
        np.testing.assert_allclose(out[0, r, 0], p[0] * v[0, 0, 0] + p[1] * v[0, 1, 0],
                                   rtol=0, atol=1e-13)
