"""Pins of the oracle's RMSNorm of q and k ahead of the 3D-RoPE (no GPU).

myzaker / QbitAI, section "背后技术原理": the attention modules use RMSNorm.
The reading (per token and head, over the 64 channels, one weight per
channel, before the rotation) is pinned by a hand-computed value, a library
routine (torch's rms_norm in fp64), per-head scale invariance (which fails if
the norm ran over all heads), and the norm-then-rotate order (which fails if
the rotation came first, since the weights are not uniform).
"""
import numpy as np
import torch

import oracle


def _rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


def test_hand_computed_row():
    x = np.zeros(64)
    x[0], x[1] = 3.0, 4.0  # mean square 25/64, root mean square 5/8
    y = oracle.rms_norm(x, np.ones(64), 0.0)
    assert y[0] == 4.8 and y[1] == 6.4 and np.all(y[2:] == 0.0)
    y = oracle.rms_norm(x, np.full(64, 0.5), 1e-6)
    np.testing.assert_allclose(y[:2], 0.5 * x[:2] / np.sqrt(25 / 64 + 1e-6), rtol=1e-15)


def test_matches_torch_rms_norm():
    x = _rand((2, 37, 3, 64), 5)
    w = 1.0 + 0.3 * _rand(64, 6)
    for eps in (0.0, 1e-6, 0.25):
        ref = torch.nn.functional.rms_norm(torch.from_numpy(x), (64,), torch.from_numpy(w),
                                           eps=eps).numpy()
        np.testing.assert_allclose(oracle.rms_norm(x, w, eps), ref, rtol=1e-14, atol=1e-14)


def test_unit_weight_gives_unit_rms():
    y = oracle.rms_norm(_rand((5, 64), 7) * 9.0, np.ones(64), 0.0)
    np.testing.assert_allclose(np.mean(y * y, axis=-1), 1.0, rtol=1e-14)


def test_per_head_scale_invariance():
    """Scaling one head's q and k leaves that head's attention unchanged (eps 0)."""
    T, H, W, heads = 2, 4, 16, 2
    N = T * H * W
    q, k, v = (_rand((1, N, heads, 64), s) for s in (11, 12, 13))
    qn, kn = 1.0 + 0.2 * _rand(64, 14), 1.0 + 0.2 * _rand(64, 15)
    kw = dict(T=T, H=H, W=W, n_cond=0, local=1, stride=2, q_norm=qn, k_norm=kn, norm_eps=0.0)
    o1, l1 = oracle.forward(q, k, v, **kw)
    q2, k2 = q.copy(), k.copy()
    q2[:, :, 0] *= 10.0
    k2[:, :, 0] *= 10.0
    q2[:, :, 1] *= 0.1
    k2[:, :, 1] *= 0.1
    o2, l2 = oracle.forward(q2, k2, v, **kw)
    np.testing.assert_allclose(o2, o1, rtol=0, atol=1e-12)
    np.testing.assert_allclose(l2, l1, rtol=0, atol=1e-12)


def test_norm_then_rotate_dense():
    """With the all-blocks mask the result is SDPA on R(rms_norm(q)), R(rms_norm(k)):
    torch's rms_norm, the pinned rotation, torch's SDPA."""
    T, H, W, heads = 2, 3, 8, 2
    N = T * H * W
    q, k, v = (_rand((1, N, heads, 64), s) for s in (21, 22, 23))
    qn, kn = 1.0 + 0.5 * _rand(64, 24), 1.0 + 0.5 * _rand(64, 25)
    eps = 1e-6
    out, lse = oracle.forward(q, k, v, T=T, H=H, W=W, n_cond=0, local=0, stride=1, q_norm=qn,
                              k_norm=kn, norm_eps=eps)
    tn = lambda x, w: torch.nn.functional.rms_norm(torch.from_numpy(x), (64,), torch.from_numpy(w),
                                                   eps=eps).numpy()
    qr = oracle.rope3d_apply(tn(q, qn), H, W)
    kr = oracle.rope3d_apply(tn(k, kn), H, W)
    for h in range(heads):
        ref = torch.nn.functional.scaled_dot_product_attention(
            *(torch.from_numpy(a[0, :, h])[None, None] for a in (qr, kr, v)))[0, 0].numpy()
        np.testing.assert_allclose(out[0, :, h], ref, rtol=0, atol=1e-12)
    # rotating first and normalising after gives something else (weights not uniform)
    qw = tn(oracle.rope3d_apply(q, H, W), qn)
    assert np.abs(qw - qr).max() > 1e-3
