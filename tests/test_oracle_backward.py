"""Pins of the oracle's attention backward (no GPU).

The gradient formulas of oracle/backward.py are checked against torch
autograd in fp64 (the forward restated with torch operations, the gradient
derived by the library), against central finite differences of the pinned C
forward, and by the invariant sum_m dv_m = sum_n dO_n; the token mask against
the C brute force; the row/key-sampled forms against the dense one.
"""
import numpy as np
import pytest
import torch

import oracle
from oracle import backward as ob

CASES = [
    dict(T=3, H=4, W=16, n_cond=1, local=1, stride=2),   # condition frame, 3 noisy blocks
    dict(T=2, H=5, W=13, n_cond=0, local=0, stride=3),   # partial blocks, globals
    dict(T=4, H=3, W=11, n_cond=2, local=2, stride=0),   # ragged condition segment
]


def _rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


def _inputs(c, heads=2, B=1, seed=0):
    N = c["T"] * c["H"] * c["W"]
    return [_rand((B, N, heads, 64), seed + i) for i in range(4)]


@pytest.mark.parametrize("c", CASES)
def test_token_mask_matches_brute_force(c):
    N = c["T"] * c["H"] * c["W"]
    Nc = c["n_cond"] * c["H"] * c["W"]
    m = ob.token_mask(N, Nc, 64, c["local"], c["stride"])
    rng = np.random.default_rng(1)
    for n, k in zip(rng.integers(0, N, 400), rng.integers(0, N, 400)):
        assert m[n, k] == oracle.token_allowed(int(n), int(k), Nc, 64, c["local"], c["stride"])
    assert m.sum() == oracle.count_token_pairs(N, Nc, 64, c["local"], c["stride"])


def _torch_grads(c, q, k, v, g, qn=None, kn=None, eps=1e-6):
    """Forward in torch fp64 (rotation from the oracle's pinned angles, SDPA
    with the boolean mask); gradients by autograd."""
    N = q.shape[1]
    Nc = c["n_cond"] * c["H"] * c["W"]
    cos, sin = (torch.from_numpy(a) for a in ob.rope_angles(N, c["H"], c["W"]))
    mask = torch.from_numpy(ob.token_mask(N, Nc, 64, c["local"], c["stride"]))
    ts = [torch.from_numpy(a).requires_grad_(True) for a in (q, k, v)]
    tq, tk, tv = ts

    def prep(x, w):
        if w is not None:
            x = torch.nn.functional.rms_norm(x, (64,), torch.from_numpy(w), eps=eps)
        a, b = x[..., 0::2], x[..., 1::2]
        c_, s_ = cos[None, :, None, :], sin[None, :, None, :]
        return torch.stack([a * c_ - b * s_, a * s_ + b * c_], dim=-1).flatten(-2)

    Q, K = prep(tq, qn), prep(tk, kn)
    o = torch.nn.functional.scaled_dot_product_attention(
        Q.transpose(1, 2), K.transpose(1, 2), tv.transpose(1, 2), attn_mask=mask).transpose(1, 2)
    (o * torch.from_numpy(g)).sum().backward()
    return o.detach().numpy(), [t.grad.numpy() for t in ts]


@pytest.mark.parametrize("c", CASES)
def test_backward_matches_torch_autograd(c):
    q, k, v, g = _inputs(c)
    o_t, (dq_t, dk_t, dv_t) = _torch_grads(c, q, k, v, g)
    o_o, _ = oracle.forward(q, k, v, **c)
    np.testing.assert_allclose(o_t, o_o, rtol=0, atol=1e-12)  # same forward
    dq, dk, dv = ob.backward(q, k, v, g, **c)
    for a, b in ((dq, dq_t), (dk, dk_t), (dv, dv_t)):
        np.testing.assert_allclose(a, b, rtol=0, atol=1e-11)


def test_backward_with_rms_norm_matches_torch_autograd():
    c = CASES[0]
    q, k, v, g = _inputs(c, seed=10)
    qn, kn = 1.0 + 0.3 * _rand(64, 20), 1.0 + 0.3 * _rand(64, 21)
    _, (dq_t, dk_t, dv_t) = _torch_grads(c, q, k, v, g, qn, kn, eps=1e-6)
    dq, dk, dv = ob.backward(q, k, v, g, **c, q_norm=qn, k_norm=kn, norm_eps=1e-6)
    for a, b in ((dq, dq_t), (dk, dk_t), (dv, dv_t)):
        np.testing.assert_allclose(a, b, rtol=0, atol=1e-10)


def test_backward_finite_differences():
    c = CASES[1]
    q, k, v, g = _inputs(c, seed=30)
    dq, dk, dv = ob.backward(q, k, v, g, **c)

    def loss(q_, k_, v_):
        return float(np.sum(oracle.forward(q_, k_, v_, **c)[0] * g))

    rng = np.random.default_rng(5)
    eps = 1e-5
    for which, grad in ((0, dq), (1, dk), (2, dv)):
        d = rng.standard_normal(q.shape)
        args_p = [q, k, v]
        args_m = [q, k, v]
        args_p[which] = args_p[which] + eps * d
        args_m[which] = args_m[which] - eps * d
        fd = (loss(*args_p) - loss(*args_m)) / (2 * eps)
        assert abs(fd - np.sum(grad * d)) <= 1e-6 * max(1.0, abs(fd)), (which, fd, np.sum(grad * d))


def test_dv_sums_to_dout_sum():
    c = CASES[2]
    q, k, v, g = _inputs(c, seed=40)
    _, _, dv = ob.backward(q, k, v, g, **c)
    np.testing.assert_allclose(dv.sum(axis=1), g.sum(axis=1), rtol=0, atol=1e-10)


def test_sampled_forms_match_dense():
    c = CASES[0]
    q, k, v, g = _inputs(c, heads=2, seed=50)
    dq, dk, dv = ob.backward(q, k, v, g, **c)
    N = q.shape[1]
    Nc = c["n_cond"] * c["H"] * c["W"]
    kw = dict(H=c["H"], W=c["W"], Nc=Nc, block=64, local=c["local"], stride=c["stride"])
    rows = np.array([(0, 1, n) for n in (0, 5, Nc - 1, Nc, N // 2, N - 1)])
    got = ob.backward_dq_rows(q, k, v, g, rows=rows, **kw)
    np.testing.assert_allclose(got, dq[0, rows[:, 2], 1], rtol=0, atol=1e-11)
    keys = np.array([0, Nc - 1, Nc, Nc + 70, N - 1])
    gk, gv = ob.backward_dkdv_keys(q, k, v, g, b=0, h=1, keys=keys, **kw)
    np.testing.assert_allclose(gk, dk[0, keys, 1], rtol=0, atol=1e-11)
    np.testing.assert_allclose(gv, dv[0, keys, 1], rtol=0, atol=1e-11)


def test_sampled_forms_with_rms_norm_match_dense():
    c = CASES[1]
    q, k, v, g = _inputs(c, heads=2, seed=60)
    rng = np.random.default_rng(61)
    qn, kn = 1 + 0.3 * rng.standard_normal(64), 1 + 0.3 * rng.standard_normal(64)
    nkw = dict(q_norm=qn, k_norm=kn, norm_eps=1e-6)
    dq, dk, dv = ob.backward(q, k, v, g, **c, **nkw)
    N = q.shape[1]
    Nc = c["n_cond"] * c["H"] * c["W"]
    kw = dict(H=c["H"], W=c["W"], Nc=Nc, block=64, local=c["local"], stride=c["stride"])
    rows = np.array([(0, 0, n) for n in (0, 3, N // 3, N - 1)] + [(0, 1, 7)])
    got = ob.backward_dq_rows(q, k, v, g, rows=rows, **kw, **nkw)
    np.testing.assert_allclose(got, dq[0, rows[:, 2], rows[:, 1]], rtol=0, atol=1e-11)
    keys = np.array([0, 1, 64, N - 1])
    gk, gv = ob.backward_dkdv_keys(q, k, v, g, b=0, h=1, keys=keys, **kw, **nkw)
    np.testing.assert_allclose(gk, dk[0, keys, 1], rtol=0, atol=1e-11)
    np.testing.assert_allclose(gv, dv[0, keys, 1], rtol=0, atol=1e-11)
