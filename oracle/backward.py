"""fp64 oracle of the attention backward pass (gradients of q, k and v).

TEST INFRASTRUCTURE ONLY (see the package docstring): the library never
imports it.

Why a backward at all: the SimpleTuner page ("Guia de Início Rápido do
LongCat-Video Edit"), section "2) Mudanças no config", trains LongCat-Video
with LoRA adapters and gradient checkpointing, which needs the gradient of
the attention layer with respect to its q, k and v inputs.  The pages give no
formula for it; it is the chain rule applied to the forward definition the
rest of the oracle states (masked softmax attention on the 3D-RoPE-rotated,
optionally RMS-normalised q and k), written out plainly:

    q' = R(norm_q(q)),  k' = R(norm_k(k))          (per token and head)
    S = scale * q' k'^T on the attended pairs, P = softmax_rows(S), O = P v
    dv = P^T dO
    dP = dO v^T,   D = rowsum(dO * O),   dS = P * (dP - D)
    dq' = scale * dS k',   dk' = scale * dS^T q'
    dq = norm_q^T(R^T dq'),   dk = norm_k^T(R^T dk')

R^T turns each channel pair back by its angle; the angles are read off the
forward rotation (R applied to the pair (1, 0) gives (cos, sin)), so no
second statement of the RoPE frequencies exists here.  The RMSNorm
transpose is that of y = x * inv * w with inv = (mean(x^2) + eps)^(-1/2):
dx = inv * (w * g) - x * inv^3 / d * sum(g * w * x).
"""
from __future__ import annotations

from typing import Optional, Sequence

import numpy as np

from . import (ROPE_DIMS, ROPE_THETA, _f64, attention_rows, rms_norm, rope3d_apply,
               segment_sizes)


def token_mask(N: int, Nc: int, block: int, local: int, stride: int,
               rows: Optional[np.ndarray] = None, cols: Optional[np.ndarray] = None):
    """Boolean [len(rows), len(cols)] attended-pair mask from the definition
    (condition queries see condition keys; noisy queries see condition keys
    and the noisy blocks |i - j| <= local or j % stride == 0)."""
    n = np.arange(N) if rows is None else np.asarray(rows)
    m = np.arange(N) if cols is None else np.asarray(cols)
    nq, mk = n[:, None], m[None, :]
    cond_q, cond_k = nq < Nc, mk < Nc
    i, j = (nq - Nc) // block, (mk - Nc) // block
    noisy = (np.abs(i - j) <= local)
    if stride > 0:
        noisy = noisy | (j % stride == 0)
    return np.where(cond_q, cond_k, cond_k | noisy)


def rope_angles(N: int, H: int, W: int, hd: int = 64, tok_offset: int = 0,
                theta: float = ROPE_THETA, dims: Sequence[int] = ROPE_DIMS):
    """(cos, sin) [N, hd/2] of every token's pair angles, read off the forward
    rotation of the pair (1, 0)."""
    e = np.zeros((1, N, 1, hd))
    e[..., 0::2] = 1.0
    r = rope3d_apply(e, H, W, tok_offset, theta, dims)[0, :, 0]
    return r[:, 0::2], r[:, 1::2]


def rope_transpose(g, cos, sin):
    """R^T g for g [..., N, hd] (pairs (2k, 2k+1) turned back by their angle)."""
    a, b = g[..., 0::2], g[..., 1::2]
    out = np.empty_like(g)
    out[..., 0::2] = a * cos + b * sin
    out[..., 1::2] = -a * sin + b * cos
    return out


def rms_norm_transpose(x, g, weight, eps: float):
    """Gradient w.r.t. x of y = rms_norm(x, weight, eps), given dL/dy = g."""
    x = _f64(x)
    w = np.asarray(weight, dtype=np.float64)
    d = x.shape[-1]
    inv = 1.0 / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps)
    return inv * (w * g) - x * inv ** 3 / d * np.sum(g * w * x, axis=-1, keepdims=True)


def backward(q, k, v, dout, *, T: int, H: int, W: int, n_cond: int, block: int = 64,
             local: int, stride: int, scale: Optional[float] = None, q_norm=None,
             k_norm=None, norm_eps: float = 1e-6):
    """Gradients (dq, dk, dv) of the whole-sequence forward for dout, dense per
    head (small sequences only: N x N matrices).  All [B, N, heads, hd]."""
    qf, kf, vf, gf = (_f64(a) for a in (q, k, v, dout))
    B, N, heads, hd = qf.shape
    Nc, _, _, _ = segment_sizes(T, H, W, n_cond, block)
    sc = 1.0 / np.sqrt(hd) if scale is None else scale
    qn = rms_norm(qf, q_norm, norm_eps) if q_norm is not None else qf
    kn = rms_norm(kf, k_norm, norm_eps) if k_norm is not None else kf
    qr, kr = rope3d_apply(qn, H, W), rope3d_apply(kn, H, W)
    cos, sin = rope_angles(N, H, W, hd)
    mask = token_mask(N, Nc, block, local, stride)
    dq, dk, dv = np.zeros_like(qf), np.zeros_like(kf), np.zeros_like(vf)
    for b in range(B):
        for h in range(heads):
            Q, K, V, G = qr[b, :, h], kr[b, :, h], vf[b, :, h], gf[b, :, h]
            S = np.where(mask, sc * (Q @ K.T), -np.inf)
            mx = S.max(axis=1, keepdims=True)
            E = np.exp(S - mx)
            P = E / E.sum(axis=1, keepdims=True)
            O = P @ V
            dv[b, :, h] = P.T @ G
            dP = G @ V.T
            Dn = np.sum(G * O, axis=1, keepdims=True)
            dS = P * (dP - Dn)
            dq[b, :, h] = rope_transpose(sc * (dS @ K), cos, sin)
            dk[b, :, h] = rope_transpose(sc * (dS.T @ Q), cos, sin)
    if q_norm is not None:
        dq = rms_norm_transpose(qf, dq, q_norm, norm_eps)
    if k_norm is not None:
        dk = rms_norm_transpose(kf, dk, k_norm, norm_eps)
    return dq, dk, dv


def backward_dq_rows(q, k, v, dout, *, H: int, W: int, Nc: int, block: int, local: int,
                     stride: int, rows, scale: Optional[float] = None, q_norm=None,
                     k_norm=None, norm_eps: float = 1e-6):
    """dq of the selected query rows (b, head, n) of the whole-sequence
    forward, row by row: a row's gradient needs only its own keys.  Returns
    [R, hd]."""
    qf, kf, vf, gf = (_f64(a) for a in (q, k, v, dout))
    B, N, heads, hd = qf.shape
    sc = 1.0 / np.sqrt(hd) if scale is None else scale
    rows = np.asarray(rows, dtype=np.int64).reshape(-1, 3)
    o, lse = attention_rows(qf, kf, vf, H=H, W=W, Nc=Nc, block=block, local=local,
                            stride=stride, rows=rows, scale=sc, q_norm=q_norm, k_norm=k_norm,
                            norm_eps=norm_eps)
    qnf = rms_norm(qf, q_norm, norm_eps) if q_norm is not None else qf
    knf = rms_norm(kf, k_norm, norm_eps) if k_norm is not None else kf
    cos, sin = rope_angles(N, H, W, hd)
    out = np.zeros((len(rows), hd))
    krot = {}
    for idx, (b, h, n) in enumerate(rows):
        if (b, h) not in krot:
            krot[(b, h)] = rope3d_apply(knf[b:b + 1, :, h:h + 1], H, W)[0, :, 0]
        K = krot[(b, h)]
        qn = rope3d_apply(qnf[b:b + 1, n:n + 1, h:h + 1], H, W, tok_offset=int(n))[0, 0, 0]
        keys = np.nonzero(token_mask(N, Nc, block, local, stride, rows=[n])[0])[0]
        p = np.exp(sc * (K[keys] @ qn) - lse[idx])
        dp = vf[b, keys, h] @ gf[b, n, h]
        ds = p * (dp - gf[b, n, h] @ o[idx])
        g = rope_transpose((sc * (ds @ K[keys]))[None], cos[n:n + 1], sin[n:n + 1])[0]
        if q_norm is not None:
            g = rms_norm_transpose(qf[b, n, h], g, q_norm, norm_eps)
        out[idx] = g
    return out


def backward_dkdv_keys(q, k, v, dout, *, H: int, W: int, Nc: int, block: int, local: int,
                       stride: int, b: int, h: int, keys, scale: Optional[float] = None,
                       q_norm=None, k_norm=None, norm_eps: float = 1e-6):
    """dk and dv of the selected key tokens of one (batch, head), gathered over
    every query that attends them (their softmax statistics come from
    attention_rows).  Returns (dk [K, hd], dv [K, hd])."""
    qf, kf, vf, gf = (_f64(a) for a in (q, k, v, dout))
    B, N, heads, hd = qf.shape
    sc = 1.0 / np.sqrt(hd) if scale is None else scale
    keys = np.asarray(keys, dtype=np.int64)
    att = token_mask(N, Nc, block, local, stride, cols=keys)  # [N, K]
    qrows = np.nonzero(att.any(axis=1))[0]
    trip = np.stack([np.full_like(qrows, b), np.full_like(qrows, h), qrows], axis=1)
    o, lse = attention_rows(qf, kf, vf, H=H, W=W, Nc=Nc, block=block, local=local,
                            stride=stride, rows=trip, scale=sc, q_norm=q_norm, k_norm=k_norm,
                            norm_eps=norm_eps)
    qnf = rms_norm(qf[b:b + 1, :, h:h + 1], q_norm, norm_eps) if q_norm is not None \
        else qf[b:b + 1, :, h:h + 1]
    knf = rms_norm(kf[b:b + 1, :, h:h + 1], k_norm, norm_eps) if k_norm is not None \
        else kf[b:b + 1, :, h:h + 1]
    Q = rope3d_apply(qnf, H, W)[0, qrows, 0]
    Kr = rope3d_apply(knf, H, W)[0, keys, 0]
    G = gf[b, qrows, h]
    A = att[qrows]
    P = np.where(A, np.exp(sc * (Q @ Kr.T) - lse[:, None]), 0.0)  # [Rq, K]
    dv = P.T @ G
    dP = G @ vf[b, keys, h].T
    Dn = np.sum(G * o, axis=1, keepdims=True)
    dS = P * (dP - Dn)
    cos, sin = rope_angles(N, H, W, hd)
    dk = rope_transpose(sc * (dS.T @ Q), cos[keys], sin[keys])
    if k_norm is not None:
        dk = rms_norm_transpose(kf[b, keys, h], dk, k_norm, norm_eps)
    return dk, dv
