"""fp64 CPU oracle for block-sparse 3D-RoPE video self-attention.

TEST INFRASTRUCTURE ONLY.  This package is the plain, slow, obviously correct
statement of what the GPU library computes.  Only the tests, the smoke check
and the CPU-baseline leg of the benchmark may import it; the library never
does, and the two share no code (only the seeded input generator, which holds
none of the method's arithmetic, feeds both).

The arithmetic lives in ``lc_oracle.c`` (plain C, fp64, OpenMP over rows).
This module compiles it on demand with gcc, upcasts inputs to fp64, and calls
it through ctypes.  Citations of the pages each function follows are in the C
file's header; the readings taken where the pages are silent are listed there
as well.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional, Sequence, Tuple

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "lc_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liblcoracle.so")
_lib = None

ROPE_THETA = 10000.0
ROPE_DIMS = (16, 24, 24)  # temporal, height, width channels of a 64-D head


def build(force: bool = False) -> str:
    """Compile lc_oracle.c into liblcoracle.so next to it (gcc, -O2, OpenMP).

    No fast-math: the oracle keeps IEEE fp64 semantics."""
    stale = (not os.path.exists(_LIB_PATH)) or (
        os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC))
    if force or stale:
        tmp = _LIB_PATH + ".tmp.%d" % os.getpid()
        subprocess.run(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c99",
                        "-o", tmp, _SRC, "-lm"], check=True)
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is not None:
        return _lib
    lib = ctypes.CDLL(build())
    dp = ctypes.POINTER(ctypes.c_double)
    ip = ctypes.POINTER(ctypes.c_int)
    lp = ctypes.POINTER(ctypes.c_long)
    L, I, D = ctypes.c_long, ctypes.c_int, ctypes.c_double
    lib.orc_rope3d_rotate_vec.argtypes = [dp, I, L, L, L, D, I, I, I]
    lib.orc_rope3d_apply.argtypes = [dp, I, L, I, I, L, I, I, D, I, I, I]
    lib.orc_noisy_block_rule.argtypes = [L, L, I, I]
    lib.orc_noisy_block_rule.restype = I
    lib.orc_token_allowed.argtypes = [L, L, L, I, I, I]
    lib.orc_token_allowed.restype = I
    lib.orc_block_csr.argtypes = [I, I, I, I, I, I, I, ip, ip]
    lib.orc_block_csr.restype = L
    lib.orc_count_token_pairs.argtypes = [L, L, I, I, I]
    lib.orc_count_token_pairs.restype = ctypes.c_longlong
    lib.orc_attention_rows.argtypes = [dp, dp, dp, I, L, L, L, I, I, L, I, I, I, D,
                                       lp, L, dp, dp, I]
    lib.orc_attention_row_probs.argtypes = [dp, dp, L, L, L, I, I, L, I, I, I, D,
                                            L, L, L, dp]
    lib.orc_max_threads.restype = I
    _lib = lib
    return lib


def _f64(x) -> np.ndarray:
    """Exact upcast of the values handed to the GPU (bf16/fp32 -> fp64)."""
    if hasattr(x, "detach"):  # a torch tensor: go through fp32 (exact for bf16)
        x = x.detach().to("cpu").float().numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _dp(a: np.ndarray):
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def max_threads() -> int:
    return int(_load().orc_max_threads())


# --------------------------------------------------------------------------
# Geometry
# --------------------------------------------------------------------------
def segment_sizes(T: int, H: int, W: int, n_cond: int, block: int = 64):
    """(Nc, Nn, Cb, Nb): condition / noisy token counts and block counts.
    Condition frames come first on the time axis (myzaker / QbitAI page,
    section on the unified tasks: no condition frame for text-to-video, one
    for image-to-video, several for continuation -- the frames after them are
    the ones generated).  Reading taken: at least one frame is generated, so
    0 <= n_cond < T."""
    if min(T, H, W, block) <= 0 or not 0 <= n_cond < T:
        raise ValueError(f"bad sizes T={T} H={H} W={W} block={block} n_cond={n_cond} "
                         "(n_cond counts latent frames, 0 <= n_cond < T)")
    Nc = n_cond * H * W
    Nn = (T - n_cond) * H * W
    return Nc, Nn, -(-Nc // block), -(-Nn // block)


def decode_position(n: int, H: int, W: int) -> Tuple[int, int, int]:
    """Token n of the t-major, h, w flattened grid -> (t, h, w)."""
    return n // (H * W), (n // W) % H, n % W


# --------------------------------------------------------------------------
# RoPE
# --------------------------------------------------------------------------
def rope3d_rotate_vec(x, t: int, h: int, w: int, theta: float = ROPE_THETA,
                      dims: Sequence[int] = ROPE_DIMS) -> np.ndarray:
    """Rotate one head vector at grid position (t, h, w) ("longcat-video-rs",
    section 03-01, Partitioned 3D-RoPE)."""
    v = _f64(x).copy()
    _load().orc_rope3d_rotate_vec(_dp(v), v.shape[-1], t, h, w, theta, *dims)
    return v


def rope3d_apply(x, H: int, W: int, tok_offset: int = 0,
                 theta: float = ROPE_THETA, dims: Sequence[int] = ROPE_DIMS) -> np.ndarray:
    """Rotate x [B, ntok, heads, hd]; token n of x is token n + tok_offset of
    the full sequence.  Returns a new fp64 array."""
    v = _f64(x).copy()
    B, ntok, heads, hd = v.shape
    assert sum(dims) == hd
    _load().orc_rope3d_apply(_dp(v), B, ntok, heads, hd, tok_offset, H, W, theta, *dims)
    return v


# --------------------------------------------------------------------------
# RMSNorm of q and k ahead of RoPE
# --------------------------------------------------------------------------
def rms_norm(x, weight, eps: float) -> np.ndarray:
    """RMSNorm over the head dimension of x [..., hd]: x / sqrt(mean(x^2) +
    eps) * weight, in fp64.  myzaker / QbitAI, section "背后技术原理": the
    self- and cross-attention modules use RMSNorm for training stability.
    Reading taken (the page gives no formula): the norm is applied to q and k
    per token and per head over the 64 channels, with one learned weight per
    channel shared by the heads, before the 3D-RoPE rotation."""
    xf = _f64(x)
    w = np.asarray(weight, dtype=np.float64).reshape(-1)
    assert w.shape[0] == xf.shape[-1]
    ms = np.mean(xf * xf, axis=-1, keepdims=True)
    return xf / np.sqrt(ms + eps) * w


# --------------------------------------------------------------------------
# Mask
# --------------------------------------------------------------------------
def noisy_block_rule(i: int, j: int, local: int, stride: int) -> bool:
    return bool(_load().orc_noisy_block_rule(i, j, local, stride))


def token_allowed(n: int, m: int, Nc: int, block: int, local: int, stride: int) -> bool:
    return bool(_load().orc_token_allowed(n, m, Nc, block, local, stride))


def block_csr(T: int, H: int, W: int, block: int, local: int, stride: int,
              n_cond: int) -> Tuple[np.ndarray, np.ndarray]:
    """Brute-force block CSR: row_ptr [Cb+Nb+1], col_idx [nnz] (int32)."""
    lib = _load()
    _, _, Cb, Nb = segment_sizes(T, H, W, n_cond, block)
    nnz = lib.orc_block_csr(T, H, W, block, local, stride, n_cond, None, None)
    row_ptr = np.zeros(Cb + Nb + 1, dtype=np.int32)
    col_idx = np.zeros(max(nnz, 1), dtype=np.int32)
    ip = ctypes.POINTER(ctypes.c_int)
    lib.orc_block_csr(T, H, W, block, local, stride, n_cond,
                      row_ptr.ctypes.data_as(ip), col_idx.ctypes.data_as(ip))
    return row_ptr, col_idx[:nnz]


def count_token_pairs(N: int, Nc: int, block: int, local: int, stride: int) -> int:
    """Attended (query, key) token pairs, counted token by token (O(N^2))."""
    return int(_load().orc_count_token_pairs(N, Nc, block, local, stride))


# --------------------------------------------------------------------------
# Attention
# --------------------------------------------------------------------------
def attention_rows(q, k, v, *, H: int, W: int, Nc: int, block: int, local: int,
                   stride: int, rows, q_offset: int = 0, scale: Optional[float] = None,
                   theta: float = ROPE_THETA, dims: Sequence[int] = ROPE_DIMS,
                   nthreads: int = 0, q_rotated: Optional[np.ndarray] = None,
                   k_rotated: Optional[np.ndarray] = None, q_norm=None, k_norm=None,
                   norm_eps: float = 1e-6):
    """Masked softmax attention on RoPE-rotated q/k for selected rows.

    q: [B, Nq, heads, hd] (query r is token r + q_offset of the sequence);
    k, v: [B, N, heads, hd] (the full condition + noisy sequence);
    rows: int array [R, 3] of (b, head, r).  q_norm / k_norm: optional
    per-channel RMSNorm weights applied to q / k before the rotation.
    Returns (out [R, hd], lse [R]).
    """
    qf = _f64(q)
    if q_norm is not None and q_rotated is None:
        qf = rms_norm(qf, q_norm, norm_eps)
    if k_norm is not None and k_rotated is None:
        k = rms_norm(k, k_norm, norm_eps)
    B, Nq, heads, hd = qf.shape
    rows = np.ascontiguousarray(np.asarray(rows, dtype=np.int64).reshape(-1, 3))
    qrot = q_rotated if q_rotated is not None else rope3d_apply(qf, H, W, q_offset, theta, dims)
    lib = _load()
    krot = k_rotated if k_rotated is not None else rope3d_apply(k, H, W, 0, theta, dims)
    vf = _f64(v)
    N = krot.shape[1]
    if scale is None:
        scale = 1.0 / np.sqrt(hd)
    R = rows.shape[0]
    out = np.zeros((R, hd), dtype=np.float64)
    lse = np.zeros(R, dtype=np.float64)
    lib.orc_attention_rows(_dp(qrot), _dp(krot), _dp(vf), B, Nq, q_offset, N, heads, hd,
                           Nc, block, local, stride, float(scale),
                           rows.ctypes.data_as(ctypes.POINTER(ctypes.c_long)), R,
                           _dp(out), _dp(lse), nthreads)
    return out, lse


def all_rows(B: int, Nq: int, heads: int) -> np.ndarray:
    b, h, r = np.meshgrid(np.arange(B), np.arange(heads), np.arange(Nq), indexing="ij")
    return np.stack([b.ravel(), h.ravel(), r.ravel()], axis=1)


def forward(q, k, v, *, T: int, H: int, W: int, n_cond: int, block: int = 64,
            local: int, stride: int, scale: Optional[float] = None, nthreads: int = 0,
            q_norm=None, k_norm=None, norm_eps: float = 1e-6):
    """Whole-layer oracle over the full sequence (q, k, v: [B, N, heads, hd]).
    Returns out [B, N, heads, hd] and lse [B, heads, N] (fp64)."""
    qf = _f64(q)
    B, N, heads, hd = qf.shape
    assert N == T * H * W
    Nc = n_cond * H * W
    rows = all_rows(B, N, heads)
    o, l = attention_rows(qf, k, v, H=H, W=W, Nc=Nc, block=block, local=local,
                          stride=stride, rows=rows, scale=scale, nthreads=nthreads,
                          q_norm=q_norm, k_norm=k_norm, norm_eps=norm_eps)
    out = np.zeros((B, N, heads, hd))
    lse = np.zeros((B, heads, N))
    out[rows[:, 0], rows[:, 2], rows[:, 1]] = o
    lse[rows[:, 0], rows[:, 1], rows[:, 2]] = l
    return out, lse


def forward_cached(q, k, v, cond_k, cond_v, *, T: int, H: int, W: int, n_cond: int,
                   block: int = 64, local: int, stride: int,
                   scale: Optional[float] = None, nthreads: int = 0,
                   q_norm=None, k_norm=None, norm_eps: float = 1e-6):
    """Oracle of the cached form: q/k/v hold the noisy tokens only, cond_k /
    cond_v the condition tokens (pre-RoPE).  The keys are the condition tokens
    followed by the noisy tokens; noisy query r is token Nc + r.
    Returns out [B, Nn, heads, hd], lse [B, heads, Nn]."""
    kf = np.concatenate([_f64(cond_k), _f64(k)], axis=1)
    vf = np.concatenate([_f64(cond_v), _f64(v)], axis=1)
    qf = _f64(q)
    B, Nn, heads, hd = qf.shape
    Nc = n_cond * H * W
    assert kf.shape[1] == T * H * W and Nc + Nn == kf.shape[1]
    rows = all_rows(B, Nn, heads)
    o, l = attention_rows(qf, kf, vf, H=H, W=W, Nc=Nc, block=block, local=local,
                          stride=stride, rows=rows, q_offset=Nc, scale=scale,
                          nthreads=nthreads, q_norm=q_norm, k_norm=k_norm,
                          norm_eps=norm_eps)
    out = np.zeros((B, Nn, heads, hd))
    lse = np.zeros((B, heads, Nn))
    out[rows[:, 0], rows[:, 2], rows[:, 1]] = o
    lse[rows[:, 0], rows[:, 1], rows[:, 2]] = l
    return out, lse


def row_probs(q, k, *, H: int, W: int, Nc: int, block: int, local: int, stride: int,
              b: int, head: int, r: int, q_offset: int = 0,
              scale: Optional[float] = None) -> np.ndarray:
    """Softmax probabilities of one query row over all keys (0 where masked)."""
    qrot = rope3d_apply(q, H, W, q_offset)
    krot = rope3d_apply(k, H, W, 0)
    _, Nq, heads, hd = qrot.shape
    N = krot.shape[1]
    if scale is None:
        scale = 1.0 / np.sqrt(hd)
    probs = np.zeros(N)
    _load().orc_attention_row_probs(_dp(qrot), _dp(krot), Nq, q_offset, N, heads, hd,
                                    Nc, block, local, stride, float(scale), b, head, r,
                                    _dp(probs))
    return probs
