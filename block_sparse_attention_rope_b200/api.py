"""Python binding of liblcbsa.so (argument marshalling only).

Every step of the computation runs in the CUDA library declared in
``include/lc_bsa.h``; this module checks tensor shapes, hands raw device
pointers and the current CUDA stream to the C ABI and turns status codes into
exceptions.  PyTorch provides device memory and streams.  There is no CPU
fallback: if the shared library is missing the import fails.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence, Tuple

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
# LC_BSA_LIB may name another build of the same library (same ABI).
LIB_PATH = os.environ.get("LC_BSA_LIB") or os.path.join(_HERE, "liblcbsa.so")

LC_OK, LC_ERR_INVALID_ARGUMENT, LC_ERR_UNSUPPORTED, LC_ERR_CUDA = 0, 1, 2, 3
LC_ERR_OUT_OF_MEMORY, LC_ERR_TIMEOUT, LC_ERR_DEVICE_CHECK = 4, 5, 6
LC_DTYPE_BF16, LC_DTYPE_F32 = 0, 1


class LcError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__("%s: %s (status %d)" % (where, status_string(status), status))


class PlanInfo(ctypes.Structure):
    _fields_ = [("num_q_blocks", ctypes.c_int), ("num_cond_blocks", ctypes.c_int),
                ("num_noisy_blocks", ctypes.c_int), ("nnz", ctypes.c_longlong),
                ("n_cond_tokens", ctypes.c_int), ("n_noisy_tokens", ctypes.c_int),
                ("attended_token_pairs", ctypes.c_longlong),
                ("attended_token_pairs_noisy", ctypes.c_longlong)]


class Opts(ctypes.Structure):
    """lc_bsa_opts."""
    _fields_ = [("flags", ctypes.c_uint), ("q_norm_weight", ctypes.c_void_p),
                ("k_norm_weight", ctypes.c_void_p), ("norm_eps", ctypes.c_float)]


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError("liblcbsa.so is not built (python -m block_sparse_attention_rope_b200.build)")
    lib = ctypes.CDLL(LIB_PATH)
    vp, I, LL, F, D = ctypes.c_void_p, ctypes.c_int, ctypes.c_longlong, ctypes.c_float, ctypes.c_double
    S = ctypes.c_int
    sig = {
        "lc_bsa_plan_create": (S, [ctypes.POINTER(vp), I, I, I, I, I, I, I, vp]),
        "lc_bsa_plan_destroy": (S, [vp, vp]),
        "lc_bsa_plan_info": (S, [vp, ctypes.POINTER(PlanInfo)]),
        "lc_bsa_plan_copy_csr": (S, [vp, vp, vp, vp]),
        "lc_rope3d_tables": (S, [ctypes.POINTER(vp), I, I, I, D, I, I, I, vp]),
        "lc_rope3d_destroy": (S, [vp, vp]),
        "lc_rope3d_copy_tables": (S, [vp, vp, vp]),
        "lc_rope3d_apply": (S, [vp, vp, I, LL, I, I, LL, I, vp, vp]),
        "lc_bsa_forward": (S, [vp, vp, vp, vp, vp, I, I, I, I, F, vp, vp, vp]),
        "lc_bsa_forward_cached": (S, [vp, vp, vp, vp, vp, vp, vp, I, I, I, I, F, vp, vp, vp]),
        "lc_bsa_forward_ex": (S, [vp, vp, vp, vp, vp, I, I, I, I, F, vp, vp, vp, vp]),
        "lc_bsa_forward_cached_ex": (S, [vp, vp, vp, vp, vp, vp, vp, I, I, I, I, F, vp, vp, vp,
                                         vp]),
        "lc_bsa_cond_cache": (S, [vp, vp, vp, vp, vp, vp, I, I, I, I, F, vp, vp, vp, vp]),
        "lc_bsa_backward": (S, [vp, vp, vp, vp, vp, vp, vp, vp, vp, I, I, I, I, F, vp, vp, vp,
                                vp]),
        "lc_bsa_plan_copy_csc": (S, [vp, vp, vp, vp]),
        "lc_bsa_forward_noalloc": (S, [vp, vp, vp, vp, vp, I, I, I, I, F, vp, vp, vp]),
        "lc_bsa_plan_create_shard": (S, [ctypes.POINTER(vp), I, I, I, I, I, I, I, I, I, I, I,
                                         vp]),
        "lc_bsa_plan_token_range": (S, [vp] + [ctypes.POINTER(LL)] * 4),
        "lc_bsa_forward_shard": (S, [vp, vp, vp, vp, vp, I, I, I, I, F, vp, vp, vp, vp]),
        "lc_bsa_lse_merge": (S, [vp, vp, vp, vp, vp, I, LL, I, I, I, ctypes.c_uint, vp]),
        "lc_bsa_lse_merge_parts": (S, [vp, vp, I, vp, vp, I, LL, I, I, I, vp]),
        "lc_rope3d_apply_ex": (S, [vp, vp, I, LL, I, I, LL, I, vp, F, vp, vp]),
        "lc_last_device_status": (S, [vp]),
        "lc_device_status_decode": (S, [I]),
        "lc_debug_watchdog_selftest": (S, [I, vp]),
        "lc_debug_scratch_pool_used_high": (S, [ctypes.POINTER(ctypes.c_ulonglong), I]),
        "lc_status_string": (ctypes.c_char_p, [S]),
        "lc_version": (ctypes.c_char_p, []),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype, fn.argtypes = res, args
    return lib


lib = _load()
COND_K_ROTATED = 1  # LC_FLAG_COND_K_ROTATED
Q_ROTATED = 2       # LC_FLAG_Q_ROTATED
K_ROTATED = 4       # LC_FLAG_K_ROTATED
KEEP_EMPTY_ROWS = 8  # LC_FLAG_KEEP_EMPTY_ROWS
OVERLAP_PREVIOUS = 16  # LC_FLAG_OVERLAP_PREVIOUS


def status_string(s: int) -> str:
    return lib.lc_status_string(int(s)).decode()


def version() -> str:
    return lib.lc_version().decode()


def _check(s: int, where: str):
    if s != LC_OK:
        raise LcError(s, where)


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return LC_DTYPE_BF16
    if t.dtype == torch.float32:
        return LC_DTYPE_F32
    raise TypeError("q/k/v must be bfloat16 or float32, got %s" % t.dtype)


def _check_bmhk(name: str, t: torch.Tensor, shape, dtype):
    if not t.is_cuda:
        raise ValueError("%s must be a CUDA tensor" % name)
    if not t.is_contiguous():
        raise ValueError("%s must be contiguous [B, N, heads, head_dim]" % name)
    if tuple(t.shape) != tuple(shape):
        raise ValueError("%s has shape %s, expected %s" % (name, tuple(t.shape), tuple(shape)))
    if t.dtype != dtype:
        raise ValueError("%s has dtype %s, expected %s" % (name, t.dtype, dtype))


class Plan:
    """Device-resident block-sparse plan (lc_bsa_plan_create), or, with
    q_blocks / k_blocks, the plan of one shard pair of ring context
    parallelism (lc_bsa_plan_create_shard): query blocks [lo, hi) against key
    blocks [lo, hi)."""

    def __init__(self, T: int, H: int, W: int, *, local: int, stride: int, n_cond: int = 0,
                 block: int = 64, q_blocks: Optional[Tuple[int, int]] = None,
                 k_blocks: Optional[Tuple[int, int]] = None, stream=None):
        self.T, self.H, self.W, self.n_cond = T, H, W, n_cond
        self.local, self.stride, self.block = local, stride, block
        h = ctypes.c_void_p()
        if q_blocks is None and k_blocks is None:
            _check(lib.lc_bsa_plan_create(ctypes.byref(h), T, H, W, block, local, stride, n_cond,
                                          _stream(stream)), "lc_bsa_plan_create")
        else:
            if q_blocks is None or k_blocks is None:
                raise ValueError("q_blocks and k_blocks go together")
            _check(lib.lc_bsa_plan_create_shard(ctypes.byref(h), T, H, W, block, local, stride,
                                                n_cond, int(q_blocks[0]), int(q_blocks[1]),
                                                int(k_blocks[0]), int(k_blocks[1]),
                                                _stream(stream)), "lc_bsa_plan_create_shard")
        self.handle = h
        r = [ctypes.c_longlong() for _ in range(4)]
        _check(lib.lc_bsa_plan_token_range(self.handle, *[ctypes.byref(x) for x in r]),
               "lc_bsa_plan_token_range")
        self.q_tokens = (r[0].value, r[1].value)  # whole-sequence token range of the queries
        self.k_tokens = (r[2].value, r[3].value)  # and of the keys

    def info(self) -> PlanInfo:
        inf = PlanInfo()
        _check(lib.lc_bsa_plan_info(self.handle, ctypes.byref(inf)), "lc_bsa_plan_info")
        return inf

    def csr(self, stream=None) -> Tuple[torch.Tensor, torch.Tensor]:
        inf = self.info()
        rp = torch.empty(inf.num_q_blocks + 1, dtype=torch.int32)
        ci = torch.empty(max(inf.nnz, 1), dtype=torch.int32)
        _check(lib.lc_bsa_plan_copy_csr(self.handle, rp.data_ptr(), ci.data_ptr(), _stream(stream)),
               "lc_bsa_plan_copy_csr")
        return rp, ci[:inf.nnz]

    def csc(self, stream=None) -> Tuple[torch.Tensor, torch.Tensor]:
        """Transpose of the block CSR: (col_ptr, row_idx), host int32."""
        inf = self.info()
        cp = torch.empty(inf.num_q_blocks + 1, dtype=torch.int32)
        ri = torch.empty(max(inf.nnz, 1), dtype=torch.int32)
        _check(lib.lc_bsa_plan_copy_csc(self.handle, cp.data_ptr(), ri.data_ptr(), _stream(stream)),
               "lc_bsa_plan_copy_csc")
        return cp, ri[:inf.nnz]

    @property
    def n_tokens(self) -> int:
        return self.T * self.H * self.W

    @property
    def n_cond_tokens(self) -> int:
        return self.n_cond * self.H * self.W

    def close(self, stream=None):
        if getattr(self, "handle", None):
            lib.lc_bsa_plan_destroy(self.handle, _stream(stream))
            self.handle = None

    def __del__(self):
        try:
            if getattr(self, "handle", None) and torch.cuda.is_available():
                lib.lc_bsa_plan_destroy(self.handle, None)
        except Exception:
            pass


class Rope3D:
    """Device-resident partitioned 3D-RoPE tables (lc_rope3d_tables)."""

    def __init__(self, T: int, H: int, W: int, theta: float = 10000.0,
                 dims: Sequence[int] = (16, 24, 24), stream=None):
        self.T, self.H, self.W, self.theta, self.dims = T, H, W, theta, tuple(dims)
        h = ctypes.c_void_p()
        _check(lib.lc_rope3d_tables(ctypes.byref(h), T, H, W, float(theta), *self.dims,
                                    _stream(stream)), "lc_rope3d_tables")
        self.handle = h

    def tables(self, stream=None) -> torch.Tensor:
        n = self.T * self.dims[0] + self.H * self.dims[1] + self.W * self.dims[2]
        out = torch.empty(n, dtype=torch.float32)
        _check(lib.lc_rope3d_copy_tables(self.handle, out.data_ptr(), _stream(stream)),
               "lc_rope3d_copy_tables")
        return out

    def apply(self, x: torch.Tensor, tok_offset: int = 0, out: Optional[torch.Tensor] = None,
              norm: Optional[torch.Tensor] = None, norm_eps: float = 1e-6,
              stream=None) -> torch.Tensor:
        """R(x), or R(norm(x)) with RMSNorm weights `norm` (lc_rope3d_apply_ex);
        token n of x is token n + tok_offset of the sequence."""
        B, n, heads, hd = x.shape
        if out is None:
            out = torch.empty_like(x)
        _check_bmhk("x", x, x.shape, x.dtype)
        _check_bmhk("out", out, x.shape, x.dtype)
        if norm is None:
            _check(lib.lc_rope3d_apply(x.data_ptr(), out.data_ptr(), B, n, heads, hd, tok_offset,
                                       _dtype_code(x), self.handle, _stream(stream)),
                   "lc_rope3d_apply")
        else:
            _opts(0, norm, None, norm_eps, hd)  # checks the weight tensor
            _check(lib.lc_rope3d_apply_ex(x.data_ptr(), out.data_ptr(), B, n, heads, hd,
                                          tok_offset, _dtype_code(x), norm.data_ptr(),
                                          float(norm_eps), self.handle, _stream(stream)),
                   "lc_rope3d_apply_ex")
        return out

    def close(self, stream=None):
        if getattr(self, "handle", None):
            lib.lc_rope3d_destroy(self.handle, _stream(stream))
            self.handle = None

    def __del__(self):
        try:
            if getattr(self, "handle", None) and torch.cuda.is_available():
                lib.lc_rope3d_destroy(self.handle, None)
        except Exception:
            pass


def _opts(flags: int = 0, q_norm: Optional[torch.Tensor] = None,
          k_norm: Optional[torch.Tensor] = None, norm_eps: float = 1e-6, hd: int = 64):
    """lc_bsa_opts for the _ex entry points, or None when nothing is set.
    q_norm / k_norm: fp32 [head_dim] device tensors (RMSNorm weights)."""
    for name, t in (("q_norm", q_norm), ("k_norm", k_norm)):
        if t is not None and (not t.is_cuda or t.dtype != torch.float32 or
                              tuple(t.shape) != (hd,) or not t.is_contiguous()):
            raise ValueError("%s must be a contiguous fp32 CUDA tensor of shape (%d,)" % (name, hd))
    if not flags and q_norm is None and k_norm is None:
        return None
    return Opts(flags, _ptr(q_norm), _ptr(k_norm), float(norm_eps))


def forward(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, plan: Plan, rope: Rope3D, *,
            out: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
            return_lse: bool = False, softmax_scale: float = 0.0,
            q_norm: Optional[torch.Tensor] = None, k_norm: Optional[torch.Tensor] = None,
            norm_eps: float = 1e-6, stream=None):
    """Block-sparse 3D-RoPE attention over the full sequence (lc_bsa_forward,
    or lc_bsa_forward_ex with RMSNorm weights q_norm / k_norm).

    q, k, v: [B, T*H*W, heads, 64], bf16 or fp32, on the plan's device.
    Returns out (and lse [B, heads, N] fp32 when asked)."""
    B, N, heads, hd = q.shape
    for name, t in (("k", k), ("v", v)):
        _check_bmhk(name, t, q.shape, q.dtype)
    _check_bmhk("q", q, (B, plan.n_tokens, heads, hd), q.dtype)
    if out is None:
        out = torch.empty_like(q)
    _check_bmhk("out", out, q.shape, q.dtype)
    if return_lse and lse is None:
        lse = torch.empty(B, heads, N, dtype=torch.float32, device=q.device)
    if lse is not None:
        _check_bmhk("lse", lse, (B, heads, N), torch.float32)
    opts = _opts(0, q_norm, k_norm, norm_eps, hd)
    if opts is not None:
        _check(lib.lc_bsa_forward_ex(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                                     _ptr(lse), B, heads, hd, _dtype_code(q), float(softmax_scale),
                                     ctypes.byref(opts), plan.handle, rope.handle,
                                     _stream(stream)), "lc_bsa_forward_ex")
    else:
        _check(lib.lc_bsa_forward(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                                  _ptr(lse), B, heads, hd, _dtype_code(q), float(softmax_scale),
                                  plan.handle, rope.handle, _stream(stream)), "lc_bsa_forward")
    return (out, lse) if (return_lse or lse is not None) else out


def forward_cached(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, cond_k: Optional[torch.Tensor],
                   cond_v: Optional[torch.Tensor], plan: Plan, rope: Rope3D, *,
                   out: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
                   return_lse: bool = False, softmax_scale: float = 0.0,
                   cond_k_rotated: bool = False, q_norm: Optional[torch.Tensor] = None,
                   k_norm: Optional[torch.Tensor] = None, norm_eps: float = 1e-6, stream=None):
    """Noisy-query attention with the condition tokens' K/V passed separately
    (lc_bsa_forward_cached / lc_bsa_forward_cached_ex).  q, k, v:
    [B, Nn, heads, 64]; cond_k, cond_v: [B, Nc, heads, 64], pre-RoPE, or
    already rotated (cond_k_rotated=True, e.g. from cond_cache)."""
    B, Nn, heads, hd = q.shape
    Nc = plan.n_cond_tokens
    _check_bmhk("q", q, (B, plan.n_tokens - Nc, heads, hd), q.dtype)
    for name, t in (("k", k), ("v", v)):
        _check_bmhk(name, t, q.shape, q.dtype)
    if Nc > 0:
        for name, t in (("cond_k", cond_k), ("cond_v", cond_v)):
            if t is None:
                raise ValueError("%s is required when the plan has condition frames" % name)
            _check_bmhk(name, t, (B, Nc, heads, hd), q.dtype)
    if out is None:
        out = torch.empty_like(q)
    _check_bmhk("out", out, q.shape, q.dtype)
    if return_lse and lse is None:
        lse = torch.empty(B, heads, Nn, dtype=torch.float32, device=q.device)
    if lse is not None:
        _check_bmhk("lse", lse, (B, heads, Nn), torch.float32)
    opts = _opts(COND_K_ROTATED if cond_k_rotated else 0, q_norm, k_norm, norm_eps, hd)
    if opts is not None:
        _check(lib.lc_bsa_forward_cached_ex(
            q.data_ptr(), k.data_ptr(), v.data_ptr(), _ptr(cond_k), _ptr(cond_v), out.data_ptr(),
            _ptr(lse), B, heads, hd, _dtype_code(q), float(softmax_scale), ctypes.byref(opts),
            plan.handle, rope.handle, _stream(stream)), "lc_bsa_forward_cached_ex")
    else:
        _check(lib.lc_bsa_forward_cached(q.data_ptr(), k.data_ptr(), v.data_ptr(), _ptr(cond_k),
                                         _ptr(cond_v), out.data_ptr(), _ptr(lse), B, heads, hd,
                                         _dtype_code(q), float(softmax_scale), plan.handle,
                                         rope.handle, _stream(stream)), "lc_bsa_forward_cached")
    return (out, lse) if (return_lse or lse is not None) else out


def backward(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, out: torch.Tensor,
             lse: torch.Tensor, dout: torch.Tensor, plan: Plan, rope: Rope3D, *,
             softmax_scale: float = 0.0, q_norm: Optional[torch.Tensor] = None,
             k_norm: Optional[torch.Tensor] = None, norm_eps: float = 1e-6, stream=None):
    """Gradients (dq, dk, dv) of forward() for dout (lc_bsa_backward); out and
    lse are the forward's results for the same q, k, v."""
    B, N, heads, hd = q.shape
    _check_bmhk("q", q, (B, plan.n_tokens, heads, hd), q.dtype)
    for name, t in (("k", k), ("v", v), ("out", out), ("dout", dout)):
        _check_bmhk(name, t, q.shape, q.dtype)
    _check_bmhk("lse", lse, (B, heads, N), torch.float32)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    opts = _opts(0, q_norm, k_norm, norm_eps, hd)
    _check(lib.lc_bsa_backward(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                               lse.data_ptr(), dout.data_ptr(), dq.data_ptr(), dk.data_ptr(),
                               dv.data_ptr(), B, heads, hd, _dtype_code(q), float(softmax_scale),
                               None if opts is None else ctypes.byref(opts), plan.handle,
                               rope.handle, _stream(stream)), "lc_bsa_backward")
    return dq, dk, dv


def cond_cache(cond_k: torch.Tensor, plan: Plan, rope: Rope3D, *,
               cond_q: Optional[torch.Tensor] = None, cond_v: Optional[torch.Tensor] = None,
               cond_k_rot: Optional[torch.Tensor] = None, cond_out: Optional[torch.Tensor] = None,
               cond_lse: Optional[torch.Tensor] = None, return_lse: bool = False,
               softmax_scale: float = 0.0, q_norm: Optional[torch.Tensor] = None,
               k_norm: Optional[torch.Tensor] = None, norm_eps: float = 1e-6, stream=None):
    """Producer side of the condition-token KV cache (lc_bsa_cond_cache):
    returns cond_k_rot = R(cond_k) and, when cond_q and cond_v are given, the
    condition tokens' own attention output (and lse with return_lse)."""
    B, Nc, heads, hd = cond_k.shape
    _check_bmhk("cond_k", cond_k, (B, plan.n_cond_tokens, heads, hd), cond_k.dtype)
    want_out = cond_q is not None or cond_v is not None
    if want_out:
        if cond_q is None or cond_v is None:
            raise ValueError("cond_q and cond_v go together")
        _check_bmhk("cond_q", cond_q, cond_k.shape, cond_k.dtype)
        _check_bmhk("cond_v", cond_v, cond_k.shape, cond_k.dtype)
    if cond_k_rot is None:
        cond_k_rot = torch.empty_like(cond_k)
    _check_bmhk("cond_k_rot", cond_k_rot, cond_k.shape, cond_k.dtype)
    if want_out and cond_out is None:
        cond_out = torch.empty_like(cond_k)
    if want_out and return_lse and cond_lse is None:
        cond_lse = torch.empty(B, heads, Nc, dtype=torch.float32, device=cond_k.device)
    if cond_out is not None:
        _check_bmhk("cond_out", cond_out, cond_k.shape, cond_k.dtype)
    if cond_lse is not None:
        _check_bmhk("cond_lse", cond_lse, (B, heads, Nc), torch.float32)
    opts = _opts(0, q_norm, k_norm, norm_eps, hd)
    _check(lib.lc_bsa_cond_cache(_ptr(cond_q), cond_k.data_ptr(), _ptr(cond_v),
                                 cond_k_rot.data_ptr(), _ptr(cond_out), _ptr(cond_lse), B, heads,
                                 hd, _dtype_code(cond_k), float(softmax_scale),
                                 None if opts is None else ctypes.byref(opts), plan.handle,
                                 rope.handle, _stream(stream)), "lc_bsa_cond_cache")
    if not want_out:
        return cond_k_rot
    return (cond_k_rot, cond_out, cond_lse) if cond_lse is not None else (cond_k_rot, cond_out)


def forward_noalloc(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, plan: Plan, rope: Rope3D,
                    *, out: torch.Tensor, lse: Optional[torch.Tensor] = None,
                    softmax_scale: float = 0.0, stream=None):
    """lc_bsa_forward_noalloc: the same attention as `forward` for callers
    that must not allocate device memory during the call; the caller passes
    `out` (and `lse` if wanted).  The library's scheduler counter lives in a
    fixed per-device array, so calls on one device must not overlap on the
    GPU; the first call on a device should come before any stream capture."""
    B, N, heads, hd = q.shape
    for name, t in (("k", k), ("v", v)):
        _check_bmhk(name, t, q.shape, q.dtype)
    _check_bmhk("q", q, (B, plan.n_tokens, heads, hd), q.dtype)
    _check_bmhk("out", out, q.shape, q.dtype)
    if lse is not None:
        _check_bmhk("lse", lse, (B, heads, N), torch.float32)
    _check(lib.lc_bsa_forward_noalloc(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                                      _ptr(lse), B, heads, hd, _dtype_code(q),
                                      float(softmax_scale), plan.handle, rope.handle,
                                      _stream(stream)), "lc_bsa_forward_noalloc")
    return out


def forward_shard(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, plan: Plan, rope: Rope3D,
                  *, out: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
                  softmax_scale: float = 0.0, q_norm: Optional[torch.Tensor] = None,
                  k_norm: Optional[torch.Tensor] = None, norm_eps: float = 1e-6,
                  q_rotated: bool = False, k_rotated: bool = False,
                  keep_empty_rows: bool = False, overlap_previous: bool = False, stream=None):
    """Partial attention of one shard pair (lc_bsa_forward_shard): q holds the
    shard plan's query tokens [B, nq, heads, 64], k / v its key tokens
    [B, nk, heads, 64] (pre-RoPE, bf16, or already normalised and rotated with
    q_rotated / k_rotated).  Returns (out, lse); rows that attend no key of
    the shard get out 0 and lse -inf."""
    B, nq, heads, hd = q.shape
    nk = plan.k_tokens[1] - plan.k_tokens[0]
    _check_bmhk("q", q, (B, plan.q_tokens[1] - plan.q_tokens[0], heads, hd), q.dtype)
    for name, t in (("k", k), ("v", v)):
        _check_bmhk(name, t, (B, nk, heads, hd), q.dtype)
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty(B, heads, nq, dtype=torch.float32, device=q.device)
    _check_bmhk("out", out, q.shape, q.dtype)
    _check_bmhk("lse", lse, (B, heads, nq), torch.float32)
    flags = ((Q_ROTATED if q_rotated else 0) | (K_ROTATED if k_rotated else 0) |
             (KEEP_EMPTY_ROWS if keep_empty_rows else 0) |
             (OVERLAP_PREVIOUS if overlap_previous else 0))
    opts = _opts(flags, q_norm, k_norm, norm_eps, hd)
    _check(lib.lc_bsa_forward_shard(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                                    lse.data_ptr(), B, heads, hd, _dtype_code(q),
                                    float(softmax_scale),
                                    None if opts is None else ctypes.byref(opts), plan.handle,
                                    rope.handle, _stream(stream)), "lc_bsa_forward_shard")
    return out, lse


MERGE_INIT = 1  # LC_MERGE_INIT


def lse_merge(o_acc: Optional[torch.Tensor], lse_acc: torch.Tensor, o_part: torch.Tensor,
              lse_part: torch.Tensor, *, out: Optional[torch.Tensor] = None, init: bool = False,
              stream=None):
    """Fold a partial result (o_part [B, n, heads, 64] bf16/fp32, lse_part
    [B, heads, n]) into a running one (o_acc fp32, lse_acc) by log-sum-exp
    (lc_bsa_lse_merge).  With `out` the merged o goes there (rounded to
    o_part's dtype) instead of o_acc; with init the running result is not read."""
    B, n, heads, hd = o_part.shape
    _check_bmhk("o_part", o_part, o_part.shape, o_part.dtype)
    _check_bmhk("lse_part", lse_part, (B, heads, n), torch.float32)
    _check_bmhk("lse_acc", lse_acc, (B, heads, n), torch.float32)
    if o_acc is not None:
        _check_bmhk("o_acc", o_acc, o_part.shape, torch.float32)
    if out is not None:
        _check_bmhk("out", out, o_part.shape, o_part.dtype)
    _check(lib.lc_bsa_lse_merge(_ptr(o_acc), lse_acc.data_ptr(), o_part.data_ptr(),
                                lse_part.data_ptr(), _ptr(out), B, n, heads, hd,
                                _dtype_code(o_part), MERGE_INIT if init else 0, _stream(stream)),
           "lc_bsa_lse_merge")
    return out if out is not None else o_acc


def lse_merge_parts(parts: torch.Tensor, lses: torch.Tensor, *, out: Optional[torch.Tensor] = None,
                    lse_out: Optional[torch.Tensor] = None, stream=None):
    """Combine P partial results over disjoint key sets in one pass
    (lc_bsa_lse_merge_parts): parts [P, B, n, heads, 64], lses [P, B, heads, n].
    Returns (out [B, n, heads, 64] of parts' dtype, lse [B, heads, n])."""
    P, B, n, heads, hd = parts.shape
    _check_bmhk("parts", parts, parts.shape, parts.dtype)
    _check_bmhk("lses", lses, (P, B, heads, n), torch.float32)
    if out is None:
        out = torch.empty(parts.shape[1:], dtype=parts.dtype, device=parts.device)
    if lse_out is None:
        lse_out = torch.empty(B, heads, n, dtype=torch.float32, device=parts.device)
    _check_bmhk("out", out, parts.shape[1:], parts.dtype)
    _check_bmhk("lse_out", lse_out, (B, heads, n), torch.float32)
    _check(lib.lc_bsa_lse_merge_parts(parts.data_ptr(), lses.data_ptr(), P, out.data_ptr(),
                                      lse_out.data_ptr(), B, n, heads, hd, _dtype_code(parts),
                                      _stream(stream)), "lc_bsa_lse_merge_parts")
    return out, lse_out


def last_device_status(stream=None) -> int:
    """Synchronise and return (and clear) the device status word as a status code."""
    return int(lib.lc_last_device_status(_stream(stream)))


def watchdog_selftest(timeout_us: int = 20000, stream=None) -> int:
    return int(lib.lc_debug_watchdog_selftest(int(timeout_us), _stream(stream)))


def scratch_pool_used_high(reset: bool = False) -> int:
    """High-water mark (bytes) of the library's scratch pool on the current
    device; with reset, the mark is first reset to the bytes in use now."""
    v = ctypes.c_ulonglong(0)
    _check(lib.lc_debug_scratch_pool_used_high(ctypes.byref(v), 1 if reset else 0),
           "lc_debug_scratch_pool_used_high")
    return int(v.value)
