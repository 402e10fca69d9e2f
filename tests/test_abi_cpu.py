"""The C-ABI library loads, exports every symbol its header declares, and
rejects bad arguments before touching the GPU (runs without a GPU)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "lc_bsa.h")


@pytest.fixture(scope="module")
def lib():
    from block_sparse_attention_rope_b200 import build
    path = build.build()
    return ctypes.CDLL(path)


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(lc_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for must in ["lc_bsa_plan_create", "lc_bsa_plan_destroy", "lc_bsa_plan_info",
                 "lc_bsa_plan_copy_csr", "lc_rope3d_tables", "lc_rope3d_destroy",
                 "lc_bsa_forward", "lc_bsa_forward_cached", "lc_last_device_status",
                 "lc_status_string"]:
        assert must in names


def test_every_declared_symbol_is_exported(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name


def test_status_strings(lib):
    lib.lc_status_string.restype = ctypes.c_char_p
    seen = set()
    for code in range(7):
        s = lib.lc_status_string(code).decode()
        assert s and s != "unknown status"
        seen.add(s)
    assert len(seen) == 7
    assert lib.lc_status_string(99).decode() == "unknown status"


def test_device_status_word_decoding(lib):
    """The device status word's bits map to the codes lc_last_device_status
    returns: bit 0 (a bounded wait gave up) before bit 1 (a failed in-kernel
    check of the plan's lists)."""
    f = lib.lc_device_status_decode
    f.argtypes, f.restype = [ctypes.c_int], ctypes.c_int
    assert f(0) == 0
    assert f(1) == 5       # LC_ERR_TIMEOUT
    assert f(2) == 6       # LC_ERR_DEVICE_CHECK
    assert f(3) == 5
    assert f(4) == 0       # bits the kernels never set


def test_plan_argument_errors_before_any_gpu_work(lib):
    h = ctypes.c_void_p()
    f = lib.lc_bsa_plan_create
    f.argtypes = [ctypes.POINTER(ctypes.c_void_p)] + [ctypes.c_int] * 7 + [ctypes.c_void_p]
    assert f(None, 4, 8, 16, 64, 2, 4, 0, None) == 1
    assert f(ctypes.byref(h), 0, 8, 16, 64, 2, 4, 0, None) == 1        # T <= 0
    assert f(ctypes.byref(h), 4, 8, 16, 64, -1, 4, 0, None) == 1       # local < 0
    assert f(ctypes.byref(h), 4, 8, 16, 64, 2, 4, 4, None) == 1        # n_cond >= T
    assert f(ctypes.byref(h), 4, 8, 16, 32, 2, 4, 0, None) == 2        # block != 64
    assert f(ctypes.byref(h), 4096, 64, 64, 64, 2, 4, 0, None) == 2    # > 2^24 tokens
    assert h.value is None


def test_rope_argument_errors(lib):
    h = ctypes.c_void_p()
    f = lib.lc_rope3d_tables
    f.argtypes = [ctypes.POINTER(ctypes.c_void_p), ctypes.c_int, ctypes.c_int, ctypes.c_int,
                  ctypes.c_double, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_void_p]
    assert f(ctypes.byref(h), 4, 8, 16, 0.0, 16, 24, 24, None) == 1    # theta
    assert f(ctypes.byref(h), 4, 8, 16, 1e4, 15, 25, 24, None) == 1    # odd dims
    assert f(ctypes.byref(h), 4, 8, 16, 1e4, 32, 16, 16, None) == 2    # other split
    assert h.value is None


def test_forward_rejects_null_handles(lib):
    f = lib.lc_bsa_forward
    f.argtypes = [ctypes.c_void_p] * 5 + [ctypes.c_int] * 4 + [ctypes.c_float] + [ctypes.c_void_p] * 3
    assert f(None, None, None, None, None, 1, 2, 64, 0, 0.0, None, None, None) == 1
    g = lib.lc_bsa_forward_cached
    g.argtypes = [ctypes.c_void_p] * 7 + [ctypes.c_int] * 4 + [ctypes.c_float] + [ctypes.c_void_p] * 3
    assert g(None, None, None, None, None, None, None, 1, 2, 64, 0, 0.0, None, None, None) == 1


def test_other_entry_points_reject_bad_arguments_before_any_gpu_work(lib):
    """The _ex forwards, the cache producer, the backward, the allocation-free
    forward and the plan / table accessors return LC_ERR_INVALID_ARGUMENT for
    NULL tensors, handles or outputs (and for bad options) on a machine
    without a GPU: none of them reaches a CUDA call first."""
    vp, I, F = ctypes.c_void_p, ctypes.c_int, ctypes.c_float

    class Opts(ctypes.Structure):
        _fields_ = [("flags", ctypes.c_uint), ("q_norm_weight", vp), ("k_norm_weight", vp),
                    ("norm_eps", F)]

    bad_flags = Opts(flags=64)
    bad_eps = Opts(flags=0, norm_eps=-1.0)
    f = lib.lc_bsa_forward_ex
    f.argtypes = [vp] * 5 + [I] * 4 + [F] + [vp] * 4
    g = lib.lc_bsa_forward_cached_ex
    g.argtypes = [vp] * 7 + [I] * 4 + [F] + [vp] * 4
    c = lib.lc_bsa_cond_cache
    c.argtypes = [vp] * 6 + [I] * 4 + [F] + [vp] * 4
    b = lib.lc_bsa_backward
    b.argtypes = [vp] * 9 + [I] * 4 + [F] + [vp] * 4
    for opts in (None, ctypes.byref(bad_flags), ctypes.byref(bad_eps)):
        assert f(None, None, None, None, None, 1, 2, 64, 0, 0.0, opts, None, None, None) == 1
        assert g(*[None] * 7, 1, 2, 64, 0, 0.0, opts, None, None, None) == 1
        assert c(*[None] * 6, 1, 2, 64, 0, 0.0, opts, None, None, None) == 1
        assert b(*[None] * 9, 1, 2, 64, 0, 0.0, opts, None, None, None) == 1
    n = lib.lc_bsa_forward_noalloc
    n.argtypes = [vp] * 5 + [I] * 4 + [F] + [vp] * 3
    assert n(None, None, None, None, None, 1, 2, 64, 0, 0.0, None, None, None) == 1
    for name, nargs in (("lc_bsa_plan_info", 2), ("lc_bsa_plan_copy_csc", 4),
                        ("lc_bsa_plan_copy_csr", 4), ("lc_bsa_plan_token_range", 5),
                        ("lc_rope3d_copy_tables", 3)):
        fn = getattr(lib, name)
        fn.argtypes = [vp] * nargs
        assert fn(*[None] * nargs) == 1, name
    s = lib.lc_debug_scratch_pool_used_high
    s.argtypes = [vp, I]
    assert s(None, 0) == 1
    # destroying a NULL handle is a no-op
    for name in ("lc_bsa_plan_destroy", "lc_rope3d_destroy"):
        fn = getattr(lib, name)
        fn.argtypes = [vp, vp]
        assert fn(None, None) == 0, name


def test_python_binding_imports_only_the_library():
    """The binding module must not reach the oracle (no CPU fallback)."""
    src = open(os.path.join(ROOT, "block_sparse_attention_rope_b200", "api.py")).read()
    assert "oracle" not in src.replace("no CPU fallback", "")
    for f in os.listdir(os.path.join(ROOT, "block_sparse_attention_rope_b200", "csrc")):
        assert "oracle" not in open(os.path.join(ROOT, "block_sparse_attention_rope_b200",
                                                 "csrc", f)).read().lower()


def test_ring_entry_points_reject_bad_arguments(lib):
    vp, I, LL, F = ctypes.c_void_p, ctypes.c_int, ctypes.c_longlong, ctypes.c_float
    h = ctypes.c_void_p()
    f = lib.lc_bsa_plan_create_shard
    f.argtypes = [ctypes.POINTER(vp)] + [I] * 11 + [vp]
    # T=5, H=8, W=40, 2 condition frames: Cb = 10, Nb = 15 (25 blocks)
    assert f(None, 5, 8, 40, 64, 1, 2, 2, 0, 4, 0, 25, None) == 1
    assert f(ctypes.byref(h), 5, 8, 40, 64, 1, 2, 2, 0, 6, 0, 25, None) == 1   # inside a group
    assert f(ctypes.byref(h), 5, 8, 40, 64, 1, 2, 2, 10, 13, 0, 25, None) == 1  # inside a group
    assert f(ctypes.byref(h), 5, 8, 40, 64, 1, 2, 2, 0, 4, 0, 26, None) == 1   # past the end
    assert f(ctypes.byref(h), 5, 8, 40, 64, 1, 2, 2, 4, 0, 0, 25, None) == 1   # lo > hi
    assert f(ctypes.byref(h), 5, 8, 40, 64, 1, 2, 2, 0, -1, 0, 25, None) == 1
    assert h.value is None
    g = lib.lc_bsa_forward_shard
    g.argtypes = [vp] * 5 + [I] * 4 + [F] + [vp] * 4
    assert g(None, None, None, None, None, 1, 2, 64, 0, 0.0, None, None, None, None) == 1
    m = lib.lc_bsa_lse_merge
    m.argtypes = [vp] * 5 + [I, LL, I, I, I, ctypes.c_uint, vp]
    buf = ctypes.create_string_buffer(4096 + 16)
    a = (ctypes.addressof(buf) + 15) & ~15
    assert m(None, a, a, a, None, 1, 4, 2, 64, 0, 0, None) == 1       # o_acc needed
    assert m(a, a, a, a, None, 1, 4, 2, 64, 0, 8, None) == 1          # unknown flag
    assert m(a, a, a, a, None, 1, 4, 2, 32, 0, 0, None) == 2          # head_dim
    assert m(a, a, a + 4, a, None, 1, 4, 2, 64, 0, 0, None) == 1      # misaligned part
    p = lib.lc_bsa_lse_merge_parts
    p.argtypes = [vp, vp, I, vp, vp, I, LL, I, I, I, vp]
    assert p(a, a, 0, a, None, 1, 4, 2, 64, 0, None) == 1             # no parts
    assert p(None, a, 2, a, None, 1, 4, 2, 64, 0, None) == 1
    assert p(a, a, 2, a, None, 1, 4, 2, 32, 0, None) == 2
    r = lib.lc_rope3d_apply_ex
    r.argtypes = [vp, vp, I, LL, I, I, LL, I, vp, F, vp, vp]
    assert r(None, None, 1, 4, 2, 64, 0, 0, None, 0.0, None, None) == 1


def test_package_never_reaches_the_oracle():
    pkg = os.path.join(ROOT, "block_sparse_attention_rope_b200")
    for f in ("api.py", "ring.py", "build.py", "__init__.py"):
        src = open(os.path.join(pkg, f)).read()
        assert "import oracle" not in src and "from oracle" not in src, f
