"""Pins of the oracle's partitioned 3D-RoPE against what the pages and the
mathematics fix (no GPU).

Page: "longcat-video-rs", header card "PARTITIONED 3D-ROPE 16T + 24H + 24W" and
section 03-01: each 64-D head is split into 16 temporal, 24 vertical and 24
horizontal channels, rotated as norm-preserving complex pairs.
"""
import os

import numpy as np
import pytest

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
THETA = 10000.0


def _golden(name):
    vals = {}
    for line in open(os.path.join(GOLDEN, name)):
        line = line.split("#", 1)[0].strip()
        if line:
            k, v = line.split()
            vals[k] = v
    return vals


def _rope1d_complex(x, pos, theta=THETA):
    """Textbook 1-D rotary embedding in complex form: pair k of a d-channel
    vector, read as x[2k] + i x[2k+1], is multiplied by exp(i pos theta^(-2k/d))."""
    d = x.shape[-1]
    z = x[0::2] + 1j * x[1::2]
    k = np.arange(d // 2)
    z = z * np.exp(1j * pos * theta ** (-2.0 * k / d))
    out = np.empty(d)
    out[0::2], out[1::2] = z.real, z.imag
    return out


def test_norm_conservation_matches_page_figure():
    printed = _golden("rope_norm_conservation.txt")["norm_ratio"]
    rng = np.random.default_rng(0)
    worst = 0.0
    for _ in range(200):
        x = rng.standard_normal(64)
        t, h, w = rng.integers(0, 100, size=3)
        y = oracle.rope3d_rotate_vec(x, int(t), int(h), int(w))
        ratio = np.linalg.norm(y) / np.linalg.norm(x)
        assert "%.5f" % ratio == printed
        worst = max(worst, abs(ratio - 1.0))
    assert worst < 1e-14


def test_origin_is_identity():
    x = np.random.default_rng(1).standard_normal(64)
    np.testing.assert_array_equal(oracle.rope3d_rotate_vec(x, 0, 0, 0), x)


@pytest.mark.parametrize("axis,lo,hi", [(0, 0, 16), (1, 16, 40), (2, 40, 64)])
def test_each_axis_is_textbook_1d_rope_on_its_channels(axis, lo, hi):
    """Moving along one axis rotates exactly that axis' channel slice, as
    1-D RoPE of that width at that position; the other channels stay put."""
    rng = np.random.default_rng(2 + axis)
    x = rng.standard_normal(64)
    for pos in [1, 2, 7, 23, 79]:
        p = [0, 0, 0]
        p[axis] = pos
        y = oracle.rope3d_rotate_vec(x, *p)
        np.testing.assert_allclose(y[lo:hi], _rope1d_complex(x[lo:hi], pos), rtol=0, atol=1e-13)
        rest = np.r_[0:lo, hi:64]
        np.testing.assert_array_equal(y[rest], x[rest])


def test_first_pair_turns_by_position_radians():
    # omega_0 = theta^0 = 1 on every axis: pair 0 of an axis turns by pos rad.
    for axis, c in [(0, 0), (1, 16), (2, 40)]:
        x = np.zeros(64)
        x[c] = 1.0
        p = [0, 0, 0]
        p[axis] = 3
        y = oracle.rope3d_rotate_vec(x, *p)
        assert abs(y[c] - np.cos(3.0)) < 1e-15 and abs(y[c + 1] - np.sin(3.0)) < 1e-15


def test_composition():
    rng = np.random.default_rng(5)
    for _ in range(20):
        x = rng.standard_normal(64)
        a = rng.integers(0, 40, size=3)
        b = rng.integers(0, 40, size=3)
        y = oracle.rope3d_rotate_vec(oracle.rope3d_rotate_vec(x, *map(int, a)), *map(int, b))
        z = oracle.rope3d_rotate_vec(x, *map(int, a + b))
        np.testing.assert_allclose(y, z, rtol=0, atol=1e-12)


def test_relative_position_property():
    """<R(p) q, R(p') k> = <q, R(p' - p) k>: scores depend on offsets only."""
    rng = np.random.default_rng(6)
    for _ in range(20):
        q, k = rng.standard_normal(64), rng.standard_normal(64)
        p = rng.integers(0, 50, size=3)
        pp = rng.integers(0, 50, size=3)
        lhs = oracle.rope3d_rotate_vec(q, *map(int, p)) @ oracle.rope3d_rotate_vec(k, *map(int, pp))
        rhs = q @ oracle.rope3d_rotate_vec(k, *map(int, pp - p))
        assert abs(lhs - rhs) < 1e-11


def test_token_positions_follow_t_h_w_order():
    """rope3d_apply on a [1, T*H*W, 1, 64] sequence: token n is rotated at
    t = n // (H W), h = (n // W) % H, w = n % W.  Checked structurally: the
    next token along w differs only in the W slice, by one unit turn; the next
    along h only in the H slice; the next frame only in the T slice."""
    T, H, W = 3, 4, 5
    x = np.tile(np.random.default_rng(7).standard_normal(64), (1, T * H * W, 1, 1))
    y = oracle.rope3d_apply(x, H, W)
    base = x[0, 0, 0]

    def tok(t, h, w):
        return y[0, (t * H + h) * W + w, 0]

    for t in range(T):
        for h in range(H):
            for w in range(W):
                v = tok(t, h, w)
                np.testing.assert_allclose(v[0:16], _rope1d_complex(base[0:16], t), atol=1e-13)
                np.testing.assert_allclose(v[16:40], _rope1d_complex(base[16:40], h), atol=1e-13)
                np.testing.assert_allclose(v[40:64], _rope1d_complex(base[40:64], w), atol=1e-13)


def test_token_offset_equals_slice_of_longer_sequence():
    T, H, W = 4, 3, 5
    rng = np.random.default_rng(8)
    x = rng.standard_normal((2, T * H * W, 3, 64))
    full = oracle.rope3d_apply(x, H, W)
    off = 2 * H * W
    tail = oracle.rope3d_apply(x[:, off:], H, W, tok_offset=off)
    np.testing.assert_array_equal(tail, full[:, off:])
