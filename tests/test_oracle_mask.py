"""Pins of the oracle's block mask and block CSR (no GPU).

Pages: "longcat-video-rs" section 03-03 (local sliding-window blocks plus
strided global key/value blocks), section 02 table row (block=64, local=2,
stride=4), section 01 studio (16x16 block figure, 41.4 % attended, 58.6 % FLOP
saving); myzaker / QbitAI page, "背后技术原理" (condition tokens unaffected by
noise tokens; attention compute below 10 % at high resolution).
"""
import os

import numpy as np
import pytest

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden(name):
    vals = {}
    for line in open(os.path.join(GOLDEN, name)):
        line = line.split("#", 1)[0].strip()
        if line:
            k, v = line.split()
            vals[k] = v
    return vals


def closed_form_row_count(i, Nb, local, stride):
    """Window [lo, hi] plus the multiples of stride outside it."""
    lo, hi = max(0, i - local), min(Nb - 1, i + local)
    L = hi - lo + 1
    if stride <= 0:
        return L
    n_glob = -(-Nb // stride)                      # multiples of s in [0, Nb)
    in_win = hi // stride - (lo - 1) // stride if lo > 0 else hi // stride + 1
    return L + n_glob - in_win


@pytest.mark.parametrize("Nb,local,stride", [(16, 0, 3), (17, 2, 4), (585, 2, 4),
                                             (585, 2, 8), (585, 1, 16), (585, 1, 32),
                                             (1350, 1, 16), (40, 3, 0), (33, 0, 1),
                                             (9, 5, 7), (1, 2, 4)])
def test_row_counts_match_closed_form(Nb, local, stride):
    # one noisy segment of Nb full blocks: T*H*W = Nb*64 with H=1, W=64
    rp, ci = oracle.block_csr(Nb, 1, 64, 64, local, stride, 0)
    counts = np.diff(rp)
    for i in range(Nb):
        assert counts[i] == closed_form_row_count(i, Nb, local, stride), i
    # sorted, unique, in range
    for i in range(Nb):
        row = ci[rp[i]:rp[i + 1]]
        assert np.all(np.diff(row) > 0) and row.min() >= 0 and row.max() < Nb


def test_16x16_figure_of_the_page():
    g = _golden("mask_16x16_figure.txt")
    nb = int(g["blocks"])
    rp, _ = oracle.block_csr(nb, 1, 64, 64, int(g["local"]), int(g["stride"]), 0)
    ratio = 100.0 * rp[-1] / nb ** 2
    assert "%.1f" % ratio == g["attended_ratio_pct"]
    assert "%.1f" % (100.0 - ratio) == g["flop_saving_pct"]


def test_refine_720p_fraction():
    """720p refine workload (latent 24x45x80, local=1, stride=16, 1,350 blocks):
    specified at about 6.5 % of block pairs, and the page puts high-resolution
    attention compute under 10 % of dense."""
    rp, _ = oracle.block_csr(24, 45, 80, 64, 1, 16, 0)
    assert rp[-1] == 118544
    frac = 100.0 * rp[-1] / 1350 ** 2
    assert round(frac, 1) == 6.5
    assert frac < float(_golden("attention_fraction_highres.txt")["max_fraction_pct"])


def test_stride_one_is_dense_and_local_zero_is_diagonal():
    rp, ci = oracle.block_csr(10, 1, 64, 64, 0, 1, 0)
    assert rp[-1] == 100
    rp, ci = oracle.block_csr(10, 1, 64, 64, 0, 0, 0)
    np.testing.assert_array_equal(ci, np.arange(10))
    np.testing.assert_array_equal(rp, np.arange(11))


def test_condition_rows_and_columns():
    # I2V geometry: 1 condition frame of 30x52 = 1,560 tokens -> 25 blocks.
    T, H, W, nc = 24, 30, 52, 1
    Nc, Nn, Cb, Nb = oracle.segment_sizes(T, H, W, nc)
    assert (Nc, Nn, Cb, Nb) == (1560, 35880, 25, 561)
    rp, ci = oracle.block_csr(T, H, W, 64, 2, 4, nc)
    for r in range(Cb):                       # condition rows: condition blocks only
        np.testing.assert_array_equal(ci[rp[r]:rp[r + 1]], np.arange(Cb))
    for r in range(Cb, Cb + Nb):              # noisy rows: all condition blocks first
        row = ci[rp[r]:rp[r + 1]]
        np.testing.assert_array_equal(row[:Cb], np.arange(Cb))
        assert len(row) - Cb == closed_form_row_count(r - Cb, Nb, 2, 4)
    assert rp[-1] == 625 + 561 * 25 + 81199


def test_token_mask_agrees_with_block_csr_on_small_grids():
    """The token-level predicate and the block CSR are written separately;
    the number of attended token pairs must equal the sum over CSR entries of
    (query block size) x (key block size), partial tail blocks included."""
    for (T, H, W, nc, local, stride) in [(4, 8, 16, 0, 2, 4), (5, 3, 7, 1, 1, 3),
                                         (6, 5, 9, 2, 0, 0), (3, 4, 11, 1, 2, 1)]:
        Nc, Nn, Cb, Nb = oracle.segment_sizes(T, H, W, nc)
        rp, ci = oracle.block_csr(T, H, W, 64, local, stride, nc)

        def bsize(b):
            if b < Cb:
                return min(64, Nc - 64 * b)
            return min(64, Nn - 64 * (b - Cb))

        expect = 0
        for r in range(Cb + Nb):
            for c in ci[rp[r]:rp[r + 1]]:
                expect += bsize(r) * bsize(c)
        got = oracle.count_token_pairs(T * H * W, Nc, 64, local, stride)
        assert got == expect


def test_condition_tokens_never_see_noise_tokens():
    Nc = 100
    for n in range(0, 300, 7):
        for m in range(0, 300, 5):
            if n < Nc and m >= Nc:
                assert not oracle.token_allowed(n, m, Nc, 64, 2, 4)
            if n >= Nc and m < Nc:
                assert oracle.token_allowed(n, m, Nc, 64, 0, 0)


def test_random_geometries_csr_against_token_mask():
    """Seeded random small geometries: the brute-force block CSR, the closed
    row counts and the token-level pair count agree (every attended block pair
    contributes exactly its two blocks' token counts)."""
    from oracle.backward import token_mask
    rng = np.random.default_rng(2024)
    for _ in range(25):
        T = int(rng.integers(1, 6))
        H, W = int(rng.integers(1, 9)), int(rng.integers(1, 40))
        n_cond = int(rng.integers(0, T))
        local, stride = int(rng.integers(0, 4)), int(rng.integers(-1, 7))
        Nc, Nn, Cb, Nb = oracle.segment_sizes(T, H, W, n_cond)
        N = Nc + Nn
        rp, ci = oracle.block_csr(T, H, W, 64, local, stride, n_cond)
        assert rp[-1] == len(ci)
        for i in range(Nb):
            assert rp[Cb + i + 1] - rp[Cb + i] == Cb + closed_form_row_count(i, Nb, local, stride)
        def ntok(b):
            return min(64, Nc - 64 * b) if b < Cb else min(64, Nn - 64 * (b - Cb))
        pairs = sum(ntok(r) * ntok(int(c)) for r in range(Cb + Nb) for c in ci[rp[r]:rp[r + 1]])
        assert pairs == int(token_mask(N, Nc, 64, local, stride).sum())


def test_every_frame_a_condition_frame_is_refused():
    """At least one frame is generated: n_cond == T is outside the domain on
    both sides of the boundary (lc_bsa_plan_create refuses it as well)."""
    with pytest.raises(ValueError):
        oracle.segment_sizes(4, 8, 16, 4)
    with pytest.raises(ValueError):
        oracle.block_csr(4, 8, 16, 64, 2, 4, 4)
    assert oracle.segment_sizes(4, 8, 16, 3) == (384, 128, 6, 2)
