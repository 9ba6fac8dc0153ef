"""Pins for the oracle's square-window variant (the comparison mask the pages contrast the circular
window with): image tokens kept iff |dx| < r and |dy| < r, clipped at the border. Each test checks
the oracle against something other than itself."""
import math

import numpy as np
import pytest
import torch
from scipy.special import logsumexp

import oracle
from clear_inputs import make_random


def _rand(shape, seed):
    return make_random(shape, seed, dtype=torch.float64).numpy()


def _brute_force_square(q, k, v, n_text, H, W, r):
    """Per-query key lists gathered with the Chebyshev test, then a textbook softmax."""
    _, _, T, d = q.shape
    scale = 1.0 / math.sqrt(d)
    O = np.zeros((T, d))
    L = np.zeros(T)
    for i in range(T):
        if i < n_text:
            keys = list(range(T))
        else:
            yi, xi = divmod(i - n_text, W)
            keys = list(range(n_text)) + [n_text + yj * W + xj for yj in range(H) for xj in range(W)
                                          if max(abs(yi - yj), abs(xi - xj)) < r]
        s = q[0, 0, i] @ k[0, 0, keys].T * scale
        lse = logsumexp(s)
        O[i] = np.exp(s - lse) @ v[0, 0, keys]
        L[i] = lse
    return O, L


@pytest.mark.parametrize("n_text,H,W", [(0, 4, 4), (3, 5, 7), (5, 8, 3)])
def test_square_matches_brute_force(n_text, H, W):
    T = n_text + H * W
    q, k, v = (_rand((1, 1, T, 8), s) for s in (40, 41, 42))
    for r in range(1, 9):
        O, LSE = oracle.clear_attention_forward(q, k, v, n_text, H, W, r, window="square")
        Ob, Lb = _brute_force_square(q, k, v, n_text, H, W, r)
        np.testing.assert_allclose(O[0, 0], Ob, rtol=0, atol=1e-12)
        np.testing.assert_allclose(LSE[0, 0], Lb, rtol=0, atol=1e-12)


@pytest.mark.parametrize("r", [1, 2, 4, 8, 16])
def test_square_interior_row_count(r):
    H = W = 4 * r + 3
    y, x = H // 2, W // 2
    M = oracle.clear_mask(0, H, W, r, rows=[y * W + x], window="square")
    assert M.sum() == (2 * r - 1) ** 2 == oracle.window_lattice_count(r, "square")


@pytest.mark.parametrize("n_text,H,W,r", [(0, 7, 9, 3), (4, 16, 16, 4), (3, 10, 5, 6), (2, 4, 4, 30)])
def test_square_kept_pairs_equals_mask_sum(n_text, H, W, r):
    M = oracle.clear_mask(n_text, H, W, r, window="square")
    assert M.sum() == oracle.kept_pairs(n_text, H, W, r, "square")
    # Separable: the clipped overlaps factor into a row part and a column part.
    rows = sum(H - abs(dy) for dy in range(-(r - 1), r) if abs(dy) < H)
    cols = sum(W - abs(dx) for dx in range(-(r - 1), r) if abs(dx) < W)
    assert oracle.window_pairs(H, W, r, "square") == rows * cols


@pytest.mark.parametrize("n_text,H,W,r", [(3, 6, 9, 2), (0, 12, 12, 5), (2, 5, 5, 3), (1, 9, 9, 4)])
def test_circle_is_inside_square(n_text, H, W, r):
    c = oracle.clear_mask(n_text, H, W, r, window="circle")
    s = oracle.clear_mask(n_text, H, W, r, window="square")
    assert not (c & ~s).any()
    # The square's corner offset (r-1, r-1) leaves the disc iff 2 (r-1)^2 >= r^2, i.e. r >= 4;
    # below that the two windows coincide.
    assert (s & ~c).any() == (r >= 4)


def test_circle_to_square_ratio_tends_to_pi_over_4():
    # [pith review, "What carries the argument"]: the circle costs about pi/4 of the square.
    for r, tol in [(64, 0.02), (256, 0.005), (1024, 0.0013)]:
        ratio = oracle.window_lattice_count(r) / oracle.window_lattice_count(r, "square")
        assert abs(ratio - math.pi / 4) < tol


@pytest.mark.parametrize("n_text,H,W", [(4, 6, 9), (0, 5, 5)])
def test_square_full_radius_is_full_attention(n_text, H, W):
    T = n_text + H * W
    q, k, v = (_rand((1, 1, T, 8), s) for s in (50, 51, 52))
    O, LSE = oracle.clear_attention_forward(q, k, v, n_text, H, W, max(H, W), window="square")
    s = q[0, 0] @ k[0, 0].T / math.sqrt(8)
    lse = logsumexp(s, axis=1)
    np.testing.assert_allclose(O[0, 0], np.exp(s - lse[:, None]) @ v[0, 0], rtol=0, atol=1e-12)
    np.testing.assert_allclose(LSE[0, 0], lse, rtol=0, atol=1e-12)


def test_square_backward_finite_differences():
    n_text, H, W, r, d = 2, 4, 4, 2, 4
    T = n_text + H * W
    q, k, v, dO = (_rand((1, 1, T, d), s) for s in (60, 61, 62, 63))
    dq, dk, dv = oracle.clear_attention_backward(q, k, v, dO, n_text, H, W, r, window="square")

    def loss(qq, kk, vv):
        O, _ = oracle.clear_attention_forward(qq, kk, vv, n_text, H, W, r, window="square")
        return float((O * dO).sum())

    h = 1e-6
    for name, x, g in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        for idx in [(0, 0, 0, 0), (0, 0, n_text + 5, 1), (0, 0, T - 1, 3)]:
            xp, xm = x.copy(), x.copy()
            xp[idx] += h
            xm[idx] -= h
            args_p = [xp if n == name else a for n, a in (("q", q), ("k", k), ("v", v))]
            args_m = [xm if n == name else a for n, a in (("q", q), ("k", k), ("v", v))]
            fd = (loss(*args_p) - loss(*args_m)) / (2 * h)
            assert abs(fd - g[idx]) < 1e-6 * max(1.0, abs(fd)), (name, idx, fd, g[idx])


# ------------------------------------------------------------------------------------------------
# Border-shifted square window (neighborhood-attention style): constant key count per query.
# ------------------------------------------------------------------------------------------------

def _shifted_keys_by_window_start(yi, xi, H, W, r):
    """Independent formulation: the window's first row / column is the query's minus (r-1),
    pushed back inside the grid; the window is 2r-1 wide."""
    k = 2 * r - 1
    y0 = min(max(yi - (r - 1), 0), H - k)
    x0 = min(max(xi - (r - 1), 0), W - k)
    return [(yj, xj) for yj in range(y0, y0 + k) for xj in range(x0, x0 + k)]


@pytest.mark.parametrize("n_text,H,W,r", [(0, 7, 9, 3), (3, 5, 5, 3), (2, 11, 8, 2), (1, 9, 13, 4)])
def test_shifted_mask_matches_window_start_formulation(n_text, H, W, r):
    M = oracle.clear_mask(n_text, H, W, r, window="shifted")
    for i in range(n_text, n_text + H * W):
        yi, xi = divmod(i - n_text, W)
        ref = np.zeros(n_text + H * W, dtype=bool)
        ref[:n_text] = True
        for yj, xj in _shifted_keys_by_window_start(yi, xi, H, W, r):
            ref[n_text + yj * W + xj] = True
        assert (M[i] == ref).all(), (yi, xi)
        assert M[i, n_text:].sum() == (2 * r - 1) ** 2  # constant count, corners included
    assert M.sum() == oracle.kept_pairs(n_text, H, W, r, "shifted")


def test_shifted_equals_square_away_from_the_border():
    n_text, H, W, r = 2, 13, 14, 3
    sh = oracle.clear_mask(n_text, H, W, r, window="shifted")
    sq = oracle.clear_mask(n_text, H, W, r, window="square")
    differs = 0
    for y in range(H):
        for x in range(W):
            i = n_text + y * W + x
            if r - 1 <= y <= H - r and r - 1 <= x <= W - r:
                assert (sh[i] == sq[i]).all(), (y, x)  # interior: the window is not shifted
            else:
                differs += int(not (sh[i] == sq[i]).all())
    assert differs == H * W - (H - 2 * (r - 1)) * (W - 2 * (r - 1))  # every border query is shifted
    assert not (sh == sh.T).all()  # border queries see farther keys than those keys see them back


def test_shifted_window_as_large_as_the_grid_is_full_attention():
    n_text, H, W, r = 3, 5, 5, 3  # 2r - 1 = 5: every window is the whole grid
    T = n_text + H * W
    q, k, v = (_rand((1, 1, T, 8), s) for s in (70, 71, 72))
    O, LSE = oracle.clear_attention_forward(q, k, v, n_text, H, W, r, window="shifted")
    s = q[0, 0] @ k[0, 0].T / math.sqrt(8)
    lse = logsumexp(s, axis=1)
    np.testing.assert_allclose(O[0, 0], np.exp(s - lse[:, None]) @ v[0, 0], rtol=0, atol=1e-12)


def test_shifted_forward_matches_brute_force():
    n_text, H, W, r = 2, 6, 7, 2
    T = n_text + H * W
    q, k, v = (_rand((1, 1, T, 8), s) for s in (80, 81, 82))
    O, LSE = oracle.clear_attention_forward(q, k, v, n_text, H, W, r, window="shifted")
    for i in range(T):
        if i < n_text:
            keys = list(range(T))
        else:
            yi, xi = divmod(i - n_text, W)
            keys = list(range(n_text)) + [n_text + yj * W + xj for yj, xj in _shifted_keys_by_window_start(yi, xi, H, W, r)]
        s = q[0, 0, i] @ k[0, 0, keys].T / math.sqrt(8)
        lse = logsumexp(s)
        np.testing.assert_allclose(O[0, 0, i], np.exp(s - lse) @ v[0, 0, keys], rtol=0, atol=1e-12)
        assert abs(LSE[0, 0, i] - lse) < 1e-12
