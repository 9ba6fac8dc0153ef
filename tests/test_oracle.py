"""Pins for the float64 CPU oracle: each test checks the oracle against something other than
itself (printed figures, closed forms, brute force, textbook routines, invariants)."""
import json
import math
import os

import numpy as np
import pytest
import torch
from scipy.special import logsumexp

import oracle
from clear_inputs import make_random

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rand(shape, seed):
    return make_random(shape, seed, dtype=torch.float64).numpy()


def _dense_softmax_attention(q, k, v, scale):
    """Textbook full attention written independently (scipy logsumexp), one (b, h) at a time."""
    S = q @ k.T * scale
    lse = logsumexp(S, axis=1)
    P = np.exp(S - lse[:, None])
    return P @ v, lse


# ------------------------------------------------------------------------------------------------
# Special case: r at least the grid diagonal reduces to full joint softmax attention.
# ------------------------------------------------------------------------------------------------

@pytest.mark.parametrize("n_text,H,W", [(16, 16, 16), (3, 5, 7), (0, 6, 4)])
def test_large_radius_is_full_attention(n_text, H, W):
    d = 16
    T = n_text + H * W
    r = math.isqrt((H - 1) ** 2 + (W - 1) ** 2) + 1  # r^2 > diagonal^2: every pair is kept
    q, k, v = (_rand((1, 2, T, d), s) for s in (1, 2, 3))
    O, LSE = oracle.clear_attention_forward(q, k, v, n_text, H, W, r)
    for h in range(2):
        ref_o, ref_lse = _dense_softmax_attention(q[0, h], k[0, h], v[0, h], 1 / math.sqrt(d))
        np.testing.assert_allclose(O[0, h], ref_o, rtol=0, atol=1e-12)
        np.testing.assert_allclose(LSE[0, h], ref_lse, rtol=0, atol=1e-12)
    # Second, library cross-check: torch SDPA in float64 on the CPU.
    sdpa = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q), torch.from_numpy(k), torch.from_numpy(v))
    np.testing.assert_allclose(O, sdpa.numpy(), rtol=0, atol=1e-12)


def test_radius_just_below_diagonal_is_not_full():
    # On a 16x16 grid the corner-to-corner distance^2 is 450; r = 21 (441) must drop that pair.
    M = oracle.clear_mask(0, 16, 16, 21)
    assert not M[0, 255] and not M[255, 0]
    # Only offsets (+-15, +-15) reach distance^2 450 >= 441: 4 ordered pairs are dropped.
    assert M.sum() == 256 * 256 - 4


# ------------------------------------------------------------------------------------------------
# Window size: lattice points of the open disc, ~ pi/4 of the square window.
# ------------------------------------------------------------------------------------------------

def _lattice_points_brute(r):
    return sum(1 for dy in range(-r, r + 1) for dx in range(-r, r + 1) if dx * dx + dy * dy < r * r)


@pytest.mark.parametrize("r", [1, 2, 3, 4, 5, 8, 16, 32])
def test_window_count_closed_form(r):
    n = oracle.window_lattice_count(r)
    assert n == _lattice_points_brute(r)
    # Gauss circle bound for the open disc of radius r.
    assert abs(n - math.pi * r * r) <= 2 * math.sqrt(2) * math.pi * r + 2 * math.pi


def test_window_counts_values_and_pi_over_4():
    counts = {r: oracle.window_lattice_count(r) for r in (4, 8, 16, 32)}
    assert counts == {4: 45, 8: 193, 16: 793, 32: 3205}
    fig = json.load(open(os.path.join(GOLDEN, "paper_figures.json")))
    assert fig["square_window_ratio"]["value"] == "pi/4"
    ratios = [counts[r] / (2 * r) ** 2 for r in (4, 8, 16, 32)]
    assert all(b > a for a, b in zip(ratios, ratios[1:]))  # increasing towards pi/4
    assert abs(oracle.window_lattice_count(256) / 512 ** 2 - math.pi / 4) < 5e-3


@pytest.mark.parametrize("r", [1, 3, 8])
def test_interior_mask_row_matches_lattice_count(r):
    n_text, H, W = 5, 2 * r + 3, 2 * r + 5
    y, x = H // 2, W // 2
    row = n_text + y * W + x
    M = oracle.clear_mask(n_text, H, W, r, rows=[row])
    assert M[0, :n_text].all()
    assert M[0, n_text:].sum() == _lattice_points_brute(r)


# ------------------------------------------------------------------------------------------------
# Kept pairs: closed form = explicit mask count; reproduces the printed 99.5 % at 8K.
# ------------------------------------------------------------------------------------------------

@pytest.mark.parametrize("n_text,H,W,r", [(0, 7, 9, 3), (4, 16, 16, 4), (3, 10, 5, 6), (2, 4, 4, 30)])
def test_kept_pairs_equals_mask_sum(n_text, H, W, r):
    assert oracle.kept_pairs(n_text, H, W, r) == int(oracle.clear_mask(n_text, H, W, r).sum())


def test_paper_99_5_percent_reduction_at_8k():
    fig = json.load(open(os.path.join(GOLDEN, "paper_figures.json")))["attention_reduction_8k"]
    wl = fig["workload"]
    assert wl["pixels"] // wl["patch_px"] == wl["grid"]
    G, n_text, r = wl["grid"], wl["n_text"], wl["r"]
    T = n_text + G * G
    kept = oracle.kept_pairs(n_text, G, G, r)
    reduction = 100.0 * (1.0 - kept / T ** 2)
    assert abs(reduction - fig["value_percent"]) <= fig["printed_precision_percent"]
    # The text accounting matters: without global text rows the figure would not round to 99.5.
    no_text_rows = 100.0 * (1.0 - (kept - n_text * T) / T ** 2)
    assert abs(no_text_rows - fig["value_percent"]) > fig["printed_precision_percent"]


# ------------------------------------------------------------------------------------------------
# Brute force: an independent per-query loop (window lists, no matrix mask) on tiny grids.
# ------------------------------------------------------------------------------------------------

def _brute_force_forward(q, k, v, n_text, H, W, r):
    B, Hh, T, d = q.shape
    scale = 1.0 / math.sqrt(d)
    O = np.zeros_like(q)
    LSE = np.zeros((B, Hh, T))
    for b in range(B):
        for h in range(Hh):
            for i in range(T):
                if i < n_text:
                    keys = list(range(T))
                else:
                    yi, xi = divmod(i - n_text, W)
                    keys = list(range(n_text))
                    for yj in range(H):
                        for xj in range(W):
                            if (yi - yj) ** 2 + (xi - xj) ** 2 < r * r:
                                keys.append(n_text + yj * W + xj)
                s = np.array([float(np.dot(q[b, h, i], k[b, h, j])) * scale for j in keys])
                m = s.max()
                e = np.exp(s - m)
                O[b, h, i] = (e[:, None] * v[b, h, keys]).sum(0) / e.sum()
                LSE[b, h, i] = m + math.log(e.sum())
    return O, LSE


@pytest.mark.parametrize("n_text", [0, 1, 5])
@pytest.mark.parametrize("H,W", [(4, 4), (3, 8), (8, 5)])
def test_brute_force_tiny_grids(n_text, H, W):
    d = 8
    T = n_text + H * W
    q, k, v = (_rand((1, 1, T, d), s) for s in (10, 11, 12))
    for r in range(1, 13):
        O, LSE = oracle.clear_attention_forward(q, k, v, n_text, H, W, r)
        Ob, LSEb = _brute_force_forward(q, k, v, n_text, H, W, r)
        np.testing.assert_allclose(O, Ob, rtol=0, atol=1e-12)
        np.testing.assert_allclose(LSE, LSEb, rtol=0, atol=1e-12)


# ------------------------------------------------------------------------------------------------
# Special cases.
# ------------------------------------------------------------------------------------------------

def test_r1_image_rows_see_text_and_self_only():
    n_text, H, W, d = 3, 4, 5, 8
    T = n_text + H * W
    q, k, v = (_rand((1, 1, T, d), s) for s in (20, 21, 22))
    O, _ = oracle.clear_attention_forward(q, k, v, n_text, H, W, 1)
    for i in range(n_text, T):
        keys = list(range(n_text)) + [i]
        ref, _ = _dense_softmax_attention(q[0, 0, i:i + 1], k[0, 0, keys], v[0, 0, keys], 1 / math.sqrt(d))
        np.testing.assert_allclose(O[0, 0, i], ref[0], rtol=0, atol=1e-12)


def test_no_text_is_pure_neighbourhood_attention():
    H, W, d, r = 6, 7, 8, 2
    q, k, v = (_rand((1, 1, H * W, d), s) for s in (30, 31, 32))
    O, _ = oracle.clear_attention_forward(q, k, v, 0, H, W, r)
    for i in range(H * W):
        yi, xi = divmod(i, W)
        keys = [yj * W + xj for yj in range(H) for xj in range(W)
                if (yi - yj) ** 2 + (xi - xj) ** 2 < r * r]
        assert len(keys) <= 9  # r = 2 keeps at most the 3 x 3 block around the query
        ref, _ = _dense_softmax_attention(q[0, 0, i:i + 1], k[0, 0, keys], v[0, 0, keys], 1 / math.sqrt(d))
        np.testing.assert_allclose(O[0, 0, i], ref[0], rtol=0, atol=1e-12)


def test_text_rows_are_dense_over_all_tokens():
    n_text, H, W, d, r = 4, 5, 5, 8, 2
    T = n_text + H * W
    q, k, v = (_rand((1, 1, T, d), s) for s in (40, 41, 42))
    O, LSE = oracle.clear_attention_forward(q, k, v, n_text, H, W, r)
    ref, ref_lse = _dense_softmax_attention(q[0, 0, :n_text], k[0, 0], v[0, 0], 1 / math.sqrt(d))
    np.testing.assert_allclose(O[0, 0, :n_text], ref, rtol=0, atol=1e-12)
    np.testing.assert_allclose(LSE[0, 0, :n_text], ref_lse, rtol=0, atol=1e-12)


def test_strict_radius_excludes_distance_exactly_r():
    # (dx, dy) = (3, 4) has distance exactly 5: excluded at r = 5, included at r = 6.
    n_text, H, W = 0, 6, 6
    i = 0
    j = 4 * W + 3
    assert not oracle.clear_mask(n_text, H, W, 5, rows=[i])[0, j]
    assert oracle.clear_mask(n_text, H, W, 6, rows=[i])[0, j]


# ------------------------------------------------------------------------------------------------
# Metamorphic relations.
# ------------------------------------------------------------------------------------------------

def _grid_perm_transpose(n_text, H, W):
    """Token permutation taking an H x W layout to its W x H transpose."""
    perm = list(range(n_text))
    for yt in range(W):          # transposed grid has H' = W rows, W' = H columns
        for xt in range(H):
            perm.append(n_text + xt * W + yt)
    return np.array(perm)


def test_transpose_grid():
    n_text, H, W, d, r = 3, 5, 8, 8, 3
    T = n_text + H * W
    q, k, v = (_rand((1, 2, T, d), s) for s in (50, 51, 52))
    O, LSE = oracle.clear_attention_forward(q, k, v, n_text, H, W, r)
    p = _grid_perm_transpose(n_text, H, W)
    Ot, LSEt = oracle.clear_attention_forward(q[:, :, p], k[:, :, p], v[:, :, p], n_text, W, H, r)
    np.testing.assert_allclose(Ot, O[:, :, p], rtol=0, atol=1e-12)
    np.testing.assert_allclose(LSEt, LSE[:, :, p], rtol=0, atol=1e-12)


def test_translation_interior_invariance():
    # Embed a 12x12 image grid into a 20x18 grid; queries at least r from the embedded border
    # (no key outside the small grid in their window) give the same outputs. No text tokens.
    r, d = 3, 8
    Hs, Ws, Hb, Wb, oy, ox = 12, 12, 20, 18, 5, 4
    kb = _rand((1, 1, Hb * Wb, d), 61)
    vb = _rand((1, 1, Hb * Wb, d), 62)
    qb = _rand((1, 1, Hb * Wb, d), 60)
    idx = np.array([(oy + y) * Wb + (ox + x) for y in range(Hs) for x in range(Ws)])
    Ob, _ = oracle.clear_attention_forward(qb, kb, vb, 0, Hb, Wb, r)
    Os, _ = oracle.clear_attention_forward(qb[:, :, idx], kb[:, :, idx], vb[:, :, idx], 0, Hs, Ws, r)
    for y in range(r - 1, Hs - r + 1):
        for x in range(r - 1, Ws - r + 1):
            np.testing.assert_allclose(Os[0, 0, y * Ws + x], Ob[0, 0, idx[y * Ws + x]], rtol=0, atol=1e-12)


def test_text_permutation_equivariance():
    n_text, H, W, d, r = 6, 4, 6, 8, 2
    T = n_text + H * W
    q, k, v = (_rand((1, 1, T, d), s) for s in (70, 71, 72))
    O, _ = oracle.clear_attention_forward(q, k, v, n_text, H, W, r)
    perm = np.concatenate([np.random.default_rng(0).permutation(n_text), np.arange(n_text, T)])
    Op, _ = oracle.clear_attention_forward(q[:, :, perm], k[:, :, perm], v[:, :, perm], n_text, H, W, r)
    np.testing.assert_allclose(Op, O[:, :, perm], rtol=0, atol=1e-12)


# ------------------------------------------------------------------------------------------------
# Sampled rows agree with the full call.
# ------------------------------------------------------------------------------------------------

def test_rows_match_full():
    n_text, H, W, d, r = 5, 9, 11, 8, 4
    T = n_text + H * W
    q, k, v = (_rand((2, 2, T, d), s) for s in (80, 81, 82))
    O, LSE = oracle.clear_attention_forward(q, k, v, n_text, H, W, r)
    rows = [0, 4, 5, 17, 60, T - 1]
    Or, Lr = oracle.clear_attention_rows(q, k, v, n_text, H, W, r, 1, 0, rows)
    np.testing.assert_allclose(Or, O[1, 0, rows], rtol=0, atol=1e-13)
    np.testing.assert_allclose(Lr, LSE[1, 0, rows], rtol=0, atol=1e-13)


# ------------------------------------------------------------------------------------------------
# Backward: central finite differences of a scalar loss <dO, O>.
# ------------------------------------------------------------------------------------------------

def test_backward_finite_differences():
    n_text, H, W, d, r = 3, 4, 4, 8, 2
    T = n_text + H * W
    q, k, v, dO = (_rand((1, 1, T, d), s) for s in (90, 91, 92, 93))
    dq, dk, dv = oracle.clear_attention_backward(q, k, v, dO, n_text, H, W, r)

    def loss(q_, k_, v_):
        O, _ = oracle.clear_attention_forward(q_, k_, v_, n_text, H, W, r)
        return float((O * dO).sum())

    eps = 1e-6
    rng = np.random.default_rng(1)
    for name, grad, which in (("q", dq, 0), ("k", dk, 1), ("v", dv, 2)):
        for _ in range(12):
            t, c = int(rng.integers(T)), int(rng.integers(d))
            args = [q.copy(), k.copy(), v.copy()]
            args[which][0, 0, t, c] += eps
            lp = loss(*args)
            args[which][0, 0, t, c] -= 2 * eps
            lm = loss(*args)
            fd = (lp - lm) / (2 * eps)
            assert abs(fd - grad[0, 0, t, c]) <= 1e-6 * max(1.0, abs(fd)), (name, t, c, fd, grad[0, 0, t, c])


def test_backward_matches_torch_autograd_full_radius():
    # With every pair kept, the analytic gradient must equal autograd through torch SDPA (fp64).
    n_text, H, W, d = 2, 3, 4, 8
    T = n_text + H * W
    r = 10
    q, k, v, dO = (_rand((1, 2, T, d), s) for s in (100, 101, 102, 103))
    dq, dk, dv = oracle.clear_attention_backward(q, k, v, dO, n_text, H, W, r)
    tq, tk, tv = (torch.from_numpy(a).requires_grad_() for a in (q, k, v))
    out = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv)
    out.backward(torch.from_numpy(dO))
    np.testing.assert_allclose(dq, tq.grad.numpy(), rtol=0, atol=1e-12)
    np.testing.assert_allclose(dk, tk.grad.numpy(), rtol=0, atol=1e-12)
    np.testing.assert_allclose(dv, tv.grad.numpy(), rtol=0, atol=1e-12)


def test_useful_flops_table():
    # Useful forward FLOPs = 4 d B h * kept pairs; spot-check the 512-grid r=8 figure (GFLOP).
    g = oracle.useful_flops_fwd(1, 24, 512, 512, 512, 8, 128) / 1e9
    assert abs(g - 3915.0) < 1.0
