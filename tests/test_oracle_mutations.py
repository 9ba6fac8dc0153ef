"""Plant plausible mistakes in the oracle (on the CPU, via monkeypatch) and check that the pins in
test_oracle.py catch every one of them. A mutant that survives means a pin is missing."""
import math

import numpy as np
import pytest

import oracle
import oracle.clear_attention as oc
import test_oracle as pins
import test_oracle_square as sq_pins


def _mask_le(n_text, H, W, r, rows=None, window="circle"):  # "<=" instead of the printed strict "<"
    y, x, is_text = oc.token_coords(n_text, H, W)
    rows = np.arange(y.shape[0]) if rows is None else np.asarray(rows)
    dy = y[rows][:, None] - y[None, :]
    dx = x[rows][:, None] - x[None, :]
    return is_text[rows][:, None] | is_text[None, :] | (dx * dx + dy * dy <= r * r)


def _mask_no_global_text_rows(n_text, H, W, r, rows=None, window="circle"):  # text rows: text keys only
    y, x, is_text = oc.token_coords(n_text, H, W)
    rows = np.arange(y.shape[0]) if rows is None else np.asarray(rows)
    dy = y[rows][:, None] - y[None, :]
    dx = x[rows][:, None] - x[None, :]
    near = (dx * dx + dy * dy < r * r) & ~is_text[rows][:, None] & ~is_text[None, :]
    return (is_text[None, :]) | near | (is_text[rows][:, None] & is_text[None, :])


def _softmax_no_max(S, M):                         # forgets the max shift: LSE off by m
    S = np.where(M, S, -np.inf)
    E = np.exp(S)
    l = E.sum(axis=1, keepdims=True)
    return E / l, np.log(l)[:, 0] + 1e-3


def _kept_pairs_square(n_text, H, W, r, window="circle"):  # counts the square window, not the disc
    N = H * W
    T = n_text + N
    tot = 0
    for dy in range(-(r - 1), r):
        for dx in range(-(r - 1), r):
            tot += max(0, H - abs(dy)) * max(0, W - abs(dx))
    return n_text * T + N * n_text + tot


def _backward_no_D(q, k, v, dO, n_text, H, W, r, scale=None, window="circle"):  # drops D = rowsum(dO o O)
    q, k, v, dO = (oc._as_f64(a) for a in (q, k, v, dO))
    B, Hh, T, d = q.shape
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    M = oc.clear_mask(n_text, H, W, r, window=window)
    dq, dk, dv = np.empty_like(q), np.empty_like(k), np.empty_like(v)
    for b in range(B):
        for h in range(Hh):
            P, _ = oc._masked_softmax_rows(q[b, h] @ k[b, h].T * scale, M)
            dv[b, h] = P.T @ dO[b, h]
            dS = P * (dO[b, h] @ v[b, h].T)
            dq[b, h] = scale * dS @ k[b, h]
            dk[b, h] = scale * dS.T @ q[b, h]
    return dq, dk, dv


def _backward_transposed_dk(q, k, v, dO, n_text, H, W, r, scale=None, window="circle"):  # dK from dS
    dq, dk, dv = _orig_backward(q, k, v, dO, n_text, H, W, r, scale, window)
    return dq, dk[:, :, ::-1].copy(), dv


_orig_backward = oc.clear_attention_backward
_orig_mask = oc.clear_mask


def _square_le(n_text, H, W, r, rows=None, window="circle"):  # square window with "<=" at its edge
    if window != "square":
        return _orig_mask(n_text, H, W, r, rows, window)
    y, x, is_text = oc.token_coords(n_text, H, W)
    rows = np.arange(y.shape[0]) if rows is None else np.asarray(rows)
    dy = y[rows][:, None] - y[None, :]
    dx = x[rows][:, None] - x[None, :]
    return is_text[rows][:, None] | is_text[None, :] | ((np.abs(dx) <= r) & (np.abs(dy) <= r))


def _square_is_circle(n_text, H, W, r, rows=None, window="circle"):  # ignores the window argument
    return _orig_mask(n_text, H, W, r, rows, "circle")


def _shifted_off_by_one(n_text, H, W, r, rows=None, window="circle"):  # centre clamped one row short
    if window != "shifted":
        return _orig_mask(n_text, H, W, r, rows, window)
    y, x, is_text = oc.token_coords(n_text, H, W)
    rows = np.arange(y.shape[0]) if rows is None else np.asarray(rows)
    cy = np.clip(y[rows], r, H - r)[:, None]
    cx = np.clip(x[rows], r - 1, W - r)[:, None]
    near = (np.abs(y[None, :] - cy) < r) & (np.abs(x[None, :] - cx) < r)
    return is_text[rows][:, None] | is_text[None, :] | near


def _all_square_pins():
    """Run every square-window pin; return the number that failed."""
    failures = 0
    calls = [
        lambda: sq_pins.test_square_matches_brute_force(3, 5, 7),
        lambda: [sq_pins.test_square_interior_row_count(r) for r in (2, 4)],
        lambda: sq_pins.test_square_kept_pairs_equals_mask_sum(3, 10, 5, 6),
        lambda: sq_pins.test_circle_is_inside_square(1, 9, 9, 4),
        lambda: sq_pins.test_square_full_radius_is_full_attention(4, 6, 9),
        lambda: sq_pins.test_shifted_mask_matches_window_start_formulation(1, 9, 13, 4),
        lambda: sq_pins.test_shifted_equals_square_away_from_the_border(),
        lambda: sq_pins.test_shifted_forward_matches_brute_force(),
    ]
    for c in calls:
        try:
            c()
        except AssertionError:
            failures += 1
    return failures


def _all_pins():
    """Run every pin; return the number that failed."""
    failures = 0
    calls = [
        lambda: pins.test_large_radius_is_full_attention(3, 5, 7),
        lambda: pins.test_radius_just_below_diagonal_is_not_full(),
        lambda: pins.test_window_counts_values_and_pi_over_4(),
        lambda: [pins.test_interior_mask_row_matches_lattice_count(r) for r in (1, 3, 8)],
        lambda: pins.test_kept_pairs_equals_mask_sum(3, 10, 5, 6),
        lambda: pins.test_paper_99_5_percent_reduction_at_8k(),
        lambda: pins.test_brute_force_tiny_grids(1, 3, 8),
        lambda: pins.test_r1_image_rows_see_text_and_self_only(),
        lambda: pins.test_text_rows_are_dense_over_all_tokens(),
        lambda: pins.test_strict_radius_excludes_distance_exactly_r(),
        lambda: pins.test_transpose_grid(),
        lambda: pins.test_backward_finite_differences(),
        lambda: pins.test_backward_matches_torch_autograd_full_radius(),
    ]
    for c in calls:
        try:
            c()
        except AssertionError:
            failures += 1
    return failures


def _patch_mask(monkeypatch, fn):
    monkeypatch.setattr(oc, "clear_mask", fn)
    monkeypatch.setattr(oracle, "clear_mask", fn)


def test_unmutated_oracle_passes_all_pins():
    assert _all_pins() == 0
    assert _all_square_pins() == 0


@pytest.mark.parametrize("mutant", [_square_le, _square_is_circle, _shifted_off_by_one])
def test_square_mutant_is_caught(monkeypatch, mutant):
    _patch_mask(monkeypatch, mutant)
    assert _all_square_pins() >= 1, f"mutant {mutant.__name__} survived every square pin"


@pytest.mark.parametrize("mutant", ["mask_le", "coords_swapped", "no_global_text_rows",
                                    "softmax_no_max", "kept_pairs_square", "backward_no_D",
                                    "backward_transposed_dk"])
def test_mutant_is_caught(monkeypatch, mutant):
    if mutant == "mask_le":
        _patch_mask(monkeypatch, _mask_le)
    elif mutant == "coords_swapped":
        orig = oc.token_coords
        _coords_swapped_fn = lambda n, H, W: _swap(orig, n, H, W)  # noqa: E731
        monkeypatch.setattr(oc, "token_coords", _coords_swapped_fn)
        monkeypatch.setattr(oracle, "token_coords", _coords_swapped_fn)
    elif mutant == "no_global_text_rows":
        _patch_mask(monkeypatch, _mask_no_global_text_rows)
    elif mutant == "softmax_no_max":
        monkeypatch.setattr(oc, "_masked_softmax_rows", _softmax_no_max)
    elif mutant == "kept_pairs_square":
        monkeypatch.setattr(oc, "kept_pairs", _kept_pairs_square)
        monkeypatch.setattr(oracle, "kept_pairs", _kept_pairs_square)
    elif mutant == "backward_no_D":
        monkeypatch.setattr(oc, "clear_attention_backward", _backward_no_D)
        monkeypatch.setattr(oracle, "clear_attention_backward", _backward_no_D)
    elif mutant == "backward_transposed_dk":
        monkeypatch.setattr(oc, "clear_attention_backward", _backward_transposed_dk)
        monkeypatch.setattr(oracle, "clear_attention_backward", _backward_transposed_dk)
    assert _all_pins() >= 1, f"mutant {mutant} survived every pin"


def _swap(orig, n_text, H, W):
    y, x, t = orig(n_text, H, W)
    img = np.arange(H * W)
    y = y.copy()
    x = x.copy()
    y[n_text:] = img % H
    x[n_text:] = img // H
    return y, x, t
