"""Pins of the oracle's patch-parallel functions (stripe rows and the Eq. 7 patch-wise average)."""
import itertools

import numpy as np
import pytest
import torch

import oracle
from clear_inputs import Workload, make_inputs


def _inputs(n_text, H, W, d=16, heads=2, seed=0):
    wl = Workload("p", 1, heads, n_text, H, W, d, 3)
    return make_inputs(wl, seed=seed, dtype=torch.float32)


def test_single_patch_average_is_the_exact_text_rows():
    q, k, v = _inputs(5, 6, 7)
    O, _ = oracle.clear_attention_forward(q, k, v, 5, 6, 7, 3)
    A = oracle.clear_text_rows_patch_average(q, k, v, 5, 6, 7, [0, 6])
    assert np.abs(A - O[:, :, :5]).max() < 1e-12


def test_patch_average_brute_force_loops():
    # An independent formulation: per text query and per patch, a loop over the patch's keys.
    n_text, H, W, d = 3, 4, 3, 8
    q, k, v = (t.double().numpy() for t in _inputs(n_text, H, W, d=d, heads=1, seed=4))
    bounds = [0, 1, 3, 4]
    A = oracle.clear_text_rows_patch_average(q, k, v, n_text, H, W, bounds)
    for i in range(n_text):
        acc = np.zeros(d)
        for p in range(3):
            keys = list(range(n_text)) + [n_text + y * W + x for y in range(bounds[p], bounds[p + 1]) for x in range(W)]
            s = [float(q[0, 0, i] @ k[0, 0, j]) / np.sqrt(d) for j in keys]
            m = max(s)
            w = [np.exp(x - m) for x in s]
            acc += sum(wj * v[0, 0, j] for wj, j in zip(w, keys)) / sum(w)
        assert np.abs(acc / 3 - A[0, 0, i]).max() < 1e-12


def test_patch_average_depends_on_text_keys_in_each_patch():
    # Mutant reading (patches without the text tokens) differs: the pin above fixes the reading.
    n_text, H, W = 4, 4, 4
    q, k, v = _inputs(n_text, H, W, seed=2)
    A = oracle.clear_text_rows_patch_average(q, k, v, n_text, H, W, [0, 2, 4])
    qd, kd, vd = (t.double().numpy() for t in (q, k, v))
    M = np.zeros_like(A)
    for p, (a, b) in enumerate([(0, 2), (2, 4)]):
        cols = list(range(n_text + a * W, n_text + b * W))
        S = qd[:, :, :n_text] @ kd[:, :, cols].transpose(0, 1, 3, 2) / 4.0
        P = np.exp(S - S.max(-1, keepdims=True))
        M += (P / P.sum(-1, keepdims=True)) @ vd[:, :, cols] / 2
    assert np.abs(A - M).max() > 1e-3


def test_patch_average_identical_patches():
    # Two patches with identical image rows give the same softmax each: the average is that result.
    n_text, H, W = 3, 4, 5
    q, k, v = _inputs(n_text, H, W, seed=5)
    for t in (k, v):
        t[:, :, n_text + 2 * W:] = t[:, :, n_text:n_text + 2 * W]
    A = oracle.clear_text_rows_patch_average(q, k, v, n_text, H, W, [0, 2, 4])
    B1 = oracle.clear_text_rows_patch_average(q[:, :, :n_text + 2 * W], k[:, :, :n_text + 2 * W],
                                              v[:, :, :n_text + 2 * W], n_text, 2, W, [0, 2])
    assert np.abs(A - B1).max() < 1e-12


@pytest.mark.parametrize("window", ["circle", "square"])
def test_whole_stripe_is_the_forward(window):
    n_text, H, W, r = 4, 7, 6, 3
    q, k, v = _inputs(n_text, H, W)
    O, L = oracle.clear_attention_forward(q, k, v, n_text, H, W, r, window=window)
    Ot, Lt, Oi, Li = oracle.clear_attention_stripe(q, k, v, n_text, H, W, r, 0, H, 0, H, True, window=window)
    assert np.abs(Ot - O[:, :, :n_text]).max() < 1e-12 and np.abs(Oi - O[:, :, n_text:]).max() < 1e-12
    assert np.abs(Lt - L[:, :, :n_text]).max() < 1e-12 and np.abs(Li - L[:, :, n_text:]).max() < 1e-12


@pytest.mark.parametrize("bounds", [[0, 3, 7], [0, 2, 4, 7]])
def test_stripes_with_halos_merge_to_the_forward(bounds):
    # Each stripe: its rows plus r - 1 halo rows each side (clipped at the grid). Its image rows equal
    # the full forward's; text rows over disjoint key shares (text keys in the first share only)
    # merge by log-sum-exp weights into the full forward's text rows.
    n_text, H, W, r = 4, 7, 6, 3
    q, k, v = _inputs(n_text, H, W, seed=7)
    O, L = oracle.clear_attention_forward(q, k, v, n_text, H, W, r)
    qd, kd, vd = (t.double().numpy() for t in (q, k, v))
    parts = []
    for p in range(len(bounds) - 1):
        lo, hi = bounds[p], bounds[p + 1]
        top, bot = max(0, lo - (r - 1)), min(H, hi + (r - 1))
        cols = list(range(n_text)) + list(range(n_text + top * W, n_text + bot * W))
        Ot, Lt, Oi, Li = oracle.clear_attention_stripe(qd[:, :, cols], kd[:, :, cols], vd[:, :, cols], n_text,
                                                       bot - top, W, r, lo - top, hi - top, lo - top, hi - top, p == 0)
        assert np.abs(Oi - O[:, :, n_text + lo * W:n_text + hi * W]).max() < 1e-12
        parts.append((Ot, Lt))
    Ls = np.stack([pl for _, pl in parts])
    Lm = np.log(np.exp(Ls - Ls.max(0)).sum(0)) + Ls.max(0)
    Om = sum(np.exp(pl - Lm)[..., None] * po for po, pl in parts)
    assert np.abs(Om - O[:, :, :n_text]).max() < 1e-12 and np.abs(Lm - L[:, :, :n_text]).max() < 1e-12
