"""The tile scheduler (the enumeration the kernels run, exposed by the host-only ABI queries) must
cover every kept (query, key) pair of the CLEAR mask exactly once and visit no useless tile. The
truth is the oracle's explicit mask."""
import itertools

import numpy as np
import pytest

import local_circular_window_b200 as L
import oracle

KQH, KQW, KKH, KKW, TILE = 8, 16, 4, 16, 128
KCHUNK = 64  # forward key tiles: 64-token chunks or 4 x 16 rectangles


def _keys_of_tile(tile, n_text, H, W, T):
    kind, a, b, flags = tile
    if kind == 0:
        return list(range(a, a + b))
    keys = []
    for y in range(a, a + KKH):
        for x in range(b, b + KKW):
            if 0 <= y < H and 0 <= x < W:
                keys.append(n_text + y * W + x)
    return keys


def _raw_keys_of_tile(tile, n_text, H, W):
    """All 128 slots of a tile, None where the slot is outside the grid / past the valid count."""
    kind, a, b, flags = tile
    if kind == 0:
        return [a + c if c < b else None for c in range(KCHUNK)]
    out = []
    for y in range(a, a + KKH):
        for x in range(b, b + KKW):
            out.append(n_text + y * W + x if (0 <= y < H and 0 <= x < W) else None)
    return out


def _queries_of_half(q_info, half, n_text, H, W):
    is_text, bh, q0, x0, valid_b = q_info
    if half == 1 and not valid_b:
        return []
    if is_text:
        start = q0 + half * TILE
        return [t for t in range(start, start + TILE) if t < n_text]
    y0 = q0 + half * KQH
    return [n_text + y * W + x for y in range(y0, y0 + KQH) for x in range(x0, x0 + KQW) if y < H and x < W]


CASES = [(16, 16, 16, 4), (0, 19, 21, 3), (5, 24, 40, 5), (3, 9, 17, 1), (200, 13, 50, 7), (1, 8, 8, 30),
         (0, 33, 47, 9), (7, 70, 18, 12), (130, 96, 96, 6), (300, 20, 20, 3)]
NEED = (1, 2)
FULL = (4, 8)


def _skip_unfit(window, H, W, r):
    if window == "shifted" and (2 * r - 1 > H or 2 * r - 1 > W):
        pytest.skip("the shifted window needs H, W >= 2r - 1")


@pytest.mark.parametrize("window", ["circle", "square", "shifted"])
@pytest.mark.parametrize("n_text,H,W,r", CASES)
def test_tiles_cover_mask_exactly(n_text, H, W, r, window):
    _skip_unfit(window, H, W, r)
    p = L.make_params(1, 1, n_text, H, W, 64, r, window)
    T = n_text + H * W
    n_txt_items, n_img_items, S, cps = L.forward_shape(p)
    M = oracle.clear_mask(n_text, H, W, r, window=window) if T <= 4000 else None
    text_cover = {}
    for item in range(n_txt_items + n_img_items):
        q_info, tiles = L.item_tiles(p, item)
        assert (item < n_txt_items) == bool(q_info[0])
        keys = [k for t in tiles for k in _keys_of_tile(t, n_text, H, W, T)]
        assert len(keys) == len(set(keys)), "a key is visited twice by one pair"
        for t in tiles:
            assert t[3] & 3, "union tile that neither half needs"
        if q_info[0]:
            text_cover.setdefault(q_info[2], []).extend(keys)
            assert all(t[0] == 0 for t in tiles)
        for half in (0, 1):
            queries = _queries_of_half(q_info, half, n_text, H, W)
            if not queries:
                assert not any(t[3] & NEED[half] for t in tiles)
                continue
            rows = M[queries] if M is not None else oracle.clear_mask(n_text, H, W, r, rows=queries, window=window)
            need = set(np.nonzero(rows.any(axis=0))[0].tolist())
            covered = set(k for t in tiles if t[3] & NEED[half] for k in _keys_of_tile(t, n_text, H, W, T))
            if not q_info[0]:  # a text split covers its own key range only (checked across splits below)
                assert need <= covered, "a kept pair of this half is not covered"
            for t in tiles:
                slots = _raw_keys_of_tile(t, n_text, H, W)
                real = [s_ for s_ in slots if s_ is not None]
                kept = rows[:, real]
                assert bool(t[3] & NEED[half]) == bool(kept.any()), ("need flag wrong", half, t)
                full = all(s_ is not None for s_ in slots) and kept.all()
                if t[3] & NEED[half]:
                    assert bool(t[3] & FULL[half]) == full, ("full flag wrong", half, t)
    # Text query pairs: the splits of one pair cover every token exactly once.
    for q0, keys in text_cover.items():
        assert sorted(keys) == list(range(T))


@pytest.mark.parametrize("window", ["circle", "square", "shifted"])
@pytest.mark.parametrize("n_text,H,W,r", CASES[:6])
def test_pair_counts(n_text, H, W, r, window):
    _skip_unfit(window, H, W, r)
    p = L.make_params(2, 3, n_text, H, W, 64, r, window)
    useful, executed = L.pair_counts(p)
    assert useful == 6 * oracle.kept_pairs(n_text, H, W, r, window)
    assert executed >= useful
    n_txt_items, n_img_items, S, cps = L.forward_shape(p)
    products = 0
    for i in range(n_txt_items + n_img_items):
        products += sum(((t[3] & 1) != 0) + ((t[3] & 2) != 0) for t in L.item_tiles(p, i)[1])
    assert executed == products * TILE * KCHUNK


def test_radius_beyond_diagonal_is_clamped_to_full_attention():
    # r larger than the grid diagonal keeps every pair; the scheduler clamps it and visits every key.
    p = L.make_params(1, 1, 16, 16, 16, 64, 1000)
    useful, executed = L.pair_counts(p)
    T = 16 + 256
    assert useful == T * T


@pytest.mark.parametrize("r,full", [(1000, True), (16, True), (15, False)])
def test_square_radius_clamp(r, full):
    # The square keeps every pair once r >= max(H, W) (here 16 x 12); r = 15 drops the far corners.
    p = L.make_params(1, 1, 8, 16, 12, 64, r, "square")
    useful, _ = L.pair_counts(p)
    T = 8 + 16 * 12
    assert (useful == T * T) == full
    assert useful == oracle.kept_pairs(8, 16, 12, min(r, 16), "square")


def test_split_shape_at_8k():
    p = L.make_params(1, 24, 512, 512, 512, 128, 8)
    n_txt_items, n_img_items, S, cps = L.forward_shape(p)
    assert n_img_items == 24 * (512 // 16) * (512 // 16)
    assert S * cps >= (512 + 512 * 512 + 63) // 64 and S <= 32
    assert n_txt_items == 24 * 2 * S
